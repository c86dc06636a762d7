"""Reference of the expert-parallel row reordering, written from its
definition (test infrastructure).

A rank that owns E_loc experts receives, from each source rank s in turn, the
source's rows of each of its experts e in turn (source-major). Local
expert-major order sorts those rows by (expert, source), keeping each
source's own order: a stable sort of the source-major rows by the key
e * W + s.
"""

import numpy as np


def labels(counts):
    """(source, expert) of every received row, in source-major order."""
    counts = np.asarray(counts, dtype=np.int64)
    W, E_loc = counts.shape
    s = np.repeat(np.repeat(np.arange(W), E_loc), counts.reshape(-1))
    e = np.repeat(np.tile(np.arange(E_loc), W), counts.reshape(-1))
    return s, e


def expert_major_order(counts):
    """order[i] = the source-major index of the row at local expert-major position i."""
    counts = np.asarray(counts, dtype=np.int64)
    W = counts.shape[0]
    s, e = labels(counts)
    return np.argsort(e * W + s, kind="stable")


def local_tables(counts, chunk_size):
    """Local expert offsets, active experts and chunk offsets of the regrouped rows."""
    tot = np.asarray(counts, dtype=np.int64).sum(axis=0)
    offsets = np.concatenate([[0], np.cumsum(tot)])
    active = np.nonzero(tot)[0]
    nch = -(-active.shape[0] // chunk_size)
    chunk_offsets = np.minimum(np.arange(nch + 1) * chunk_size, active.shape[0])
    return offsets, active, chunk_offsets
