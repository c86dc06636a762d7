"""Expert parallelism, world size 2 over gloo on the CPU: the dispatch and
combine bookkeeping of quantized_rl_fine_b200.ep against the oracle.

Each rank owns half of the experts and routes its own share of one batch
(oracle routing). The ranks exchange their per-expert row counts and rows with
ep.exchange_counts / ep.exchange_rows (gloo all-to-all), each owner reorders
what it received to local expert-major order (the definition in
tests/_ep_reference.py, which the GPU kernel is checked against), runs its own
experts with the oracle, reorders back, and the rows return by the reverse
exchange. Each rank's combined y must equal the oracle's single-process layer
on its tokens (float64, exact mode: only the order in which the float64
matrix products sum differs, so within 1e-12). The GPU transport is NCCL; it
has not run on more than one GPU here.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from quantized_rl_fine_b200 import dp, ep, synth
from quantized_rl_fine_b200.configs import MoEConfig

import _ep_reference as ref

CFG = MoEConfig("ep_tiny_int4", E=8, k=3, d=64, f=64, T=40, fmt="int4", swiglu=True,
                logits="normal", adapter=False, train=False, seed=3201)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    wl = synth.make_workload(CFG, "cpu")

    def qw(w):
        sc = w.scales.view(torch.int16).numpy().view(np.uint16) if w.fmt == "int4" else w.scales.numpy()
        return O.QWeight(w.fmt, w.packed.numpy(), sc)

    return dict(x=wl["x"].float().numpy().astype(np.float64), logits=wl["logits"].numpy(),
                w_gu=qw(wl["w_gu"]), w_d=qw(wl["w_d"]))


def _local(w, lo, hi):
    return O.QWeight(w.fmt, w.packed[lo:hi], w.scales[lo:hi])


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=20))
    try:
        inp = _inputs()
        t0, t1 = dp.token_shard(CFG.T, rank, world)
        x, logits = inp["x"][t0:t1], inp["logits"][t0:t1]
        T = t1 - t0
        # phase 1: route this rank's tokens over all experts
        topk, gates = O.route_topk(logits, CFG.k)
        g = O.group_by_expert(topk, CFG.E, CFG.chunk_size)
        x_perm = O.permute_rows(x, g)
        send = ep.send_splits(g.offsets, CFG.E, world)
        counts = torch.as_tensor(np.diff(g.offsets), dtype=torch.int32)
        recv_counts = ep.exchange_counts(counts, world)
        recv = recv_counts.sum(dim=1).tolist()
        rows = ep.exchange_rows(torch.from_numpy(x_perm), send, recv).numpy()
        # phase 2 on the owner: regroup, own experts, regroup back
        lo, hi = ep.expert_range(CFG.E, world, rank)
        order = ref.expert_major_order(recv_counts.numpy())
        offs, active, _ = ref.local_tables(recv_counts.numpy(), CFG.chunk_size)
        xl = rows[order]
        row_expert = np.repeat(np.arange(hi - lo), np.diff(offs))
        h, _ = O.grouped_gemm_fwd(xl, row_expert, _local(inp["w_gu"], lo, hi), O.EPI_SWIGLU, exact=True)
        yl, _ = O.grouped_gemm_fwd(h, row_expert, _local(inp["w_d"], lo, hi), O.EPI_NONE, exact=True)
        back = np.empty_like(yl)
        back[order] = yl
        # phase 3: the rows come home; combine this rank's tokens
        y_perm = ep.exchange_rows(torch.from_numpy(back), recv, send).numpy()
        y = O.combine(y_perm, g.inv_perm, gates, T, CFG.k, exact=True)
        want = O.moe_forward(x, logits, CFG.k, CFG.chunk_size, inp["w_gu"], inp["w_d"], exact=True)["y"]
        out[rank] = float(np.abs(y - want).max())
    except Exception as e:  # reported to the parent
        out[rank] = repr(e)
    finally:
        dist.destroy_process_group()


def test_expert_parallel_forward_matches_the_oracle():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert isinstance(out[r], float) and out[r] <= 1e-12, f"rank {r}: {out[r]}"


def test_expert_ranges_and_splits():
    assert ep.expert_range(384, 8, 0) == (0, 48) and ep.expert_range(384, 8, 7) == (336, 384)
    with pytest.raises(ValueError):
        ep.expert_range(10, 4, 0)
    off = [0, 3, 3, 7, 9, 9, 12, 12, 20]          # 8 experts
    assert ep.send_splits(off, 8, 2) == [9, 11] and ep.send_splits(off, 8, 4) == [3, 6, 3, 8]


def test_reference_regroup_by_brute_force():
    rng = np.random.default_rng(3)
    counts = rng.integers(0, 4, size=(3, 5))
    counts[1, 2] = 0
    s, e = ref.labels(counts)
    order = ref.expert_major_order(counts)
    # brute force: visit experts, then sources, then the source's rows in order
    want = []
    start = np.concatenate([[0], np.cumsum(counts.reshape(-1))])
    for ee in range(5):
        for ss in range(3):
            j = ss * 5 + ee
            want.extend(range(start[j], start[j + 1]))
    assert order.tolist() == want
    assert np.all(np.diff(e[order]) >= 0)
    offs, active, chunks = ref.local_tables(counts, 2)
    assert offs[-1] == counts.sum() and list(active) == [i for i in range(5) if counts[:, i].sum() > 0]
