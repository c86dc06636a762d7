"""Batch invariance of the forward: a token's output bits do not depend on the
rest of the batch.

The Orbit article runs the same low-bit base + BF16 adapter for rollout and
for training, so that the two sides see the same numbers (its train/rollout
precision-alignment goal). Rollout batches are small (decode-like, a few rows
per expert) and training batches large (hundreds of rows per expert); the
kernels then pick different token-tile widths, pipeline-lane counts and tile
splits. Every plan accumulates a tile's whole reduction in one accumulator in
fill order, each output column of an MMA is its own dot product, and the
epilogues, the adapter and the combine work row by row, so the same token
must give the same bits. Here the first 128 tokens of one draw are run alone
and inside batches of 2048 and 16384 (and 4096 with the adapter), and their
outputs are compared bit for bit.
"""

import pytest
import torch

from quantized_rl_fine_b200 import layer, moeq, synth
from quantized_rl_fine_b200.configs import TRAIN_INT4, TRILLION_INT4

pytestmark = pytest.mark.gpu


def _first_rows(cfg, wl, T, n=128):
    st = layer.forward(wl["x"][:T].contiguous(), wl["logits"][:T].contiguous(), wl["w_gu"],
                       wl["w_d"], cfg.k, cfg.chunk_size, adapter=wl.get("adapter"))
    return st["y"][:n].clone()


def test_trillion_int4_forward_is_batch_invariant():
    cfg = TRILLION_INT4
    wl = synth.make_workload(cfg, "cuda", T=16384)
    ys = {T: _first_rows(cfg, wl, T) for T in (128, 2048, 16384)}
    assert torch.equal(ys[128], ys[2048])
    assert torch.equal(ys[128], ys[16384])
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


def test_forward_with_adapter_is_batch_invariant():
    cfg = TRAIN_INT4
    wl = synth.make_workload(cfg, "cuda", T=4096)
    ys = {T: _first_rows(cfg, wl, T) for T in (128, 4096)}
    assert torch.equal(ys[128], ys[4096])
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
