"""The GEMM kernels' failure path, made to run without faulting the GPU.

Every pipeline wait of the grouped GEMM is bounded by a cycle budget. When a
wait runs out, the kernel records MOE_DEVERR_WAIT_TIMEOUT in the device error
word, lets the copies and MMAs it already issued finish, frees its tensor
memory and returns; the host reads the word with moe_get_device_error. Here
the budget is shrunk to a few hundred cycles, so ordinary waits of a GEMM
whose tiles take tens of microseconds run out. Then the default budget is
restored and the same GEMM must run clean and give the same bits as before.
"""

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import moeq, synth
from quantized_rl_fine_b200.configs import TRILLION_INT4

from _common import assert_close_intermediate, f64, oracle_qweight

pytestmark = pytest.mark.gpu

# d = 7168 gives 56 reduction steps per tile: the epilogue's first wait for an
# accumulator lasts far longer than one suspended try-wait (a few microseconds).
CFG = TRILLION_INT4.with_(name="wait_budget_case", E=4, k=2, f=256, T=64, seed=77)


def _gemm(wl, r):
    h, _ = moeq.moe_grouped_qgemm_fwd(r.x_perm, wl["w_gu"], r, moeq.EPI_SWIGLU)
    return h


def test_wait_timeout_is_reported_and_the_next_call_is_clean():
    wl = synth.make_workload(CFG, "cuda")
    r = moeq.moe_route_permute(wl["logits"], wl["x"], CFG.k, CFG.chunk_size)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
    h_ref = _gemm(wl, r).clone()
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
    try:
        moeq.moe_test_set_wait_budget(200)
        _gemm(wl, r)
        code = moeq.moe_get_device_error()      # synchronizes, reads and clears
    finally:
        moeq.moe_test_set_wait_budget(0)        # the default budget again
    assert code == moeq.DEVERR_WAIT_TIMEOUT
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE   # cleared by the read
    h = _gemm(wl, r)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
    assert torch.equal(h, h_ref)
    # and the bits are the layer's: against the oracle on the same rows
    rows = r.perm_token.cpu().numpy()
    off = r.expert_offsets.cpu().numpy()
    row_expert = np.repeat(np.arange(CFG.E), np.diff(off))
    want, _ = O.grouped_gemm_fwd(f64(wl["x"])[rows], row_expert, oracle_qweight(wl["w_gu"]),
                                 O.EPI_SWIGLU)
    assert_close_intermediate(f64(h), want, "h after the timeout")
