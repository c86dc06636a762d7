"""The comparator of the temporary-buffer scheme (Orbit article,
"Active-expert-chunked dequantization"): its whole-expert dequantization is
bit-exact with the oracle's, and its layer output matches the oracle within
the final-output tolerance, so the timings it gives compare like with like."""

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import moeq, prior_art, synth
from quantized_rl_fine_b200.configs import MXFP4_UP, TINY_INT4

from _common import assert_close_final, bf16_bits, f64, oracle_qweight

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_dequant_experts_bit_exact(fmt):
    g = torch.Generator(device="cuda").manual_seed(31)
    w = synth.random_qweight(g, 5, 192, 256, fmt, "cuda")
    ids = torch.tensor([4, 0, 2, 2], dtype=torch.int32, device="cuda")
    got = bf16_bits(moeq.moe_dequant_experts(w, ids))
    ow = oracle_qweight(w)
    for i, e in enumerate(ids.tolist()):
        want = O.bf16_bits_from_values(O.dequant_expert(ow, e))
        assert np.array_equal(got[i], want), (fmt, i, e)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


def test_dequant_experts_rejects_a_foreign_id_in_the_error_word():
    g = torch.Generator(device="cuda").manual_seed(32)
    w = synth.random_qweight(g, 3, 64, 64, "int4", "cuda")
    out = moeq.moe_dequant_experts(w, torch.tensor([1, 7], dtype=torch.int32, device="cuda"))
    assert moeq.moe_get_device_error() == moeq.DEVERR_BAD_OFFSETS
    assert torch.count_nonzero(out[1]) == 0


@pytest.mark.parametrize("cfg,C", [(TINY_INT4, 3), (MXFP4_UP, 16)])
def test_prior_art_layer_matches_the_oracle(cfg, C):
    wl = synth.make_workload(cfg, "cuda")
    r = moeq.moe_route_permute(wl["logits"], wl["x"], cfg.k, C)
    first = wl["w_gu"] if cfg.swiglu else wl["w_up"]
    y_perm, peak = prior_art.forward(r.x_perm, r, first, wl.get("w_d"), C, swiglu=cfg.swiglu)
    if cfg.swiglu:
        ref = O.moe_forward(f64(wl["x"]), wl["logits"].cpu().numpy(), cfg.k, C,
                            oracle_qweight(wl["w_gu"]), oracle_qweight(wl["w_d"]))
        y = moeq.moe_unpermute_combine(y_perm, r, r.gates, cfg.T, mode=0)
        assert_close_final(f64(y), ref["y"], "prior-art y")
    else:
        ref = O.up_projection(f64(wl["x"]), wl["logits"].cpu().numpy(), cfg.k, C, oracle_qweight(first))
        assert_close_final(f64(y_perm), ref["out"], "prior-art out")
    # one chunk of dequantized weights is the bulk of the temporary memory
    per_expert = (first.N * first.K + (wl["w_d"].N * wl["w_d"].K if cfg.swiglu else 0)) * 2
    assert peak >= min(C, cfg.E) * first.N * first.K * 2
    assert peak < (min(C, cfg.E) + 1) * per_expert + 64 * 2 ** 20
