"""Parity of the CUDA library (through the C ABI) with the CPU oracle.

Bit-exact: dequantized weights, top-k indices, offsets, active list, chunk
table, permutation and permuted rows. BF16 outputs that end the computation:
max-abs <= 2e-2 and rel-L2 <= 5e-3 against the oracle (the workload's
criterion); per-slot intermediates: |err| <= 2e-2 + one BF16 ulp.
"""

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import layer, moeq, synth
from quantized_rl_fine_b200.configs import MXFP4_UP, TINY_INT4, MoEConfig

from _common import (assert_close_final, assert_close_intermediate, bf16_bits, f64,
                     oracle_qweight)

pytestmark = pytest.mark.gpu

DEV = "cuda"

TINY_TRAIN = MoEConfig("tiny_train_int4_adapter", E=8, k=2, d=256, f=256, T=96, fmt="int4",
                       swiglu=True, logits="normal", adapter=True, train=True, seed=2001)
RAGGED_MX = MoEConfig("ragged_mxfp4", E=5, k=3, d=128, f=192, T=37, fmt="mxfp4", swiglu=True,
                      logits="normal", adapter=True, train=True, seed=2002, chunk_size=2)
# About 150 rows per expert: the backward plans 192-row token tiles (one tile
# of 160 or more rows per expert), wider than any forward tile.
WIDE = MoEConfig("wide_int4", E=4, k=2, d=256, f=256, T=300, fmt="int4", swiglu=True,
                 logits="normal", adapter=True, train=True, seed=2003)
# More than 128 rows per expert: the forward takes the wide-tile plan (one
# token tile of up to 384 rows per expert, two MMAs per K step past 192 rows).
# About 256 rows per expert (one tile each, 192 + 64 columns), and about 500
# (two tiles, 384 + the rest), MXFP4 with a 192-long down reduction.
WIDE_FWD = MoEConfig("wide_fwd_int4", E=4, k=2, d=256, f=256, T=512, fmt="int4", swiglu=True,
                     logits="normal", adapter=True, train=True, seed=2004)
WIDE_MX = MoEConfig("wide_fwd_mxfp4", E=2, k=1, d=128, f=192, T=1000, fmt="mxfp4", swiglu=True,
                    logits="normal", adapter=False, train=True, seed=2005)


def _to(wl, dev):
    out = {}
    for key, v in wl.items():
        if isinstance(v, torch.Tensor):
            out[key] = v.to(dev)
        elif isinstance(v, synth.QWeightT):
            out[key] = v.to(dev)
        else:
            out[key] = v
    return out


def _gpu_workload(cfg, T=None):
    return _to(synth.make_workload(cfg, "cpu", T=T), DEV)


# ----------------------------------------------------------------------------- dequant

def test_dequant_int4_exhaustive_bit_exact():
    # every code x every BF16 scale bit pattern (65536 rows, 64 elements each)
    R, K = 65536, 64
    codes = np.tile(np.arange(16, dtype=np.uint8), K // 16)
    row = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    packed = np.tile(row, (R, 1))
    scales = np.tile(np.arange(R, dtype=np.uint16), (K // 32, 1))          # [K/32, R]
    got = moeq.moe_test_dequant(torch.from_numpy(packed).to(DEV),
                                torch.from_numpy(scales.view(np.int16)).to(DEV).view(torch.bfloat16),
                                "int4")
    want = O.dequant_int4_rows(packed, scales.T)
    g = bf16_bits(got)
    w = O.bf16_bits_from_values(want)
    nan_both = np.isnan(want) & np.isnan(f64(got))
    assert np.array_equal(g[~nan_both], w[~nan_both])
    assert np.array_equal(np.isnan(want), np.isnan(f64(got)))


def test_dequant_mxfp4_exhaustive_bit_exact():
    R, K = 256, 64
    codes = np.tile(np.arange(16, dtype=np.uint8), K // 16)
    row = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    packed = np.tile(row, (R, 1))
    scales = np.tile(np.arange(R, dtype=np.uint8), (K // 32, 1))
    got = moeq.moe_test_dequant(torch.from_numpy(packed).to(DEV), torch.from_numpy(scales).to(DEV),
                                "mxfp4")
    want = O.dequant_mxfp4_rows(packed, scales.T)
    gv = f64(got)
    nan_both = np.isnan(want) & np.isnan(gv)
    assert np.array_equal(np.isnan(want), np.isnan(gv))
    assert np.array_equal(bf16_bits(got)[~nan_both], O.bf16_bits_from_values(want)[~nan_both])


# ----------------------------------------------------------------------------- routing

def _check_routing(r: moeq.Routing, logits, x, k, C, E):
    topk, gates = O.route_topk(logits.cpu().numpy(), k)
    g = O.group_by_expert(topk, E, C)
    assert np.array_equal(r.topk_idx.cpu().numpy(), topk)
    assert np.allclose(r.gates.cpu().numpy(), gates, rtol=2e-6, atol=1e-7)
    assert np.array_equal(r.expert_offsets.cpu().numpy(), g.offsets)
    A = int(r.num_active.item())
    assert A == g.num_active
    assert np.array_equal(r.active.cpu().numpy()[:A], g.active)
    nch = int(r.num_chunks.item())
    assert nch == g.num_chunks
    assert np.array_equal(r.chunk_offsets.cpu().numpy()[:nch + 1], g.chunk_offsets)
    assert np.array_equal(r.perm_token.cpu().numpy(), g.perm_token)
    assert np.array_equal(r.inv_perm.cpu().numpy(), g.inv_perm)
    if x is not None and r.x_perm is not None:
        xp = r.x_perm.cpu().view(torch.int16).numpy()
        assert np.array_equal(xp, x.cpu().view(torch.int16).numpy()[g.perm_token])
    return g


@pytest.mark.parametrize("T,E,k,C", [(1, 4, 4, 1), (37, 5, 3, 2), (64, 8, 2, 8), (1000, 64, 4, 16),
                                     (130, 384, 8, 32), (4097, 256, 8, 8)])
def test_route_permute_bit_exact(T, E, k, C):
    g = torch.Generator().manual_seed(T * 7 + E)
    logits = torch.randn((T, E), generator=g)
    logits[: T // 3] = torch.round(logits[: T // 3] * 2) / 2          # many exact ties
    x = torch.randn((T, 64), generator=g).to(torch.bfloat16)
    r = moeq.moe_route_permute(logits.to(DEV), x.to(DEV), k, C)
    torch.cuda.synchronize()
    _check_routing(r, logits, x, k, C, E)


@pytest.mark.parametrize("T,E,k,d", [(1500, 64, 4, 1032), (2048, 128, 8, 8)])
def test_route_permute_copies_rows_of_any_width(T, E, k, d):
    # More than 1024 tokens: the histogram path and its row copy (one warp per
    # token, 128 16-byte units a step), with a ragged last step (129 units)
    # and with a single unit per row.
    g = torch.Generator().manual_seed(T + d)
    logits = torch.randn((T, E), generator=g)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    r = moeq.moe_route_permute(logits.to(DEV), x.to(DEV), k, 8)
    torch.cuda.synchronize()
    _check_routing(r, logits, x, k, 8, E)


def test_route_uniform_logits_full_size():
    wl = _gpu_workload(MXFP4_UP)
    r = moeq.moe_route_permute(wl["logits"], wl["x"], MXFP4_UP.k, MXFP4_UP.chunk_size)
    torch.cuda.synchronize()
    _check_routing(r, wl["logits"], wl["x"], MXFP4_UP.k, MXFP4_UP.chunk_size, MXFP4_UP.E)


# ----------------------------------------------------------------------------- GEMMs

def _zero_sign_free(bits):
    # The sum of one exact term and zero products is exact, except that the
    # sign of a zero weight is lost (-0 + +0 = +0): compare zeros as equal.
    b = np.array(bits, dtype=np.uint16)
    b[b == 0x8000] = 0
    return b


def test_one_hot_probe_reads_weights_bit_exact():
    # a = e_k rows make out[:, n] = W[n, k] exactly: checks layout and placement
    # of the dequantized tile inside the real GEMM without writing it to memory.
    for fmt in ("int4", "mxfp4"):
        gen = torch.Generator().manual_seed(5)
        E, N, K = 3, 256, 192
        w = synth.random_qweight(gen, E, N, K, fmt, "cpu", std=0.5)
        kk = np.array([0, 1, 31, 32, 63, 64, 100, 191])
        rows_per_e = len(kk)
        M = E * rows_per_e
        a = torch.zeros((M, K), dtype=torch.bfloat16)
        logits = torch.full((M, E), -10.0)
        for e in range(E):
            for i, c in enumerate(kk):
                a[e * rows_per_e + i, c] = 1.0
                logits[e * rows_per_e + i, e] = 10.0
        r = moeq.moe_route_permute(logits.to(DEV), a.to(DEV), 1, 2)
        out = moeq.moe_grouped_qgemm_fwd(r.x_perm, w.to(DEV), r, moeq.EPI_NONE)
        ow = oracle_qweight(w)
        got = _zero_sign_free(bf16_bits(out))
        for e in range(E):
            W = O.dequant_expert(ow, e)
            for i, c in enumerate(kk):
                want = _zero_sign_free(O.bf16_bits_from_values(W[:, c]))
                assert np.array_equal(got[e * rows_per_e + i], want), (fmt, e, c)
        # backward orientation: d = e_n rows pick row n of W
        d = torch.zeros((M, N), dtype=torch.bfloat16)
        nn = np.array([0, 5, 63, 64, 200, 255, 128, 7])
        for e in range(E):
            for i, n in enumerate(nn):
                d[e * rows_per_e + i, n] = 1.0
        din = moeq.moe_grouped_qgemm_bwd_dx(d.to(DEV), w.to(DEV), r, moeq.EPI_NONE)
        got = _zero_sign_free(bf16_bits(din))
        for e in range(E):
            W = O.dequant_expert(ow, e)
            for i, n in enumerate(nn):
                want = _zero_sign_free(O.bf16_bits_from_values(W[n, :]))
                assert np.array_equal(got[e * rows_per_e + i], want), (fmt, e, n)


def _oracle_weights(wl):
    out = {}
    for key in ("w_gu", "w_d", "w_up"):
        if key in wl:
            out[key] = oracle_qweight(wl[key])
    return out


def _run_layer_and_compare(cfg, T=None, gather=None):
    wl = _gpu_workload(cfg, T)
    ow = _oracle_weights(wl)
    R = f64(wl["adapter"]) if cfg.adapter else None
    st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, cfg.chunk_size,
                       adapter=wl.get("adapter"), train=cfg.train, gather=gather)
    torch.cuda.synchronize()
    ref = O.moe_forward(f64(wl["x"]), wl["logits"].cpu().numpy(), cfg.k, cfg.chunk_size,
                        ow["w_gu"], ow["w_d"], R=R)
    _check_routing(st["routing"], wl["logits"], wl["x"], cfg.k, cfg.chunk_size, cfg.E)
    assert_close_intermediate(f64(st["h"]), ref["h"], "h")
    assert_close_intermediate(f64(st["y_perm"]), ref["y_perm"], "y_perm")
    assert_close_final(f64(st["y"]), ref["y"], "y")
    if cfg.train:
        assert_close_intermediate(f64(st["saved_gu"]), ref["saved_gu"], "saved_gu")
        bw = layer.backward(st, wl["dy"], wl["w_gu"], wl["w_d"], adapter=wl.get("adapter"))
        torch.cuda.synchronize()
        rb = O.moe_backward(ref, f64(wl["dy"]), ow["w_gu"], ow["w_d"], R=R)
        # The gate-scaled scatter rounds g * dy once to BF16: bit-exact given
        # the same gates. The kernel's gates match the oracle's only within
        # the routing check's 2e-6, and a one-ulp gate difference moves a few
        # products across a BF16 rounding boundary, so the expected rows are
        # the oracle's scatter of the kernel's gates.
        r = st["routing"]
        want = O.gather_scaled(f64(wl["dy"]), r.inv_perm.cpu().numpy(), r.gates.cpu().numpy(),
                               wl["dy"].shape[0], cfg.k)
        assert np.array_equal(bf16_bits(bw["dy_perm"]), O.bf16_bits_from_values(want))
        assert_close_intermediate(f64(bw["dgu"]), rb["dgu"], "dgu")
        assert_close_final(f64(bw["dx"]), rb["dx"], "dx")
        if cfg.adapter:
            assert_close_final(bw["d_adapter"].cpu().numpy().astype(np.float64), rb["d_adapter"],
                               "d_adapter")
    return st


@pytest.mark.parametrize("gather", [True, False], ids=["gathered_rows", "x_perm"])
def test_tiny_int4_layer_forward(gather):
    _run_layer_and_compare(TINY_INT4, gather=gather)


@pytest.mark.parametrize("gather", [True, False], ids=["gathered_rows", "x_perm"])
def test_tiny_train_forward_backward_with_adapter(gather):
    _run_layer_and_compare(TINY_TRAIN, gather=gather)


@pytest.mark.parametrize("gather", [True, False], ids=["gathered_rows", "x_perm"])
def test_ragged_mxfp4_train_with_adapter(gather):
    _run_layer_and_compare(RAGGED_MX, gather=gather)


@pytest.mark.parametrize("cfg", [TINY_INT4, TINY_TRAIN, RAGGED_MX, MXFP4_UP],
                         ids=["int4", "int4_train_adapter", "mxfp4_ragged", "mxfp4_up"])
def test_gathered_rows_give_the_bits_of_materialized_rows(cfg):
    """Reading row p as x[perm_token[p]] inside the kernels (no x_perm) and
    reading a materialized x_perm give bit-identical outputs, forward and
    backward."""
    wl = _gpu_workload(cfg)
    outs = []
    for gather in (True, False):
        if not cfg.swiglu:
            st = layer.up_projection(wl["x"], wl["logits"], wl["w_up"], cfg.k, cfg.chunk_size,
                                     gather=gather)
            outs.append((st["out"].clone(),))
            continue
        st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, cfg.chunk_size,
                           adapter=wl.get("adapter"), train=cfg.train, gather=gather)
        o = [st["y"].clone(), st["h"].clone()]
        if cfg.train:
            bw = layer.backward(st, wl["dy"], wl["w_gu"], wl["w_d"], adapter=wl.get("adapter"))
            o += [bw["dx"].clone()] + ([bw["d_adapter"].clone()] if cfg.adapter else [])
        outs.append(tuple(o))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


def test_single_token():
    _run_layer_and_compare(RAGGED_MX.with_(T=1, seed=2003))


def test_adapter_identity_is_bitwise_noop():
    wl = _gpu_workload(TINY_INT4)
    eye = torch.eye(32, dtype=torch.bfloat16, device=DEV).expand(TINY_INT4.E, TINY_INT4.d // 32, 32, 32).contiguous()
    a = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], 2, 8)
    b = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], 2, 8, adapter=eye)
    assert torch.equal(a["y"], b["y"])


def test_outputs_identical_across_chunk_sizes():
    cfg = TINY_TRAIN
    wl = _gpu_workload(cfg)
    ys = []
    for C in (1, 3, 8, 16, 32):
        st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, C,
                           adapter=wl["adapter"], train=True)
        bw = layer.backward(st, wl["dy"], wl["w_gu"], wl["w_d"], adapter=wl["adapter"])
        ys.append((st["y"].clone(), bw["dx"].clone(), bw["d_adapter"].clone()))
    for y, dx, da in ys[1:]:
        assert torch.equal(y, ys[0][0]) and torch.equal(dx, ys[0][1]) and torch.equal(da, ys[0][2])


def test_mxfp4_up_projection_full_size():
    """The bench workload at its full size: every output compared with the oracle."""
    cfg = MXFP4_UP
    wl = _gpu_workload(cfg)
    st = layer.up_projection(wl["x"], wl["logits"], wl["w_up"], cfg.k, cfg.chunk_size, gather=False)
    torch.cuda.synchronize()
    ref = O.up_projection(f64(wl["x"]), wl["logits"].cpu().numpy(), cfg.k, cfg.chunk_size,
                          oracle_qweight(wl["w_up"]))
    _check_routing(st["routing"], wl["logits"], wl["x"], cfg.k, cfg.chunk_size, cfg.E)
    assert_close_final(f64(st["out"]), ref["out"], "out")


def test_device_error_word_is_clear_after_runs():
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


# ----------------------------------------------------------------------------- every kernel variant

@pytest.mark.parametrize("lanes,bn", [(2, 16), (2, 48), (2, 96), (4, 16), (4, 48), (4, 64)])
@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX], ids=["int4", "mxfp4_ragged"])
def test_each_lane_count_and_tile_width_matches_the_oracle(monkeypatch, cfg, lanes, bn):
    """The planner picks one lane count per shape; this runs every pipeline
    variant (two or four lanes, forward and backward, both formats, with and
    without the K % 128 == 64 tail) at several token-tile widths on the same
    inputs and checks each against the oracle."""
    monkeypatch.setenv("MOEQ_LANES", str(lanes))
    monkeypatch.setenv("MOEQ_BN", str(bn))
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("bn", [None, "176", "192"], ids=["planned", "forced176", "forced192"])
def test_wide_token_tiles_match_the_oracle(monkeypatch, bn):
    """Token tiles wider than 96 rows: planned for the backward at about 150
    rows per expert, and forced for both directions (the forward then runs
    two tile pipelines with two A stages handed over in halves, as two
    accumulators of more than 128 columns leave room for only two)."""
    if bn is not None:
        monkeypatch.setenv("MOEQ_BN", bn)
    _run_layer_and_compare(WIDE)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("env", [{"MOEQ_HALVES": "1"}, {"MOEQ_HALVES": "1", "MOEQ_LANES": "4"},
                                 {"MOEQ_HALVES": "1", "MOEQ_PIPES": "0"}, {"MOEQ_DQW": "8"},
                                 {"MOEQ_DQW": "8", "MOEQ_HALVES": "1"}],
                         ids=["halves", "halves_4lanes", "halves_nopipes", "dqw8", "dqw8_halves"])
@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX], ids=["int4", "mxfp4_ragged"])
def test_a_stage_halves_and_dequant_warp_counts_match_the_oracle(monkeypatch, cfg, env):
    """The forward A stages handed over in 64-wide halves (two barriers per
    stage), with two or four lanes and with or without tile pipelines, and the
    eight-dequant-warp kernels, against the oracle (K % 128 == 64 tail
    included)."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("pipes", ["1", "0"], ids=["pipelines", "one_issuer"])
@pytest.mark.parametrize("cfg", [TINY_TRAIN, WIDE], ids=["int4", "wide_int4"])
def test_cta_pair_forward_matches_the_oracle(monkeypatch, cfg, pipes):
    """The CTA-pair forward kernels (clusters of two CTAs, M = 256 MMAs issued
    by the even CTA, each CTA holding half of the token rows), with two tile
    pipelines (and, at 192-row tiles, A stages handed over in halves) or one
    issuer, against the oracle; both shapes have an even number of feature
    tiles in both forward GEMMs, so every forward launch runs on pairs."""
    monkeypatch.setenv("MOEQ_PAIR", "1")
    monkeypatch.setenv("MOEQ_PIPES", pipes)
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX], ids=["int4", "mxfp4_ragged"])
def test_forward_without_tile_pipelines_matches_the_oracle(monkeypatch, cfg):
    """Two-lane forward kernels run as two tile pipelines by default (each
    issuer accumulates whole tiles); this runs them with every issuer taking
    every other fill of every tile instead, the layout the four-lane and the
    one-issuer plans use."""
    monkeypatch.setenv("MOEQ_PIPES", "0")
    monkeypatch.setenv("MOEQ_LANES", "2")
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX, WIDE], ids=["int4", "mxfp4_ragged", "wide_int4"])
def test_shared_memory_backward_matches_the_oracle(monkeypatch, cfg):
    """The backward GEMMs keep their A operand in tensor memory by default
    (128-wide fills, the dequantized rows transposed on the way); this runs
    the shared-memory form (64-wide fills, MN-major A; 192-row tiles from 128
    rows per expert on) against the oracle."""
    monkeypatch.setenv("MOEQ_BWD_SMEM_A", "1")
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX, WIDE], ids=["int4", "mxfp4_ragged", "wide_int4"])
def test_even_token_tile_split_matches_the_oracle(monkeypatch, cfg):
    """An expert's rows go to token tiles of BN rows and a shorter last one by
    default; this runs the equal-width split (every tile ceil(m / nrt) rows
    rounded up to 16) against the oracle."""
    monkeypatch.setenv("MOEQ_SPLIT", "even")
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [WIDE_FWD, WIDE_MX], ids=["int4_256_rows", "mxfp4_500_rows"])
def test_wide_token_tile_forward_matches_the_oracle(cfg):
    """The planned wide-tile forward (more than 128 rows per expert): token
    tiles of up to 384 rows, two MMAs per K step past 192 rows, 64-wide fills
    with 32-column A stages, one accumulator."""
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [TINY_TRAIN, RAGGED_MX, WIDE], ids=["int4", "mxfp4_ragged", "wide_int4"])
def test_forced_wide_plan_matches_the_oracle(monkeypatch, cfg):
    """The wide-tile forward forced on small shapes (token tiles of 16 to 240
    rows, one MMA per K step below 193 rows)."""
    monkeypatch.setenv("MOEQ_WIDE", "1")
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [RAGGED_MX, WIDE], ids=["mxfp4_ragged", "wide_int4"])
def test_forced_wide_plan_without_tile_pipelines_matches_the_oracle(monkeypatch, cfg):
    """The wide-tile forward with two issuers taking every other fill into
    partial accumulators (no tile pipelines; token rows and weights share the
    shared-memory stages)."""
    monkeypatch.setenv("MOEQ_WIDE", "1")
    monkeypatch.setenv("MOEQ_PIPES", "0")
    _run_layer_and_compare(cfg)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


@pytest.mark.parametrize("cfg", [WIDE_FWD, WIDE_MX], ids=["int4_256_rows", "mxfp4_500_rows"])
def test_wide_and_narrow_forward_give_the_same_bits(monkeypatch, cfg):
    """Every plan accumulates a token's column in the same K order, one MMA
    column per token: the wide-tile forward and the narrow one (96-row tiles,
    two tile pipelines) give bit-identical outputs."""
    wl = _gpu_workload(cfg)
    outs = []
    for env in ("1", "0"):
        monkeypatch.setenv("MOEQ_WIDE", env)
        st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, cfg.chunk_size,
                           adapter=wl.get("adapter"), train=cfg.train)
        outs.append((st["h"].clone(), st["y"].clone(), st["saved_gu"].clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
