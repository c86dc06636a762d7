"""Pins of the CPU oracle against things other than itself (CPU only).

Hand-worked tables (tests/golden), closed forms, brute force on tiny inputs,
invariants, finite differences and the storage figures printed by the pages.
Each test is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign or index, a transposed operand, a wrong nibble or scale layout)
fails it.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import accounting, synth
from quantized_rl_fine_b200.configs import TINY_INT4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(tok: str) -> float:
    t = tok.strip()
    if t.lstrip("-").startswith("0x"):
        return float.fromhex(t)
    return float(t)


def _load_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, vals = line.split(":")
            rows.append((key.strip(), [_num(v) for v in vals.split()]))
    return rows


def _same_bf16(a, b):
    """Bitwise equality of BF16 values, any NaN equal to any NaN."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nan = np.isnan(a) & np.isnan(b)
    ba = O.bf16_bits_from_values(np.where(nan, 0, a))
    bb = O.bf16_bits_from_values(np.where(nan, 0, b))
    return bool(np.all((ba == bb) | nan)) and bool(np.all(np.isnan(a) == np.isnan(b)))


# --------------------------------------------------------------------------- bf16

def test_bf16_round_hand_cases():
    cases = [
        (1 + 2 ** -8, 1.0),                       # tie -> even (1.0000000)
        (1 + 3 * 2 ** -8, 1 + 2 ** -6),           # tie -> even (1.0000010)
        (1 + 2 ** -8 + 2 ** -30, 1 + 2 ** -7),    # just above the tie
        (2 ** -134, 0.0),                          # half the subnormal step -> even 0
        (3 * 2 ** -134, 2 ** -132),                # tie between 1 and 2 steps -> 2
        (5 * 2 ** -135, 2 ** -133),                # 1.25 steps -> 1 step
        (O.BF16_MAX + 2 ** 119, math.inf),         # tie with 2**128 -> even -> overflow
        (O.BF16_MAX + 2 ** 118, O.BF16_MAX),
        (-(1 + 3 * 2 ** -8), -(1 + 2 ** -6)),
        (-2 ** -140, -0.0),
        (0.1, float.fromhex("0x1.9ap-4")),     # 0.1 = 1.6 * 2**-4 -> 1.6015625
    ]
    for x, want in cases:
        got = O.bf16_round(np.array([x]))[0]
        assert _same_bf16(got, want), (x, got, want)


def test_bf16_round_matches_torch_on_float32_inputs():
    # For float32 inputs one rounding to BF16 is exactly torch's RNE conversion.
    g = torch.Generator().manual_seed(7)
    raw = torch.randint(0, 2 ** 32, (200000,), generator=g, dtype=torch.int64)
    f32 = raw.to(torch.int32).view(torch.float32)
    f32 = f32[torch.isfinite(f32)]
    ours = O.bf16_round(f32.numpy().astype(np.float64))
    ref = f32.to(torch.bfloat16).float().numpy().astype(np.float64)
    assert _same_bf16(ours, ref)


# --------------------------------------------------------------------------- dequant

def _row_of(code: int) -> np.ndarray:
    return np.full((1, 16), code | (code << 4), dtype=np.uint8)    # 32 elements, one group


def test_int4_dequant_hand_table():
    for scale_txt, values in _load_table("int4_dequant_table.txt"):
        s = float.fromhex(scale_txt)
        s_bits = O.bf16_bits_from_values(np.array([s]))
        assert O.bf16_values_from_bits(s_bits)[0] == s, "table scale must be a BF16 number"
        for code in range(16):
            w = O.dequant_int4_rows(_row_of(code), s_bits.reshape(1, 1))
            assert w.shape == (1, 32)
            assert _same_bf16(w, np.full(32, values[code])), (scale_txt, code, w[0, 0], values[code])


def test_mxfp4_dequant_hand_table():
    for x_txt, values in _load_table("mxfp4_dequant_table.txt"):
        X = np.array([[int(x_txt)]], dtype=np.uint8)
        for code in range(16):
            w = O.dequant_mxfp4_rows(_row_of(code), X)
            assert _same_bf16(w, np.full(32, values[code])), (x_txt, code, w[0, 0], values[code])


def test_nibble_order_low_nibble_is_even_element():
    packed = np.array([[0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE] * 2], dtype=np.uint8)
    codes = O.unpack_nibbles(packed)
    assert codes[0].tolist() == list(range(16)) * 2
    w = O.dequant_int4_rows(packed, O.bf16_bits_from_values(np.array([[1.0]])))
    assert w[0, :16].tolist() == [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1]


def test_scale_layout_is_group_major():
    # E=1, N=3 rows, K=96 (3 groups); every code 1, scale[g][n] = (n + 1) * 2**g.
    N, K = 3, 96
    packed = np.full((1, N, K // 2), 0x11, dtype=np.uint8)
    sc = np.array([[(n + 1) * 2.0 ** g for n in range(N)] for g in range(K // 32)])
    w = O.QWeight("int4", packed, O.bf16_bits_from_values(sc)[None])
    W = O.dequant_expert(w, 0)
    for n in range(N):
        for k in range(K):
            assert W[n, k] == (n + 1) * 2.0 ** (k // 32)


# --------------------------------------------------------------------------- routing

def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(0)
    for T, E, k in [(6, 5, 2), (9, 8, 3), (4, 7, 7), (5, 3, 1)]:
        logits = rng.integers(-2, 3, size=(T, E)).astype(np.float32)   # many ties
        logits[0, :] = 0.0
        logits[1, 0] = -0.0
        topk, gates = O.route_topk(logits, k)
        for t in range(T):
            # pure-Python selection: repeatedly take the largest, lowest id first
            left = list(range(E))
            want = []
            for _ in range(k):
                best = left[0]
                for e in left[1:]:
                    if logits[t, e] > logits[t, best]:
                        best = e
                want.append(best)
                left.remove(best)
            assert topk[t].tolist() == want


def test_gate_closed_forms():
    a, b = 1.25, -0.5
    _, g = O.route_topk(np.array([[a, b, -9.0]], np.float32), 2)
    want = 1.0 / (1.0 + math.exp(b - a))                     # logistic of the gap
    assert abs(g[0, 0] - want) < 1e-7 and abs(g[0, 1] - (1 - want)) < 1e-7
    _, g = O.route_topk(np.array([[3.0, 3.0, 3.0, 3.0]], np.float32), 4)
    assert np.allclose(g, 0.25, rtol=0, atol=1e-8)
    rng = np.random.default_rng(1)
    _, g = O.route_topk(rng.standard_normal((100, 16)).astype(np.float32), 5)
    assert np.all(np.abs(g.astype(np.float64).sum(1) - 1) <= 1e-6)
    assert np.all(np.diff(g, axis=1) <= 0)                    # descending logits -> descending gates


def test_grouping_hand_example():
    # 4 tokens, k=2, E=6: expert counts [2, 0, 1, 0, 0, 3] (+ expert 4 once -> see below)
    topk = np.array([[5, 0], [2, 5], [0, 5], [4, 3]])
    g = O.group_by_expert(topk, 6, chunk_size=2)
    assert g.counts.tolist() == [2, 0, 1, 1, 1, 3]
    assert g.offsets.tolist() == [0, 2, 2, 3, 4, 5, 8]
    assert g.active.tolist() == [0, 2, 3, 4, 5]
    assert g.chunk_offsets.tolist() == [0, 2, 4, 5]
    # rows: expert 0 <- t0, t2 ; expert 2 <- t1 ; expert 3 <- t3 ; expert 4 <- t3 ; expert 5 <- t0, t1, t2
    assert g.perm_token.tolist() == [0, 2, 1, 3, 3, 0, 1, 2]
    assert g.inv_perm.tolist() == [5, 0, 2, 6, 1, 7, 4, 3]
    g1 = O.group_by_expert(topk, 6, chunk_size=8)
    assert g1.chunk_offsets.tolist() == [0, 5]


def test_grouping_bruteforce_and_invariants():
    rng = np.random.default_rng(2)
    for T, E, k, C in [(33, 7, 3, 2), (50, 12, 4, 5), (1, 4, 4, 1), (17, 9, 1, 3)]:
        logits = rng.standard_normal((T, E)).astype(np.float32)
        topk, _ = O.route_topk(logits, k)
        g = O.group_by_expert(topk, E, C)
        # brute force of the definition pos(t, j) = offsets[e] + #{t' < t routed to e}
        for t in range(T):
            for j in range(k):
                e = topk[t, j]
                before = sum(1 for t2 in range(t) if e in topk[t2])
                assert g.inv_perm[t * k + j] == g.offsets[e] + before
        assert np.all(np.diff(g.offsets) >= 0) and g.offsets[-1] == T * k
        assert np.array_equal(np.bincount(g.perm_token, minlength=T), np.full(T, k))
        assert np.array_equal(g.perm_token[g.inv_perm], np.repeat(np.arange(T), k))
        assert np.array_equal(np.sort(g.inv_perm), np.arange(T * k))
        A = g.num_active
        assert g.chunk_offsets[0] == 0 and g.chunk_offsets[-1] == A
        assert np.all(np.diff(g.chunk_offsets)[:-1] == C) and 1 <= np.diff(g.chunk_offsets)[-1] <= C
        for e in range(E):
            seg = g.perm_token[g.offsets[e]:g.offsets[e + 1]]
            assert np.all(np.diff(seg) > 0)
        x = rng.standard_normal((T, 32))
        xp = O.permute_rows(x, g)
        assert np.array_equal(xp[g.inv_perm.reshape(T, k)[:, 0]], x)


def test_combine_of_replicated_rows_is_identity():
    rng = np.random.default_rng(3)
    T, E, k = 40, 10, 4
    topk, gates = O.route_topk(rng.standard_normal((T, E)).astype(np.float32), k)
    g = O.group_by_expert(topk, E, 4)
    x = O.bf16_round(rng.standard_normal((T, 64)))
    y = O.combine(O.permute_rows(x, g), g.inv_perm, gates, T, k)
    ulp = np.ldexp(1.0, np.frexp(np.abs(x))[1] - 8)
    assert np.all(np.abs(y - x) <= ulp)


# --------------------------------------------------------------------------- GEMMs

def _qweight_from_codes(codes, scale, fmt="int4"):
    """codes: int array [E, N, K] of 4-bit codes; one scale value for every group."""
    codes = np.asarray(codes, dtype=np.uint8)
    E, N, K = codes.shape
    packed = codes[..., 0::2] | (codes[..., 1::2] << 4)
    if fmt == "int4":
        sc = O.bf16_bits_from_values(np.full((E, K // 32, N), scale))
    else:
        sc = np.full((E, K // 32, N), scale, dtype=np.uint8)
    return O.QWeight(fmt, packed.astype(np.uint8), sc)


def test_gemm_closed_form_all_ones():
    K, N = 96, 8
    w = _qweight_from_codes(np.ones((1, N, K)), 1.0)
    out, _ = O.grouped_gemm_fwd(np.ones((3, K)), np.zeros(3, dtype=np.int64), w)
    assert np.all(out == K)
    wm = _qweight_from_codes(np.full((1, N, K), 2), 127, "mxfp4")          # code 2 = 1.0
    out, _ = O.grouped_gemm_fwd(np.ones((2, K)), np.zeros(2, dtype=np.int64), wm)
    assert np.all(out == K)


def test_gemm_one_hot_reads_weight_elements():
    rng = np.random.default_rng(4)
    E, N, K = 2, 5, 64
    codes = rng.integers(0, 16, size=(E, N, K))
    w = _qweight_from_codes(codes, 0.5)
    values = np.array([0, .5, 1, 1.5, 2, 2.5, 3, 3.5, -4, -3.5, -3, -2.5, -2, -1.5, -1, -.5])
    for e in range(E):
        for kk in (0, 1, 31, 32, 63):
            a = np.zeros((1, K))
            a[0, kk] = 1.0
            out, _ = O.grouped_gemm_fwd(a, np.array([e]), w)
            assert np.array_equal(out[0], values[codes[e, :, kk]])
            # backward orientation: d = one-hot over N picks a row of W
            d = np.zeros((1, N))
            d[0, 2] = 1.0
            dx = O.grouped_gemm_bwd_dx(d, np.array([e]), w)
            assert np.array_equal(dx[0], values[codes[e, 2, :]])


def _py_ffn(xrow, Wgu, Wd):
    """Pure-Python SwiGLU expert FFN: loops over every multiply-add."""
    two_f, d = Wgu.shape
    f = two_f // 2
    gu = [sum(xrow[i] * Wgu[n, i] for i in range(d)) for n in range(two_f)]
    h = [gu[j] / (1 + math.exp(-gu[j])) * gu[f + j] for j in range(f)]
    return [sum(h[j] * Wd[n, j] for j in range(f)) for n in range(d)]


def test_dense_masked_moe_bruteforce():
    rng = np.random.default_rng(5)
    E, k, d, f, T = 3, 2, 32, 32, 5
    wgu = _qweight_from_codes(rng.integers(0, 16, (E, 2 * f, d)), 2.0 ** -4)
    wd = _qweight_from_codes(rng.integers(0, 16, (E, d, f)), 2.0 ** -4)
    x = O.bf16_round(rng.standard_normal((T, d)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    fwd = O.moe_forward(x, logits, k, 2, wgu, wd, exact=True)
    Wg = [O.dequant_expert(wgu, e) for e in range(E)]
    Wd = [O.dequant_expert(wd, e) for e in range(E)]
    for t in range(T):
        lg = logits[t].astype(np.float64)
        top = sorted(range(E), key=lambda e: (-lg[e], e))[:k]
        z = [math.exp(lg[e] - lg[top[0]]) for e in top]
        want = np.zeros(d)
        for e in range(E):                         # dense over every expert, masked
            if e in top:
                gate = z[top.index(e)] / sum(z)
                want += np.float32(gate) * np.array(_py_ffn(x[t], Wg[e], Wd[e]))
        assert np.allclose(fwd["y"][t], want, rtol=1e-12, atol=1e-12)


def test_adapter_bruteforce_and_identity():
    rng = np.random.default_rng(6)
    E, K, P = 2, 64, 4
    R = rng.standard_normal((E, K // 32, 32, 32))
    rows = rng.standard_normal((P, K))
    re = np.array([0, 1, 1, 0])
    out = O.adapter_fwd(rows, re, R, exact=True)
    for p in range(P):
        for b in range(K // 32):
            for j in range(32):
                want = sum(rows[p, 32 * b + i] * R[re[p], b, i, j] for i in range(32))
                assert abs(out[p, 32 * b + j] - want) < 1e-12
    eye = np.broadcast_to(np.eye(32), (E, K // 32, 32, 32))
    xb = O.bf16_round(rows)
    assert np.array_equal(O.adapter_fwd(xb, re, eye), xb)


def _tiny_layer(seed=8, E=4, k=2, d=64, f=32, T=6):
    rng = np.random.default_rng(seed)
    wgu = _qweight_from_codes(rng.integers(0, 16, (E, 2 * f, d)), 2.0 ** -3)
    wd = _qweight_from_codes(rng.integers(0, 16, (E, d, f)), 2.0 ** -3)
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    R = np.eye(32) + 0.1 * rng.standard_normal((E, d // 32, 32, 32))
    dy = rng.standard_normal((T, d))
    return wgu, wd, x, logits, R, dy, k


def test_adapter_identity_leaves_forward_unchanged():
    wgu, wd, x, logits, _, _, k = _tiny_layer()
    eye = np.broadcast_to(np.eye(32), (4, 2, 32, 32))
    xb = O.bf16_round(x)
    a = O.moe_forward(xb, logits, k, 2, wgu, wd)
    b = O.moe_forward(xb, logits, k, 2, wgu, wd, R=eye)
    assert np.array_equal(a["y"], b["y"])


def test_backward_matches_finite_differences():
    wgu, wd, x, logits, R, dy, k = _tiny_layer()

    def loss(xv, Rv):
        return float(np.sum(dy * O.moe_forward(xv, logits, k, 2, wgu, wd, R=Rv, exact=True)["y"]))

    fwd = O.moe_forward(x, logits, k, 2, wgu, wd, R=R, exact=True)
    bwd = O.moe_backward(fwd, dy, wgu, wd, R=R, exact=True)
    h = 1e-5
    rng = np.random.default_rng(9)
    for _ in range(12):
        t, i = rng.integers(0, x.shape[0]), rng.integers(0, x.shape[1])
        xp, xm = x.copy(), x.copy()
        xp[t, i] += h
        xm[t, i] -= h
        fd = (loss(xp, R) - loss(xm, R)) / (2 * h)
        assert abs(fd - bwd["dx"][t, i]) <= 1e-6 * max(1.0, abs(fd)), (t, i, fd, bwd["dx"][t, i])
    used = np.unique(fwd["grouping"].row_expert)
    for _ in range(12):
        e = used[rng.integers(0, len(used))]
        b, i, j = rng.integers(0, R.shape[1]), rng.integers(0, 32), rng.integers(0, 32)
        Rp, Rm = R.copy(), R.copy()
        Rp[e, b, i, j] += h
        Rm[e, b, i, j] -= h
        fd = (loss(x, Rp) - loss(x, Rm)) / (2 * h)
        assert abs(fd - bwd["d_adapter"][e, b, i, j]) <= 1e-6 * max(1.0, abs(fd))
    unused = [e for e in range(R.shape[0]) if e not in used]
    for e in unused:
        assert np.all(bwd["d_adapter"][e] == 0)


def test_bwd_dx_is_adjoint_of_fwd():
    rng = np.random.default_rng(10)
    E, N, K, P = 3, 48, 64, 9
    w = _qweight_from_codes(rng.integers(0, 16, (E, N, K)), 0.25)
    re = rng.integers(0, E, P)
    a = rng.standard_normal((P, K))
    dd = rng.standard_normal((P, N))
    fa, _ = O.grouped_gemm_fwd(a, re, w, exact=True)
    bd = O.grouped_gemm_bwd_dx(dd, re, w, exact=True)
    assert abs(np.sum(fa * dd) - np.sum(a * bd)) <= 1e-10 * np.sum(np.abs(fa * dd))


def test_swiglu_bwd_matches_finite_differences():
    rng = np.random.default_rng(11)
    P, f = 3, 32
    g = rng.standard_normal((P, f)) * 3
    u = rng.standard_normal((P, f))
    dh = rng.standard_normal((P, f))
    # identity weight: bwd acc = dh exactly (N = f rows, K = f columns, code 1, scale 1)
    eye_codes = np.eye(f, dtype=np.int64)[None]
    w = _qweight_from_codes(eye_codes, 1.0)
    out = O.grouped_gemm_bwd_dx(dh, np.zeros(P, dtype=np.int64), w, O.EPI_SWIGLU_BWD,
                                np.concatenate([g, u], 1), exact=True)
    hstep = 1e-6
    fd_g = (O.silu(g + hstep) * u - O.silu(g - hstep) * u) / (2 * hstep) * dh
    fd_u = O.silu(g) * dh
    assert np.allclose(out[:, :f], fd_g, rtol=1e-6, atol=1e-8)
    assert np.allclose(out[:, f:], fd_u, rtol=1e-12, atol=1e-12)


def test_outputs_do_not_depend_on_chunk_size():
    wgu, wd, x, logits, R, dy, k = _tiny_layer()
    xb = O.bf16_round(x)
    ys = [O.moe_forward(xb, logits, k, c, wgu, wd, R=R)["y"] for c in (1, 3, 8)]
    assert all(np.array_equal(ys[0], y) for y in ys[1:])


def test_silu_closed_forms():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([1.0]))[0] - 1 / (1 + math.exp(-1))) < 1e-15
    assert O.silu(np.array([-800.0]))[0] == 0.0
    assert O.silu(np.array([50.0]))[0] == pytest.approx(50.0, rel=1e-15)


# --------------------------------------------------------------------------- accounting

def test_storage_arithmetic_matches_pages():
    want = {}
    with open(os.path.join(GOLDEN, "storage_arithmetic.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].split()
            if line:
                want[line[0]] = (float(line[1]), float(line[2]))
    P = 2.8e12
    got = {
        "fp16_2p8T_bytes": P * 2,
        "pure4bit_2p8T_bytes": accounting.storage_estimate(P, sensitive_ratio=0.0, scale_bits=0),
        "mxfp4_2p8T_bytes": accounting.storage_estimate(P),
        "fourbit_280B_bytes": accounting.storage_estimate(280e9, sensitive_ratio=0.0, scale_bits=0),
    }
    got["fp16_over_mxfp4_ratio"] = got["fp16_2p8T_bytes"] / got["mxfp4_2p8T_bytes"]
    for name, (value, rtol) in want.items():
        assert abs(got[name] - value) <= rtol * value, (name, got[name], value)


def test_bytes_per_param_and_expert_bytes():
    assert accounting.bytes_per_param("int4") == 0.5625
    assert accounting.bytes_per_param("mxfp4") == 0.53125
    # one trillion-shaped expert (gate/up 4096 x 7168 + down 7168 x 2048), INT4
    b = accounting.expert_weight_bytes(4096, 7168, "int4") + accounting.expert_weight_bytes(7168, 2048, "int4")
    assert b == 3 * 7168 * 2048 * 0.5625


# --------------------------------------------------------------------------- generator

def test_generator_is_seeded_and_decodes_close_to_source():
    a = synth.make_workload(TINY_INT4)
    b = synth.make_workload(TINY_INT4)
    assert torch.equal(a["w_gu"].packed, b["w_gu"].packed) and torch.equal(a["x"], b["x"])
    g = torch.Generator().manual_seed(3)
    w = torch.randn((64, 128), generator=g) * 0.02
    p, s = synth.quantize_int4(w)
    deq = O.dequant_int4_rows(p.numpy(), s.view(torch.int16).numpy().view(np.uint16).T)
    step = np.repeat(O.bf16_values_from_bits(s.view(torch.int16).numpy().view(np.uint16).T), 32, 1)
    # half a quantization step, plus the BF16 rounding of q*s (half an ulp, at most 2**-8 relative)
    assert np.all(np.abs(deq - w.double().numpy()) <= 0.5 * step + np.abs(deq) * 2.0 ** -8 + 1e-12)
    p, X = synth.quantize_mxfp4(w)
    deq = O.dequant_mxfp4_rows(p.numpy(), X.numpy().T)
    unit = np.repeat(O.e8m0_value(X.numpy().T), 32, 1)
    err = np.abs(deq - w.double().numpy())
    assert np.all(err <= 2.0 * unit)                 # saturation at 6 bounds the worst case
    assert np.mean(err / unit) < 0.3
