"""Plain float64 CPU oracle of the low-bit MoE hot path (test infrastructure only).

What the path computes, step by step, following the source pages:

* Orbit article, section "technical details" (时刻细节), paragraph
  "Active-expert-chunked dequantization": the experts the router selects are
  grouped into fixed-size batches, their low-bit weights are dequantized and a
  grouped GEMM runs over them; the high-precision weights live only while the
  batch is computed.
* Orbit article, same section, DeepSeek-V4 paragraph: the GEMM backward
  bypasses the base-weight gradient (the base is frozen; only activation and
  adapter gradients are formed).
* Orbit article, Kimi-K2.6 and DeepSeek-V4-Flash result sections: the frozen
  base is INT4 (resp. FP4) and the trainable adapter is BF16, on the same path
  for training and rollout.
* Orbit issue #1 ("difference from slime"), maintainer reply: the adapter is
  OFT/QOFT and the quantized weights are fine-tuned directly, without storing a
  dequantized base.
* Open-weight MoE explainer, section 三 (MXFP4 quantization), "microscaling"
  paragraph: weights are split into groups of 32, stored as 4-bit elements,
  with one shared higher-precision scale per group.

Readings taken where the pages are silent (each is repeated where it is used):

* INT4: two's-complement nibble (-8..7), one BF16 scale per 32 consecutive
  elements along the reduction dimension, w = bf16(q * s) with one rounding.
* MXFP4: E2M1 element (sign bit 3, magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6) and an
  E8M0 group scale 2**(X-127) (X = 255 is NaN), w = bf16(e2m1 * 2**(X-127)).
* Packing: byte i of a weight row holds element 2i in its low nibble and
  element 2i+1 in its high nibble. Scales are stored group-major:
  scales[e][g][n] is the scale of row n, elements 32g..32g+31.
* Top-k: the k largest raw logits, in descending order, ties to the lower
  expert id; gates are the softmax over the k selected logits.
* Permutation: expert-major, then ascending token id (stable).
* Chunks: consecutive runs of ``chunk_size`` active experts in ascending id.
* Adapter: per expert a block-diagonal d x d matrix of 32 x 32 blocks applied to
  the gate/up input, x' = x R (row vectors); the down projection has none.
* SwiGLU: gate rows 0..f-1 and up rows f..2f-1 of the gate/up weight,
  h = silu(g) * u with silu(g) = g / (1 + exp(-g)).
* Gate weights are applied in the combine, not inside the GEMM.
* BF16 storage points: x', h, the per-slot down output, saved g|u, the
  gradient rows dg|du and dx'; everything else accumulates in float64 here.

``exact=True`` skips every BF16 rounding of intermediates and outputs, which
turns the oracle into the pure real-number function used by the
finite-difference and adjoint pins.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = [
    "BF16_MAX", "bf16_round", "bf16_bits_from_values", "bf16_values_from_bits",
    "unpack_nibbles", "int4_code_value", "e2m1_value", "e8m0_value",
    "dequant_int4_rows", "dequant_mxfp4_rows", "QWeight", "dequant_expert",
    "route_topk", "Grouping", "group_by_expert", "permute_rows",
    "adapter_fwd", "adapter_bwd", "silu", "grouped_gemm_fwd",
    "grouped_gemm_bwd_dx", "combine", "gather_scaled",
    "moe_forward", "moe_backward", "up_projection", "EPI_NONE", "EPI_SWIGLU",
    "EPI_SWIGLU_BWD",
]

EPI_NONE = "none"
EPI_SWIGLU = "swiglu"
EPI_SWIGLU_BWD = "swiglu_bwd"

# Largest finite bfloat16: (2 - 2**-7) * 2**127.
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# --------------------------------------------------------------------------
# bfloat16 rounding (the method's storage type for activations and adapter)
# --------------------------------------------------------------------------

def bf16_round(x, exact: bool = False) -> np.ndarray:
    """Round real values (float64) to the nearest bfloat16, ties to even.

    One rounding straight from float64: bfloat16 keeps 8 significant bits for
    normal numbers (|x| >= 2**-126) and a fixed spacing of 2**-133 below that;
    results above the largest finite value become +-inf. NaN passes through.
    """
    x = np.asarray(x, dtype=np.float64)
    if exact:
        return x
    out = x.copy()
    finite = np.isfinite(x)
    xf = x[finite]
    _, expo = np.frexp(xf)                      # |xf| in [2**(expo-1), 2**expo)
    quantum = np.ldexp(1.0, np.maximum(expo - 8, -133))
    big = np.abs(xf) >= 2.0 ** 128
    r = np.rint(np.where(big, 0.0, xf) / quantum) * quantum   # rint = ties-to-even
    r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, xf), r)
    r = np.where(big, np.copysign(np.inf, xf), r)
    # rint keeps the sign of zero, so -tiny -> -0.0 as IEEE rounding does.
    out[finite] = r
    return out


def bf16_bits_from_values(v) -> np.ndarray:
    """uint16 bit patterns of values that are already bfloat16 numbers (NaN -> 0x7FC0)."""
    v = np.asarray(v, dtype=np.float64)
    f = np.atleast_1d(v.astype(np.float32))
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    bits = np.where(np.isnan(f), np.uint16(0x7FC0), bits).astype(np.uint16)
    return bits.reshape(v.shape)


def bf16_values_from_bits(bits) -> np.ndarray:
    """float64 values of bfloat16 bit patterns."""
    b = np.asarray(bits).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Dequantization of the frozen 4-bit base
# --------------------------------------------------------------------------

def unpack_nibbles(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] 4-bit codes; element 2i = low nibble of byte i."""
    packed = np.asarray(packed, dtype=np.uint8)
    codes = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    codes[..., 0::2] = packed & 0x0F
    codes[..., 1::2] = packed >> 4
    return codes


def int4_code_value(codes) -> np.ndarray:
    """Two's-complement nibble: 0..7 -> 0..7, 8..15 -> -8..-1 (Orbit article, Kimi-K2.6 section: INT4 base)."""
    c = np.asarray(codes).astype(np.int64)
    return np.where(c >= 8, c - 16, c).astype(np.float64)


# E2M1 magnitudes of codes 0..7: exponent bits 2..1, mantissa bit 0, bias 1,
# code 1 is the subnormal 0.5.
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_value(codes) -> np.ndarray:
    """E2M1 element value; bit 3 is the sign, so code 8 is -0.0."""
    c = np.asarray(codes).astype(np.int64)
    mag = _E2M1_MAG[c & 7]
    return np.where((c >> 3) & 1 == 1, -mag, mag)


def e8m0_value(x) -> np.ndarray:
    """E8M0 shared scale 2**(X-127); X = 255 encodes NaN."""
    x = np.asarray(x).astype(np.int64)
    v = np.ldexp(1.0, x - 127)
    return np.where(x == 255, np.nan, v)


def dequant_int4_rows(packed_rows, scale_bits_rows, exact: bool = False) -> np.ndarray:
    """INT4 rows -> BF16 values: w[n, k] = bf16(q[n, k] * s[n, k // 32]).

    packed_rows: uint8 [R, K/2]; scale_bits_rows: uint16 [R, K/32] BF16 bit
    patterns. The product of a 4-bit integer and a BF16 scale is exact in
    float64, so the one rounding is the BF16 one.
    """
    q = int4_code_value(unpack_nibbles(packed_rows))
    s = np.repeat(bf16_values_from_bits(scale_bits_rows), 32, axis=-1)
    return bf16_round(q * s, exact)


def dequant_mxfp4_rows(packed_rows, scale_rows, exact: bool = False) -> np.ndarray:
    """MXFP4 rows -> BF16 values: w[n, k] = bf16(e2m1(code) * 2**(X[n, k//32] - 127)).

    Explainer section 三: 32-element groups of 4-bit elements sharing one
    higher-precision scale. The product is exact except where it overflows
    BF16 (-> inf); X = 255 gives NaN.
    """
    v = e2m1_value(unpack_nibbles(packed_rows))
    s = np.repeat(e8m0_value(scale_rows), 32, axis=-1)
    with np.errstate(invalid="ignore"):
        return bf16_round(v * s, exact)


@dataclass
class QWeight:
    """A frozen low-bit expert weight stack, W[e] of shape [N, K].

    fmt: "int4" (scales: uint16 BF16 bits) or "mxfp4" (scales: uint8 E8M0).
    packed: uint8 [E, N, K/2]; scales: [E, K/32, N] (group-major).
    """
    fmt: str
    packed: np.ndarray
    scales: np.ndarray

    @property
    def E(self) -> int:
        return self.packed.shape[0]

    @property
    def N(self) -> int:
        return self.packed.shape[1]

    @property
    def K(self) -> int:
        return self.packed.shape[2] * 2


def dequant_expert(w: QWeight, e: int, exact: bool = False) -> np.ndarray:
    """Dequantized float64 [N, K] weight of expert e (the values are BF16 numbers)."""
    packed = w.packed[e]
    scales = np.ascontiguousarray(w.scales[e].T)      # [N, K/32]
    if w.fmt == "int4":
        return dequant_int4_rows(packed, scales, exact)
    if w.fmt == "mxfp4":
        return dequant_mxfp4_rows(packed, scales, exact)
    raise ValueError(f"unknown weight format {w.fmt!r}")


# --------------------------------------------------------------------------
# Routing: top-k, per-expert groups, active-expert chunks, permutation
# --------------------------------------------------------------------------

def route_topk(logits, k: int):
    """Per token the k largest logits (descending, ties -> lower expert id) and
    gates = softmax over those k logits (float64 math, stored float32).

    Orbit article, "Active-expert-chunked dequantization": each token activates
    only the experts its router selects.
    """
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids, -lg), axis=-1)        # primary key -logit, then id
    topk = order[:, :k].astype(np.int64)
    sel = np.take_along_axis(lg, topk, axis=1)
    z = np.exp(sel - sel[:, :1])
    gates = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    return topk, gates


@dataclass
class Grouping:
    counts: np.ndarray          # [E]
    offsets: np.ndarray         # [E+1], exclusive scan of counts
    active: np.ndarray          # [A], experts with counts > 0, ascending
    chunk_offsets: np.ndarray   # [num_chunks+1], into ``active``
    perm_token: np.ndarray      # [T*k], token of each permuted row
    inv_perm: np.ndarray        # [T*k], row of (token t, slot j) at t*k + j
    row_expert: np.ndarray      # [T*k], expert of each permuted row

    @property
    def num_active(self) -> int:
        return int(self.active.shape[0])

    @property
    def num_chunks(self) -> int:
        return int(self.chunk_offsets.shape[0] - 1)


def group_by_expert(topk, E: int, chunk_size: int) -> Grouping:
    """Counts, offsets, the active-expert list, fixed-size chunks and the
    stable permutation pos(t, j) = offsets[e] + #{t' < t routed to e}.

    Orbit article, "Active-expert-chunked dequantization": the selected experts
    are batched into fixed-size groups. Reading: chunk c holds active experts
    chunk_size*c .. chunk_size*(c+1)-1 (ascending id); the last may be short.
    """
    topk = np.asarray(topk, dtype=np.int64)
    T, k = topk.shape
    if chunk_size < 1:
        raise ValueError("chunk_size must be >= 1")
    flat = topk.ravel()
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    active = np.nonzero(counts)[0].astype(np.int64)
    A = active.shape[0]
    num_chunks = -(-A // chunk_size)
    chunk_offsets = np.minimum(np.arange(num_chunks + 1) * chunk_size, A).astype(np.int64)
    # A stable sort by expert keeps the flat (token, slot) order inside each
    # expert; a token reaches an expert at most once, so that is token order.
    order = np.argsort(flat, kind="stable")
    perm_token = (order // k).astype(np.int64)
    inv_perm = np.empty(T * k, dtype=np.int64)
    inv_perm[order] = np.arange(T * k)
    row_expert = flat[order]
    return Grouping(counts, offsets, active, chunk_offsets, perm_token, inv_perm, row_expert)


def permute_rows(x, g: Grouping) -> np.ndarray:
    """x_perm[p] = x[perm_token[p]] (an exact copy of BF16 rows)."""
    return np.asarray(x)[g.perm_token]


# --------------------------------------------------------------------------
# BF16 block-diagonal adapter (OFT-style, per expert)
# --------------------------------------------------------------------------

def _blocks(rows) -> np.ndarray:
    m, K = rows.shape
    return rows.reshape(m, K // 32, 32)


def adapter_fwd(rows, row_expert, R, exact: bool = False) -> np.ndarray:
    """x'[p, 32b+j] = sum_i x[p, 32b+i] * R[e, b, i, j], rounded to BF16.

    Orbit issue #1: the adapter is orthogonal fine-tuning; its form here is a
    per-expert block-diagonal matrix of 32 x 32 blocks acting on the
    activations before the frozen base GEMM. R: float64 [E, K/32, 32, 32].
    """
    rows = np.asarray(rows, dtype=np.float64)
    out = np.empty_like(rows)
    for e in np.unique(row_expert):
        sel = row_expert == e
        xb = _blocks(rows[sel])
        out[sel] = np.einsum("mbi,bij->mbj", xb, R[e]).reshape(xb.shape[0], -1)
    return bf16_round(out, exact)


def adapter_bwd(x_rows, dxp_rows, row_expert, R, E: int, exact: bool = False):
    """Adapter backward given dx' (the gradient at the adapter output).

    dx[p, 32b+i] = sum_j dx'[p, 32b+j] * R[e, b, i, j]   (BF16 output)
    dR[e, b, i, j] = sum_{p in e} x[p, 32b+i] * dx'[p, 32b+j]   (float32 output)
    Experts with no rows get dR = 0.
    """
    x_rows = np.asarray(x_rows, dtype=np.float64)
    dxp_rows = np.asarray(dxp_rows, dtype=np.float64)
    nb = x_rows.shape[1] // 32
    dx = np.empty_like(dxp_rows)
    dR = np.zeros((E, nb, 32, 32), dtype=np.float64)
    for e in np.unique(row_expert):
        sel = row_expert == e
        gb = _blocks(dxp_rows[sel])
        xb = _blocks(x_rows[sel])
        dx[sel] = np.einsum("mbj,bij->mbi", gb, R[e]).reshape(gb.shape[0], -1)
        dR[e] = np.einsum("mbi,mbj->bij", xb, gb)
    dR_out = dR if exact else dR.astype(np.float32).astype(np.float64)
    return bf16_round(dx, exact), dR_out


# --------------------------------------------------------------------------
# Grouped GEMM over the dequantized experts (forward and dX backward)
# --------------------------------------------------------------------------

def silu(g) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def _sigmoid(g) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-g))


def grouped_gemm_fwd(a_rows, row_expert, w: QWeight, epilogue: str = EPI_NONE,
                     exact: bool = False, weight_cache: dict | None = None):
    """Forward grouped GEMM: for each row p of expert e, acc[p] = a[p] @ W[e]^T.

    Orbit article, "Active-expert-chunked dequantization" (dequantize the
    selected experts, then grouped GEMM). Epilogues:
      none   -> out = bf16(acc)                                   [P, N]
      swiglu -> out = bf16(silu(acc[:, :N/2]) * acc[:, N/2:])     [P, N/2]
                saved = bf16(acc) (the g|u rows kept for backward) [P, N]
    Returns (out, saved) with saved None for "none".
    """
    a_rows = np.asarray(a_rows, dtype=np.float64)
    P = a_rows.shape[0]
    acc = np.zeros((P, w.N), dtype=np.float64)
    for e in np.unique(row_expert):
        sel = row_expert == e
        W = _weight(w, int(e), exact, weight_cache)
        acc[sel] = a_rows[sel] @ W.T
    if epilogue == EPI_NONE:
        return bf16_round(acc, exact), None
    if epilogue == EPI_SWIGLU:
        f = w.N // 2
        h = silu(acc[:, :f]) * acc[:, f:]
        return bf16_round(h, exact), bf16_round(acc, exact)
    raise ValueError(f"unknown forward epilogue {epilogue!r}")


def grouped_gemm_bwd_dx(d_rows, row_expert, w: QWeight, epilogue: str = EPI_NONE,
                        saved_gu=None, exact: bool = False,
                        weight_cache: dict | None = None) -> np.ndarray:
    """Activation-gradient grouped GEMM, no base-weight gradient.

    Orbit article, DeepSeek-V4 paragraph: the backward GEMM bypasses the frozen
    base's weight gradient. For each row p of expert e: acc[p] = d[p] @ W[e]
    (contraction over W's N rows, output over its K columns). Epilogues:
      none       -> bf16(acc)                                     [P, K]
      swiglu_bwd -> acc is dh; with saved g|u (BF16, [P, 2K]):
                    du = dh * silu(g), dg = dh * u * s * (1 + g * (1 - s)),
                    s = sigmoid(g); out = bf16([dg | du])          [P, 2K]
    """
    d_rows = np.asarray(d_rows, dtype=np.float64)
    P = d_rows.shape[0]
    acc = np.zeros((P, w.K), dtype=np.float64)
    for e in np.unique(row_expert):
        sel = row_expert == e
        W = _weight(w, int(e), exact, weight_cache)
        acc[sel] = d_rows[sel] @ W
    if epilogue == EPI_NONE:
        return bf16_round(acc, exact)
    if epilogue == EPI_SWIGLU_BWD:
        saved_gu = np.asarray(saved_gu, dtype=np.float64)
        f = w.K
        g, u = saved_gu[:, :f], saved_gu[:, f:]
        s = _sigmoid(g)
        du = acc * g * s
        dg = acc * u * s * (1.0 + g * (1.0 - s))
        return bf16_round(np.concatenate([dg, du], axis=1), exact)
    raise ValueError(f"unknown backward epilogue {epilogue!r}")


def _weight(w: QWeight, e: int, exact: bool, cache: dict | None) -> np.ndarray:
    if cache is None:
        return dequant_expert(w, e, exact)
    key = (id(w), e, exact)
    if key not in cache:
        cache[key] = dequant_expert(w, e, exact)
    return cache[key]


# --------------------------------------------------------------------------
# Unpermute + combine, and the gate-scaled gather of the backward
# --------------------------------------------------------------------------

def combine(rows, inv_perm, gates, T: int, k: int, exact: bool = False) -> np.ndarray:
    """y[t] = bf16(sum_j g[t, j] * rows[inv_perm[t*k + j]]); gates=None means all 1."""
    rows = np.asarray(rows, dtype=np.float64)
    idx = np.asarray(inv_perm).reshape(T, k)
    g = np.ones((T, k)) if gates is None else np.asarray(gates, np.float32).astype(np.float64).reshape(T, k)
    y = np.zeros((T, rows.shape[1]), dtype=np.float64)
    for j in range(k):
        y += g[:, j:j + 1] * rows[idx[:, j]]
    return bf16_round(y, exact)


def gather_scaled(dy, inv_perm, gates, T: int, k: int, exact: bool = False) -> np.ndarray:
    """Backward of the combine with respect to the per-slot rows:
    out[inv_perm[t*k + j]] = bf16(g[t, j] * dy[t])."""
    dy = np.asarray(dy, dtype=np.float64)
    idx = np.asarray(inv_perm).reshape(T, k)
    g = np.ones((T, k)) if gates is None else np.asarray(gates, np.float32).astype(np.float64).reshape(T, k)
    out = np.zeros((T * k, dy.shape[1]), dtype=np.float64)
    for j in range(k):
        out[idx[:, j]] = g[:, j:j + 1] * dy
    return bf16_round(out, exact)


# --------------------------------------------------------------------------
# Whole-layer chains
# --------------------------------------------------------------------------

def moe_forward(x, logits, k: int, chunk_size: int, w_gu: QWeight, w_d: QWeight,
                R=None, exact: bool = False, weight_cache: dict | None = None) -> dict:
    """Route -> permute -> [adapter] -> gate/up GEMM + SwiGLU -> down GEMM -> combine."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    topk, gates = route_topk(logits, k)
    g = group_by_expert(topk, w_gu.E, chunk_size)
    x_perm = permute_rows(x, g)
    xa = adapter_fwd(x_perm, g.row_expert, R, exact) if R is not None else x_perm
    h, saved = grouped_gemm_fwd(xa, g.row_expert, w_gu, EPI_SWIGLU, exact, weight_cache)
    y_perm, _ = grouped_gemm_fwd(h, g.row_expert, w_d, EPI_NONE, exact, weight_cache)
    y = combine(y_perm, g.inv_perm, gates, T, k, exact)
    return dict(topk=topk, gates=gates, grouping=g, x_perm=x_perm, x_adapted=xa,
                h=h, saved_gu=saved, y_perm=y_perm, y=y)


def moe_backward(fwd: dict, dy, w_gu: QWeight, w_d: QWeight, R=None,
                 exact: bool = False, weight_cache: dict | None = None) -> dict:
    """Backward to the activations and the adapter blocks; the base stays frozen.

    gather (gate-scaled) -> down bwd_dx + SwiGLU bwd -> gate/up bwd_dx ->
    [adapter bwd] -> unpermute-sum. The gates are treated as constants.
    """
    g: Grouping = fwd["grouping"]
    dy = np.asarray(dy, dtype=np.float64)
    T = dy.shape[0]
    k = fwd["topk"].shape[1]
    dy_perm = gather_scaled(dy, g.inv_perm, fwd["gates"], T, k, exact)
    dgu = grouped_gemm_bwd_dx(dy_perm, g.row_expert, w_d, EPI_SWIGLU_BWD, fwd["saved_gu"],
                              exact, weight_cache)
    dxa = grouped_gemm_bwd_dx(dgu, g.row_expert, w_gu, EPI_NONE, None, exact, weight_cache)
    if R is not None:
        dx_perm, dR = adapter_bwd(fwd["x_perm"], dxa, g.row_expert, R, w_gu.E, exact)
    else:
        dx_perm, dR = dxa, None
    dx = combine(dx_perm, g.inv_perm, None, T, k, exact)
    return dict(dy_perm=dy_perm, dgu=dgu, dx_adapted=dxa, dx_perm=dx_perm, dx=dx, d_adapter=dR)


def up_projection(x, logits, k: int, chunk_size: int, w_up: QWeight,
                  exact: bool = False, weight_cache: dict | None = None) -> dict:
    """Single grouped up-projection (no SwiGLU): route -> permute -> GEMM."""
    topk, gates = route_topk(logits, k)
    g = group_by_expert(topk, w_up.E, chunk_size)
    x_perm = permute_rows(np.asarray(x, dtype=np.float64), g)
    out, _ = grouped_gemm_fwd(x_perm, g.row_expert, w_up, EPI_NONE, exact, weight_cache)
    return dict(topk=topk, gates=gates, grouping=g, x_perm=x_perm, out=out)
