"""Full-size parity of the layer workloads (trillion-shaped INT4 at T = 128,
2048 and 16384; skewed-routing MXFP4; the INT4 training step with adapter).

At these sizes the oracle cannot run the whole layer in seconds, so each
launch is checked in three ways:

1. Routing (top-k, gates, offsets, active list, chunk table, permutation) is
   compared bit-exactly in full.
2. Every tile of every grouped-GEMM launch is compared with the oracle, step by
   step. For every active expert and every output-feature tile of a launch the
   oracle computes some output features for ALL of the expert's rows, so every
   (expert, feature tile, token tile) of the launch is covered:
   - gate/up + SwiGLU (64 h features per tile): one h feature per
     tensor-memory lane quarter, at an offset that rotates with the expert and
     the tile;
   - down projection (128 features per tile): one feature per lane quarter,
     rotating with the tile (the same for every expert, so that the combine
     can be checked on every token, step 3);
   - backward down projection with the SwiGLU backward (128 features of dh per
     tile): one whole 32-wide quantization group per tile, rotating with the
     expert and the tile (the weight is read across its groups here);
   - backward gate/up (128 features per tile): one 32-wide group per tile,
     rotating with the tile, the same for every expert; with the adapter, the
     oracle's adapter backward on those 32-wide blocks.
   The oracle is fed the library's own BF16 input to each step: x_perm (and
   the oracle's adapter output of it), h for the down projection, the
   gate-scaled dy with the library's saved g|u for the backward down
   projection, dg|du for the backward gate/up. Criterion: per-slot values
   within 2e-2 + one BF16 ulp of the oracle value.
3. The outputs that end the computation are compared on EVERY token at the
   checked features, against the combine (slot order, gates) of the oracle's
   per-slot rows of step 2, with the final-output criterion (max-abs <= 2e-2,
   rel-L2 <= 5e-3): y at the down projection's features, dx at the backward
   gate/up's blocks.

Besides, for a few sampled experts (first and last active, the busiest, one at
random) the oracle runs the whole chain of those experts' rows from the raw
inputs (adapter, gate/up + SwiGLU, down, and for training the gate-scaled
gather, SwiGLU backward, gate/up backward, adapter backward), every output
feature of every row. The FP32 adapter gradient is compared per block, for
those experts in full and for every expert at the checked blocks, within 2e-2
plus the spread that one-ulp differences of its BF16 input dx' can cause
(dx' stays inside the library's backward call, so the oracle forms its own).
"""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import layer, moeq, synth
from quantized_rl_fine_b200.configs import TRAIN_INT4, TRILLION_INT4, ZIPF_MXFP4

from _common import (adapter_grad_bound, assert_close_bounded, assert_close_final,
                     assert_close_intermediate, bf16_bits, bf16_ulp, f64)

pytestmark = pytest.mark.gpu

DEV = "cuda"
THREADS = max(1, min(32, os.cpu_count() or 1))


# ------------------------------------------------------------------ routing and sampled chains

def _check_routing_full(r, x, topk, gates, g, rows):
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
    if r.x_perm is not None:
        idx = torch.as_tensor(rows, device=r.x_perm.device)
        xp = bf16_bits(r.x_perm.index_select(0, idx))
        xs = bf16_bits(x.index_select(0, torch.as_tensor(g.perm_token[rows], device=x.device)))
        assert np.array_equal(xp, xs)


def _sample_experts(g, seed):
    counts = np.diff(g.offsets)
    act = g.active
    rng = np.random.default_rng(seed)
    pick = {int(act[0]), int(act[-1]), int(np.argmax(counts)), int(rng.choice(act))}
    return sorted(pick)


def _local_qweight(w, experts):
    """Oracle view of the selected experts only (local expert index = position)."""
    sel = torch.as_tensor(experts, device=w.packed.device)
    packed = w.packed.index_select(0, sel).cpu().numpy()
    sc = w.scales.index_select(0, sel)
    scales = bf16_bits(sc) if w.fmt == "int4" else sc.cpu().numpy()
    return O.QWeight(w.fmt, packed, scales)


def _rows_of(g, experts):
    rows, local = [], []
    for i, e in enumerate(experts):
        r = np.arange(g.offsets[e], g.offsets[e + 1])
        rows.append(r)
        local.append(np.full(r.shape[0], i))
    return np.concatenate(rows), np.concatenate(local)


def _take(t, rows):
    return f64(t.index_select(0, torch.as_tensor(rows, device=t.device)))


def _sampled_chain(cfg, wl, st, bw, g, gates, experts):
    """The whole chain of the sampled experts' rows from the raw inputs."""
    rows, local = _rows_of(g, experts)
    wgu = _local_qweight(wl["w_gu"], experts)
    wd = _local_qweight(wl["w_d"], experts)
    x_rows = _take(wl["x"], g.perm_token[rows])
    R = None
    if cfg.adapter:
        R = f64(wl["adapter"].index_select(0, torch.as_tensor(experts, device=DEV)))
        xa = O.adapter_fwd(x_rows, local, R)
    else:
        xa = x_rows
    h, saved = O.grouped_gemm_fwd(xa, local, wgu, O.EPI_SWIGLU)
    y_perm, _ = O.grouped_gemm_fwd(h, local, wd, O.EPI_NONE)
    assert_close_intermediate(_take(st["h"], rows), h, "h (sampled chain)")
    assert_close_intermediate(_take(st["y_perm"], rows), y_perm, "y_perm (sampled chain)")
    if not cfg.train:
        return
    T = wl["x"].shape[0]
    assert_close_intermediate(_take(st["saved_gu"], rows), saved, "saved_gu (sampled chain)")
    dy_perm = O.gather_scaled(f64(wl["dy"]), g.inv_perm, gates, T, cfg.k)[rows]
    assert np.array_equal(bf16_bits(bw["dy_perm"].index_select(0, torch.as_tensor(rows, device=DEV))),
                          O.bf16_bits_from_values(dy_perm))
    dgu = O.grouped_gemm_bwd_dx(dy_perm, local, wd, O.EPI_SWIGLU_BWD, saved)
    assert_close_intermediate(_take(bw["dgu"], rows), dgu, "dgu (sampled chain)")
    dxa = O.grouped_gemm_bwd_dx(dgu, local, wgu, O.EPI_NONE)
    if cfg.adapter:
        dx_perm, dR = O.adapter_bwd(x_rows, dxa, local, R, len(experts))
        got_dR = bw["d_adapter"].index_select(0, torch.as_tensor(experts, device=DEV))
        bound = adapter_grad_bound(x_rows, dxa, local, len(experts))
        assert_close_bounded(got_dR.cpu().numpy().astype(np.float64), dR, bound,
                             "d_adapter (sampled chain)")
    else:
        dx_perm = dxa
    assert_close_intermediate(_take(bw["dx_perm"], rows), dx_perm, "dx_perm (sampled chain)")


# ------------------------------------------------------------------ every tile

def _quarter_features(n_tiles, tile, e=0):
    """One output feature per tensor-memory lane quarter (tile / 4 features)
    of each feature tile, at an offset that rotates with the tile and, when
    e is given, the expert."""
    quarter = tile // 4
    t = np.arange(n_tiles)[:, None]
    q = np.arange(4)[None, :]
    off = (e * 5 + t * 3 + q * 7) % quarter
    return (tile * t + quarter * q + off).reshape(-1)


def _tile_groups(n_tiles, e=0):
    """One 32-wide quantization group of each 128-feature tile, rotating with
    the tile and, when e is given, the expert."""
    t = np.arange(n_tiles)
    return 4 * t + (e + 2 * t + 1) % 4


def _group_cols(groups):
    return (32 * groups[:, None] + np.arange(32)[None, :]).reshape(-1)


def _scale_host(sc, fmt):
    return bf16_bits(sc) if fmt == "int4" else sc.cpu().numpy()


def _row_weights(w, experts, feats):
    """Per expert an oracle QWeight holding its weight rows feats[e] (all of K):
    one gather on the device, one copy to the host."""
    E, N, K2 = w.packed.shape
    idx = np.concatenate([e * N + feats[e] for e in experts])
    it = torch.as_tensor(idx, device=w.packed.device)
    packed = w.packed.reshape(E * N, K2).index_select(0, it).cpu().numpy()
    sc = w.scales.permute(0, 2, 1).reshape(E * N, -1).index_select(0, it)   # [rows][K/32]
    sc = _scale_host(sc, w.fmt)
    out, o = {}, 0
    for e in experts:
        n = feats[e].shape[0]
        out[e] = O.QWeight(w.fmt, packed[None, o:o + n], np.ascontiguousarray(sc[o:o + n].T)[None])
        o += n
    return out


def _col_weights(w, experts, groups):
    """Per expert an oracle QWeight restricted to the reduction-dimension
    groups groups[e] (32 consecutive K columns each): [1][N][16 * ng] bytes."""
    E, N, K2 = w.packed.shape
    out = {}
    for e in experts:
        gt = torch.as_tensor(groups[e], device=w.packed.device)
        packed = w.packed[e].reshape(N, K2 // 16, 16).index_select(1, gt).reshape(N, -1)
        sc = w.scales[e].index_select(0, gt)                                    # [ng][N]
        out[e] = O.QWeight(w.fmt, packed.cpu().numpy()[None], _scale_host(sc, w.fmt)[None])
    return out


# The oracle dequantizes a whole weight matrix per call; its temporaries stay
# in cache (and so run several times faster) when each call covers at most a
# few hundred thousand weights, so the oracle's GEMM functions are called on
# slices of the selected weight rows or groups and the results concatenated.

def _sub_rows(w, idx):
    return O.QWeight(w.fmt, w.packed[:, idx], w.scales[:, :, idx])


def _fwd_swiglu(a, r0, w, step=8):
    """grouped_gemm_fwd(SwiGLU) of rows [gate 0..n-1 | up 0..n-1], in slices."""
    n = w.N // 2
    hs, gs, us = [], [], []
    for i in range(0, n, step):
        j = np.arange(i, min(n, i + step))
        h, sv = O.grouped_gemm_fwd(a, r0, _sub_rows(w, np.concatenate([j, n + j])), O.EPI_SWIGLU)
        hs.append(h)
        gs.append(sv[:, :j.size])
        us.append(sv[:, j.size:])
    return np.concatenate(hs, 1), np.concatenate(gs + us, 1)


def _fwd_none(a, r0, w, step=32):
    return np.concatenate([O.grouped_gemm_fwd(a, r0, _sub_rows(w, np.arange(i, min(w.N, i + step))),
                                              O.EPI_NONE)[0] for i in range(0, w.N, step)], 1)


def _sub_group(w, j):
    return O.QWeight(w.fmt, w.packed[:, :, 16 * j:16 * j + 16], w.scales[:, j:j + 1, :])


def _bwd_groups(d_rows, r0, w, epi=O.EPI_NONE, saved=None):
    """grouped_gemm_bwd_dx over a group-restricted weight, one group per call;
    with the SwiGLU backward, saved = [g | u] of the same columns."""
    ng = w.K // 32
    outs_g, outs_u = [], []
    for j in range(ng):
        if epi == O.EPI_SWIGLU_BWD:
            c = slice(32 * j, 32 * j + 32)
            sv = np.concatenate([saved[:, c], saved[:, 32 * ng + 32 * j:32 * ng + 32 * j + 32]], 1)
            o = O.grouped_gemm_bwd_dx(d_rows, r0, _sub_group(w, j), epi, sv)
            outs_g.append(o[:, :32])
            outs_u.append(o[:, 32:])
        else:
            outs_g.append(O.grouped_gemm_bwd_dx(d_rows, r0, _sub_group(w, j), epi))
    return np.concatenate(outs_g + outs_u, 1)


class _Errors:
    """Per-slot comparison statistics gathered over the experts."""

    def __init__(self, what):
        self.what, self.bad, self.n, self.worst = what, 0, 0, 0.0

    def add(self, got, want):
        assert got.shape == want.shape, (self.what, got.shape, want.shape)
        err = np.abs(got - want)
        lim = 2e-2 + bf16_ulp(want)
        self.bad += int((err > lim).sum()) + int((~np.isfinite(got)).sum())
        self.n += err.size
        self.worst = max(self.worst, float(np.nanmax(err)) if err.size else 0.0)

    def check(self):
        assert self.n > 0, f"{self.what}: nothing compared"
        assert self.bad == 0, \
            f"{self.what}: {self.bad} of {self.n} values out of tolerance, worst {self.worst:.3e}"


def _rows_host(t):
    return None if t is None else t.cpu()


def _every_tile_forward(cfg, wl, st, g, R):
    f, d = cfg.f, cfg.d
    act = [int(e) for e in g.active]
    gu_feat = {e: _quarter_features(f // 64, 64, e) for e in act}
    dn_cols = _quarter_features(d // 128, 128)
    w_gu = _row_weights(wl["w_gu"], act, {e: np.concatenate([gu_feat[e], f + gu_feat[e]]) for e in act})
    w_d = _row_weights(wl["w_d"], act, {e: dn_cols for e in act})
    # the GEMM's input rows: x[perm_token] (x_perm, or gathered in the kernels)
    x_perm = wl["x"].cpu()[torch.as_tensor(g.perm_token)]
    h_all, yp_all, sv_all = _rows_host(st["h"]), _rows_host(st["y_perm"]), _rows_host(st["saved_gu"])
    errs = {k: _Errors(k) for k in ("h", "y_perm", "saved_gu")}
    M = x_perm.shape[0]
    y_rows = np.zeros((M, dn_cols.shape[0]))

    def work(e):
        lo, hi = int(g.offsets[e]), int(g.offsets[e + 1])
        r0 = np.zeros(hi - lo, dtype=np.int64)
        a = x_perm[lo:hi].double().numpy()
        if R is not None:
            a = O.adapter_fwd(a, r0, R[e][None])
        h, saved = _fwd_swiglu(a, r0, w_gu[e])
        hl = h_all[lo:hi].double().numpy()
        yp = _fwd_none(hl, r0, w_d[e])
        out = [("h", hl[:, gu_feat[e]], h), ("y_perm", yp_all[lo:hi].double().numpy()[:, dn_cols], yp)]
        if sv_all is not None:
            sl = sv_all[lo:hi].double().numpy()
            out.append(("saved_gu", np.concatenate([sl[:, gu_feat[e]], sl[:, f + gu_feat[e]]], 1), saved))
        return lo, hi, out, yp

    with ThreadPoolExecutor(THREADS) as ex:
        for lo, hi, out, yp in ex.map(work, act):
            for key, got, want in out:
                errs[key].add(got, want)
            y_rows[lo:hi] = yp
    errs["h"].check()
    errs["y_perm"].check()
    if sv_all is not None:
        errs["saved_gu"].check()
    return y_rows, dn_cols


def _every_tile_backward(cfg, wl, st, bw, g, R):
    f, d = cfg.f, cfg.d
    act = [int(e) for e in g.active]
    dn_groups = {e: _tile_groups(f // 128, e) for e in act}        # dh features (over f)
    gu_groups = _tile_groups(d // 128)                              # dx' features (over d)
    gu_cols = _group_cols(gu_groups)
    w_d = _col_weights(wl["w_d"], act, dn_groups)
    w_gu = _col_weights(wl["w_gu"], act, {e: gu_groups for e in act})
    dyp_all, sv_all = bw["dy_perm"].cpu(), st["saved_gu"].cpu()
    dgu_all, dxp_all = bw["dgu"].cpu(), bw["dx_perm"].cpu()
    x_perm = wl["x"].cpu()[torch.as_tensor(g.perm_token)]
    Rsel = None if R is None else R[:, gu_groups]                   # [E][ng][32][32]
    dR_lib = None
    if R is not None:
        sel = torch.as_tensor(act, device=DEV)
        gsel = torch.as_tensor(gu_groups, device=DEV)
        dR_lib = bw["d_adapter"].index_select(0, sel).index_select(1, gsel).cpu().numpy().astype(np.float64)
    errs = {k: _Errors(k) for k in ("dgu", "dx_perm")}
    dR_bad = []
    M = dyp_all.shape[0]
    dx_rows = np.zeros((M, gu_cols.shape[0]))

    def work(i_e):
        i, e = i_e
        lo, hi = int(g.offsets[e]), int(g.offsets[e + 1])
        r0 = np.zeros(hi - lo, dtype=np.int64)
        cols = _group_cols(dn_groups[e])
        sv = sv_all[lo:hi].double().numpy()
        saved = np.concatenate([sv[:, cols], sv[:, f + cols]], 1)
        dgu = _bwd_groups(dyp_all[lo:hi].double().numpy(), r0, w_d[e], O.EPI_SWIGLU_BWD, saved)
        dl = dgu_all[lo:hi].double().numpy()
        out = [("dgu", np.concatenate([dl[:, cols], dl[:, f + cols]], 1), dgu)]
        dxa = _bwd_groups(dl, r0, w_gu[e])
        bad = None
        if Rsel is not None:
            xr = x_perm[lo:hi].double().numpy()[:, gu_cols]
            dxp, dR = O.adapter_bwd(xr, dxa, r0, Rsel[e][None], 1)
            bound = adapter_grad_bound(xr, dxa, r0, 1)[0]
            err = np.abs(dR_lib[i] - dR[0])
            bad = (int((err > bound).sum()), float(err.max()))
        else:
            dxp = dxa
        out.append(("dx_perm", dxp_all[lo:hi].double().numpy()[:, gu_cols], dxp))
        return lo, hi, out, dxp, bad

    with ThreadPoolExecutor(THREADS) as ex:
        for lo, hi, out, dxp, bad in ex.map(work, list(enumerate(act))):
            for key, got, want in out:
                errs[key].add(got, want)
            dx_rows[lo:hi] = dxp
            if bad is not None:
                dR_bad.append(bad)
    errs["dgu"].check()
    errs["dx_perm"].check()
    if dR_bad:
        nbad = sum(b for b, _ in dR_bad)
        assert nbad == 0, f"d_adapter: {nbad} values above their bound, worst {max(w for _, w in dR_bad):.3e}"
    return dx_rows, gu_cols


def _combine_all_tokens(rows_oracle, g, gates, T, k, out_lib, cols, what):
    """out[t, cols] = bf16(sum_j g_j * row[inv_perm[t, j], cols]) on every token."""
    want = O.combine(rows_oracle, g.inv_perm, gates, T, k)
    got = out_lib.cpu().double().numpy()[:, cols]
    assert_close_final(got, want, what)


# ------------------------------------------------------------------ the runs

def _run(cfg, T, seed):
    wl = synth.make_workload(cfg, DEV, T=T)
    C = cfg.chunk_size
    st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, C,
                       adapter=wl.get("adapter"), train=cfg.train)
    bw = None
    if cfg.train:
        bw = layer.backward(st, wl["dy"], wl["w_gu"], wl["w_d"], adapter=wl.get("adapter"))
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE

    # 1. routing, in full
    topk, gates = O.route_topk(wl["logits"].cpu().numpy(), cfg.k)
    g = O.group_by_expert(topk, cfg.E, C)
    experts = _sample_experts(g, seed)
    rows, _ = _rows_of(g, experts)
    _check_routing_full(st["routing"], wl["x"], topk, gates, g, rows)
    gates_lib = st["routing"].gates.cpu().numpy()

    # the sampled experts' whole chain from the raw inputs
    _sampled_chain(cfg, wl, st, bw, g, gates, experts)

    # 2. every tile of every launch; 3. the combined outputs on every token
    R = f64(wl["adapter"]) if cfg.adapter else None
    y_rows, dn_cols = _every_tile_forward(cfg, wl, st, g, R)
    _combine_all_tokens(y_rows, g, gates_lib, T, cfg.k, st["y"], dn_cols, "y (every token)")
    if cfg.train:
        dx_rows, gu_cols = _every_tile_backward(cfg, wl, st, bw, g, R)
        _combine_all_tokens(dx_rows, g, None, T, cfg.k, bw["dx"], gu_cols, "dx (every token)")
    return wl, st


@pytest.mark.parametrize("T", [128, 2048, 16384])
def test_trillion_int4_layer_full_size(T):
    _run(TRILLION_INT4, T, seed=T)


def test_trillion_int4_chunk_sizes_give_identical_outputs():
    """The chunk size only changes the chunk table: every output bit is the same."""
    cfg = TRILLION_INT4
    T = 2048
    wl = synth.make_workload(cfg, DEV, T=T)
    ys = []
    for C in (8, 16, 32):
        st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, C)
        topk, _ = O.route_topk(wl["logits"].cpu().numpy(), cfg.k)
        g = O.group_by_expert(topk, cfg.E, C)
        nch = int(st["routing"].num_chunks.item())
        assert nch == g.num_chunks
        assert np.array_equal(st["routing"].chunk_offsets.cpu().numpy()[:nch + 1], g.chunk_offsets)
        ys.append(st["y"].clone())
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_zipf_mxfp4_layer_full_size():
    wl, st = _run(ZIPF_MXFP4, ZIPF_MXFP4.T, seed=4)
    counts = np.diff(st["routing"].expert_offsets.cpu().numpy())
    assert (counts == 0).sum() > 0, "the skewed routing should leave some experts empty"


def test_train_int4_step_full_size():
    _run(TRAIN_INT4, TRAIN_INT4.T, seed=5)
