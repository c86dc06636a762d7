"""Full-size parity of the layer workloads (trillion-shaped INT4 at T = 128,
2048 and 16384; skewed-routing MXFP4; the INT4 training step with adapter).

At these sizes the oracle cannot run the whole layer in seconds, so:
- routing (top-k, gates, offsets, active list, chunk table, permutation) is
  compared bit-exactly in full, and the permuted rows on every row of the
  sampled experts;
- for a sample of experts (first and last active, the busiest, one drawn at
  random) the oracle computes the whole chain of those experts' rows from the
  raw inputs (adapter, gate/up + SwiGLU, down, and for training the gate-scaled
  gather, SwiGLU backward, gate/up backward, adapter backward) and every row
  is compared: per-slot intermediates within 2e-2 + one BF16 ulp; the FP32
  adapter gradient of each sampled expert within 2e-2 plus the spread that
  one-ulp differences of its BF16 input dx' can cause (and rel-L2 <= 5e-3);
- the combined outputs y and dx, which mix all experts, are checked on 512
  sampled tokens (and the first and last) by the combine's definition applied
  to the library's own per-slot rows (a property that holds at any size), with
  the final-output criterion.
"""

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import layer, moeq, synth
from quantized_rl_fine_b200.configs import TRAIN_INT4, TRILLION_INT4, ZIPF_MXFP4

from _common import (adapter_grad_bound, assert_close_bounded, assert_close_final,
                     assert_close_intermediate, bf16_bits, f64)

pytestmark = pytest.mark.gpu

DEV = "cuda"


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


def _sample_tokens(T, seed, n=512):
    rng = np.random.default_rng(seed + 1)
    return np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, size=min(n, T))]))


def _combine_tokens(rows_t, inv_perm, gates, tokens, k):
    """The combine's definition on a subset of tokens, over the given per-slot rows."""
    idx = np.asarray(inv_perm).reshape(-1, k)[tokens].reshape(-1)
    g = None if gates is None else np.asarray(gates).reshape(-1, k)[tokens]
    return O.combine(_take(rows_t, idx), np.arange(idx.shape[0]), g, tokens.shape[0], k)


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

    # routing, in full
    topk, gates = O.route_topk(wl["logits"].cpu().numpy(), cfg.k)
    g = O.group_by_expert(topk, cfg.E, C)
    experts = _sample_experts(g, seed)
    rows, local = _rows_of(g, experts)
    _check_routing_full(st["routing"], wl["x"], topk, gates, g, rows)

    # the sampled experts' chain, computed by the oracle from the raw inputs
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
    assert_close_intermediate(_take(st["h"], rows), h, "h")
    assert_close_intermediate(_take(st["y_perm"], rows), y_perm, "y_perm")

    # y by the combine's definition over the library's per-slot rows
    toks = _sample_tokens(T, seed)
    y_def = _combine_tokens(st["y_perm"], g.inv_perm, gates, toks, cfg.k)
    assert_close_final(_take(st["y"], toks), y_def, "y")

    if cfg.train:
        assert_close_intermediate(_take(st["saved_gu"], rows), saved, "saved_gu")
        dy_perm = O.gather_scaled(f64(wl["dy"]), g.inv_perm, gates, T, cfg.k)[rows]
        assert np.array_equal(bf16_bits(bw["dy_perm"].index_select(0, torch.as_tensor(rows, device=DEV))),
                              O.bf16_bits_from_values(dy_perm))
        dgu = O.grouped_gemm_bwd_dx(dy_perm, local, wd, O.EPI_SWIGLU_BWD, saved)
        assert_close_intermediate(_take(bw["dgu"], rows), dgu, "dgu")
        dxa = O.grouped_gemm_bwd_dx(dgu, local, wgu, O.EPI_NONE)
        if cfg.adapter:
            dx_perm, dR = O.adapter_bwd(x_rows, dxa, local, R, len(experts))
            got_dR = bw["d_adapter"].index_select(0, torch.as_tensor(experts, device=DEV))
            bound = adapter_grad_bound(x_rows, dxa, local, len(experts))
            assert_close_bounded(got_dR.cpu().numpy().astype(np.float64), dR, bound, "d_adapter")
        else:
            dx_perm = dxa
        assert_close_intermediate(_take(bw["dx_perm"], rows), dx_perm, "dx_perm")
        dx_def = _combine_tokens(bw["dx_perm"], g.inv_perm, None, toks, cfg.k)
        assert_close_final(_take(bw["dx"], toks), dx_def, "dx")
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
