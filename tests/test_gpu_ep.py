"""Expert parallelism on one GPU: the regroup kernel against its definition,
and a two-rank layer forward whose exchange is emulated by copies.

The emulation runs the ranks' phases one after the other on one GPU and
moves the row runs between them with plain tensor copies, in exactly the
layout the all-to-all delivers; no kernel waits on another. The result must
equal the single-GPU layer on the same tokens within the final-output
tolerance, and the oracle as well.
"""

import numpy as np
import pytest
import torch

import oracle as O
from quantized_rl_fine_b200 import ep, layer, moeq, synth
from quantized_rl_fine_b200.configs import MoEConfig

import _ep_reference as ref
from _common import assert_close_final, bf16_bits, f64, oracle_qweight

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,E_loc,D,C", [(4, 96, 128, 8), (2, 3, 64, 2), (8, 48, 7168, 16), (1, 5, 8, 1)])
def test_regroup_kernel_matches_the_definition(W, E_loc, D, C):
    rng = np.random.default_rng(W * 1000 + E_loc)
    counts = rng.integers(0, 6, size=(W, E_loc)).astype(np.int32)
    counts[:, rng.integers(0, E_loc)] = 0            # an expert nobody chose
    R = int(counts.sum())
    rows = torch.randn((R, D), generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).cuda()
    ct = torch.from_numpy(counts).cuda()
    out, grp = moeq.moe_ep_regroup(ct, rows, 0, C)
    order = ref.expert_major_order(counts)
    assert np.array_equal(bf16_bits(out), bf16_bits(rows)[order])
    offs, active, chunks = ref.local_tables(counts, C)
    A = int(grp.num_active.item())
    nch = int(grp.num_chunks.item())
    assert np.array_equal(grp.expert_offsets.cpu().numpy(), offs)
    assert A == active.shape[0] and np.array_equal(grp.active.cpu().numpy()[:A], active)
    assert nch == chunks.shape[0] - 1 and np.array_equal(grp.chunk_offsets.cpu().numpy()[:nch + 1], chunks)
    back = moeq.moe_ep_regroup(ct, out, 1)
    assert torch.equal(back, rows)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


def test_regroup_kernel_flags_counts_that_do_not_sum_to_R():
    ct = torch.tensor([[2, 1], [0, 3]], dtype=torch.int32, device="cuda")
    rows = torch.zeros((5, 8), dtype=torch.bfloat16, device="cuda")      # counts sum to 6
    moeq.moe_ep_regroup(ct, rows, 1)
    assert moeq.moe_get_device_error() == moeq.DEVERR_BAD_OFFSETS


def _local(w, lo, hi):
    return synth.QWeightT(w.fmt, w.packed[lo:hi].contiguous(), w.scales[lo:hi].contiguous())


CFG = MoEConfig("ep_int4", E=16, k=4, d=256, f=256, T=400, fmt="int4", swiglu=True,
                logits="normal", adapter=False, train=False, seed=3301)


def test_two_rank_forward_with_emulated_exchange():
    W = 2
    wl = synth.make_workload(CFG, "cuda")
    T = CFG.T
    shards = [(0, T // 2), (T // 2, T)]
    # phase 1 on each rank
    dsp = [ep.route(wl["x"][a:b], wl["logits"][a:b], CFG.k, CFG.chunk_size, W) for a, b in shards]
    # emulated count and row exchange: rank r receives, from each source s,
    # s's counts and rows of r's experts, source-major
    outs = []
    for r in range(W):
        lo, hi = ep.expert_range(CFG.E, W, r)
        recv_counts = torch.stack([d.counts[lo:hi] for d in dsp]).contiguous()
        runs = []
        for d in dsp:
            off = d.routing.expert_offsets.cpu().tolist()
            runs.append(d.routing.x_perm[off[lo]:off[hi]])
        rows = torch.cat(runs).contiguous()
        out = ep.expert_compute(rows, recv_counts, _local(wl["w_gu"], lo, hi),
                                _local(wl["w_d"], lo, hi), CFG.chunk_size)
        outs.append((recv_counts.sum(dim=1).cpu().tolist(), out))
    # emulated return: source s gets, from each owner r, the run it sent there
    for s, (a, b) in enumerate(shards):
        parts = []
        for r in range(W):
            recv, out = outs[r]
            start = sum(recv[:s])
            parts.append(out[start:start + recv[s]])
        y_perm = torch.cat(parts).contiguous()
        y = ep.combine(dsp[s], y_perm, b - a)
        single = layer.forward(wl["x"][a:b], wl["logits"][a:b], wl["w_gu"], wl["w_d"], CFG.k,
                               CFG.chunk_size)["y"]
        assert_close_final(f64(y), f64(single), f"rank {s} y against the single-GPU layer")
        want = O.moe_forward(f64(wl["x"][a:b]), wl["logits"][a:b].cpu().numpy(), CFG.k,
                             CFG.chunk_size, oracle_qweight(wl["w_gu"]), oracle_qweight(wl["w_d"]))
        assert_close_final(f64(y), want["y"], f"rank {s} y against the oracle")
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE
