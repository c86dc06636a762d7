"""moe_route_permute_noalloc: routing for callers that cannot allocate.

Some callers of the routing step cannot give the library scratch memory: a
serving runtime that reserves all device memory in one arena at start-up, code
that enqueues work during CUDA graph capture (where cudaMalloc is not allowed),
or a C host without a caching allocator, for which a cudaMalloc/cudaFree pair
per call would synchronize the device. This entry point keeps its histogram
scratch in a fixed array inside the library instead.

The test calls it through the C ABI twice in a row and checks every output
against moe_route_permute, which uses a caller workspace. Both problems are
large enough for the histogram path (more than 1024 tokens), which is the one
that uses the fixed array: the first fills 47 x 384 histogram entries, the
second reads 32 x 128 of them back after rewriting them, so it runs over the
first call's leftovers.
"""

import ctypes

import pytest
import torch

from quantized_rl_fine_b200 import moeq

pytestmark = pytest.mark.gpu


def _noalloc(logits, x, k, chunk_size):
    T, E = logits.shape
    dev = logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    r = moeq.Routing(
        topk_idx=torch.empty((T, k), **i32), gates=torch.empty((T, k), dtype=torch.float32, device=dev),
        expert_offsets=torch.empty(E + 1, **i32), active=torch.empty(E, **i32),
        num_active=torch.empty(1, **i32), chunk_offsets=torch.empty(E + 1, **i32),
        num_chunks=torch.empty(1, **i32), perm_token=torch.empty(T * k, **i32),
        inv_perm=torch.empty(T * k, **i32),
        x_perm=torch.empty((T * k, x.shape[1]), dtype=torch.bfloat16, device=dev), E=E, k=k)
    st = moeq.lib().moe_route_permute_noalloc(
        logits.data_ptr(), x.data_ptr(), T, E, k, x.shape[1], chunk_size, r.topk_idx.data_ptr(),
        r.gates.data_ptr(), r.expert_offsets.data_ptr(), r.active.data_ptr(),
        r.num_active.data_ptr(), r.chunk_offsets.data_ptr(), r.num_chunks.data_ptr(),
        r.perm_token.data_ptr(), r.inv_perm.data_ptr(), r.x_perm.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == moeq.MOE_OK, moeq.STATUS_NAMES.get(st, st)
    return r


def test_noalloc_routing_matches_workspace_routing_twice_in_a_row():
    cases = [(3000, 384, 8, 16, 11), (2048, 128, 4, 8, 12)]    # larger first, then smaller
    for T, E, k, C, seed in cases:
        g = torch.Generator().manual_seed(seed)
        logits = torch.randn((T, E), generator=g)
        logits[: T // 4] = torch.round(logits[: T // 4] * 2) / 2   # exact ties
        x = torch.randn((T, 128), generator=g).to(torch.bfloat16)
        logits, x = logits.cuda(), x.cuda()
        want = moeq.moe_route_permute(logits, x, k, C)
        got = _noalloc(logits, x, k, C)
        torch.cuda.synchronize()
        A = int(want.num_active.item())
        nch = int(want.num_chunks.item())
        assert int(got.num_active.item()) == A and int(got.num_chunks.item()) == nch
        assert torch.equal(got.topk_idx, want.topk_idx)
        assert torch.equal(got.gates, want.gates)                # same top-k kernel
        assert torch.equal(got.expert_offsets, want.expert_offsets)
        assert torch.equal(got.active[:A], want.active[:A])
        assert torch.equal(got.chunk_offsets[: nch + 1], want.chunk_offsets[: nch + 1])
        assert torch.equal(got.perm_token, want.perm_token)
        assert torch.equal(got.inv_perm, want.inv_perm)
        assert torch.equal(got.x_perm, want.x_perm)
    assert moeq.moe_get_device_error() == moeq.DEVERR_NONE


def test_noalloc_rejects_problems_beyond_its_fixed_scratch():
    # ceil(T/64) * E histogram entries must fit the 2^20-entry array; this does not.
    p = 0x10000
    T, E = 64 * 1025, 1024
    st = moeq.lib().moe_route_permute_noalloc(p, p, T, E, 8, 128, 8, p, p, p, p, p, p, p, p, p, p,
                                              None)
    assert st == 4   # MOE_ERR_WORKSPACE, nothing launched
