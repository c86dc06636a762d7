"""The Orbit article's own scheme, kept only as a comparator of the fused path.

Orbit article, section "technical details", paragraph "Active-expert-chunked
dequantization": the experts the router selects are taken in fixed-size
chunks; each chunk's low-bit weights are dequantized into a temporary
high-precision buffer, the grouped GEMM runs on that buffer, and the buffer is
released, so the temporary memory is bounded by one chunk instead of the
whole model.

Here each chunk of C active experts is dequantized with this library's
moe_dequant_experts (the same bits as the fused kernels) into a BF16 buffer
that PyTorch allocates, the GEMMs run as cuBLAS BF16 matrix products (one per
expert of the chunk), the SwiGLU is applied with PyTorch elementwise ops, and
the buffer is freed before the next chunk. It reports the peak of the
temporary memory. The product path is the fused kernels of layer.py; nothing
there calls this module.
"""

from __future__ import annotations

import torch
import torch.nn.functional as F

from . import moeq as M
from .synth import QWeightT


def _chunks(active: list[int], C: int):
    for i in range(0, len(active), C):
        yield active[i:i + C]


def forward(x_perm: torch.Tensor, routing: M.Routing, w_gu: QWeightT, w_d: QWeightT,
            chunk_size: int, swiglu: bool = True) -> tuple[torch.Tensor, int]:
    """Gate/up + SwiGLU + down (or one up-projection when swiglu is False) of
    the permuted rows, chunk by chunk through temporary BF16 weights.

    Returns (the per-slot output rows [M, N_out], the peak of the memory the
    call allocated beyond its output, in bytes)."""
    dev = x_perm.device
    off = routing.expert_offsets.cpu().tolist()
    A = int(routing.num_active.item())
    active = routing.active[:A].cpu().tolist()
    M_rows = x_perm.shape[0]
    n_out = w_d.N if swiglu else w_gu.N
    out = torch.empty((M_rows, n_out), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    f = w_gu.N // 2
    for chunk in _chunks(active, chunk_size):
        ids = torch.tensor(chunk, dtype=torch.int32, device=dev)
        wbuf = M.moe_dequant_experts(w_gu, ids)                     # [C, N, K] bf16, temporary
        hs = []
        for i, e in enumerate(chunk):
            rows = x_perm[off[e]:off[e + 1]]
            acc = rows @ wbuf[i].t()
            if swiglu:
                hs.append((F.silu(acc[:, :f].float()) * acc[:, f:].float()).to(torch.bfloat16))
            else:
                out[off[e]:off[e + 1]] = acc
        del wbuf
        if swiglu:
            dbuf = M.moe_dequant_experts(w_d, ids)
            for i, e in enumerate(chunk):
                out[off[e]:off[e + 1]] = hs[i] @ dbuf[i].t()
            del dbuf, hs
    torch.cuda.synchronize(dev)
    peak = torch.cuda.max_memory_allocated(dev) - base
    return out, int(peak)
