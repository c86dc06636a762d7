"""One MoE layer step through the C ABI: the orchestration of the calls only.

forward : route_permute -> fwd GEMM (gate/up, SwiGLU [, adapter]) -> fwd GEMM
          (down) -> combine
backward: scatter (gate-scaled dy) -> bwd_dx down (SwiGLU backward) ->
          bwd_dx gate/up [+ adapter backward] -> combine (unpermute-sum)
up-projection only: route_permute -> fwd GEMM (no epilogue)

With the adapter the permuted token rows are never written: routing returns
the permutation only and the adapter kernels read row p as x[perm_token[p]]
(plain loads, at no extra cost). Without it the routing call writes x_perm
and the gate/up GEMM reads it through its tensor map; gather=True makes the
GEMM gather the rows itself instead (same bits; at 341 rows per expert on
B200 its gathering producer is about 2.2x slower than the tensor-map copy,
because each stage is handed over only once its row copies have landed).
"""

from __future__ import annotations

import torch

from . import moeq as M
from .synth import QWeightT


def forward(x: torch.Tensor, logits: torch.Tensor, w_gu: QWeightT, w_d: QWeightT, k: int,
            chunk_size: int, adapter: torch.Tensor | None = None, train: bool = False,
            stream=None, gather: bool | None = None) -> dict:
    T = x.shape[0]
    if gather is None:
        gather = adapter is not None
    r = M.moe_route_permute(logits, None if gather else x, k, chunk_size, stream=stream)
    a, a_rows = (x, r.perm_token) if gather else (r.x_perm, None)
    h, saved = M.moe_grouped_qgemm_fwd(a, w_gu, r, M.EPI_SWIGLU, adapter=adapter,
                                       save_gu=train, stream=stream, a_rows=a_rows)
    y_perm = M.moe_grouped_qgemm_fwd(h, w_d, r, M.EPI_NONE, stream=stream)
    y = M.moe_unpermute_combine(y_perm, r, r.gates, T, mode=0, stream=stream)
    return dict(routing=r, x=x, a=a, a_rows=a_rows, h=h, saved_gu=saved, y_perm=y_perm, y=y)


def backward(state: dict, dy: torch.Tensor, w_gu: QWeightT, w_d: QWeightT,
             adapter: torch.Tensor | None = None, stream=None) -> dict:
    r: M.Routing = state["routing"]
    T = dy.shape[0]
    dy_perm = M.moe_unpermute_combine(dy, r, r.gates, T, mode=1, stream=stream)
    dgu = M.moe_grouped_qgemm_bwd_dx(dy_perm, w_d, r, M.EPI_SWIGLU_BWD, saved_gu=state["saved_gu"],
                                     stream=stream)
    if adapter is not None:
        dx_perm, d_adapter = M.moe_grouped_qgemm_bwd_dx(dgu, w_gu, r, M.EPI_NONE, adapter=adapter,
                                                        a=state["a"], a_rows=state["a_rows"],
                                                        stream=stream)
    else:
        dx_perm = M.moe_grouped_qgemm_bwd_dx(dgu, w_gu, r, M.EPI_NONE, stream=stream)
        d_adapter = None
    dx = M.moe_unpermute_combine(dx_perm, r, None, T, mode=0, stream=stream)
    return dict(dy_perm=dy_perm, dgu=dgu, dx_perm=dx_perm, dx=dx, d_adapter=d_adapter)


def up_projection(x: torch.Tensor, logits: torch.Tensor, w_up: QWeightT, k: int, chunk_size: int,
                  stream=None, gather: bool = False) -> dict:
    r = M.moe_route_permute(logits, None if gather else x, k, chunk_size, stream=stream)
    a, a_rows = (x, r.perm_token) if gather else (r.x_perm, None)
    out = M.moe_grouped_qgemm_fwd(a, w_up, r, M.EPI_NONE, stream=stream, a_rows=a_rows)
    return dict(routing=r, a=a, a_rows=a_rows, out=out)
