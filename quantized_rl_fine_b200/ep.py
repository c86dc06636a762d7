"""Expert parallelism over the ranks of a process group: the host orchestration
of one MoE layer forward whose experts are split over the ranks.

The Orbit article trains a trillion-parameter INT4 MoE in one 8xB200 node:
about 562 GB of frozen base weights, more than one GPU holds, so the experts
are spread over the node's GPUs. Here rank r owns the E/W consecutive experts
r*E/W .. (r+1)*E/W-1 (their 4-bit weights, and their adapter blocks) and routes
its own tokens. Then:

1. route locally (moe_route_permute): x_perm is expert-major over all E
   experts, so the rows that belong to rank r's experts are one contiguous run;
2. exchange the per-expert row counts (all-to-all of E/W counts per rank);
3. exchange the rows (all-to-all with those counts as split sizes; NCCL over
   NVLink between GPUs, so remote rows land in local HBM before any kernel
   reads them);
4. reorder the received rows to local expert-major order and build the local
   group tables (moe_ep_regroup, direction 0);
5. the grouped GEMMs on the local experts (gate/up + SwiGLU, down);
6. reorder the results back (moe_ep_regroup, direction 1) and return them with
   the reverse all-to-all;
7. combine each rank's own tokens (moe_unpermute_combine).

Every step that touches the rows runs in the library's kernels; this module
only computes split sizes and issues the collectives. The phases are separate
functions so that the exchange between them can be any transport with the
same semantics (torch.distributed here).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import moeq as M
from .synth import QWeightT


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """Experts [lo, hi) owned by `rank`: E/W consecutive experts (E % W == 0)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if E % world != 0:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    n = E // world
    return rank * n, (rank + 1) * n


def send_splits(expert_offsets_host, E: int, world: int) -> list[int]:
    """Rows of the expert-major x_perm that go to each rank (host ints)."""
    off = [int(v) for v in expert_offsets_host]
    out = []
    for r in range(world):
        lo, hi = expert_range(E, world, r)
        out.append(off[hi] - off[lo])
    return out


def exchange_counts(counts: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """counts [E] (rows per expert of this rank's tokens) -> [W, E/W]: the rows
    each source rank sends for each of this rank's experts."""
    E = counts.shape[0]
    recv = torch.empty_like(counts)
    if world == 1:
        recv.copy_(counts)
    else:
        dist.all_to_all_single(recv, counts.contiguous(), group=group)
    return recv.view(world, E // world)


def exchange_rows(rows: torch.Tensor, send: list[int], recv: list[int], group=None) -> torch.Tensor:
    """All-to-all of row runs: send[r] rows go to rank r, recv[s] rows come from s."""
    out = rows.new_empty((sum(recv),) + tuple(rows.shape[1:]))
    if len(send) == 1:
        out.copy_(rows)
    else:
        dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=list(recv),
                               input_split_sizes=list(send), group=group)
    return out


@dataclass
class Dispatch:
    """What one rank keeps between the phases of the layer."""
    routing: M.Routing
    counts: torch.Tensor          # [E] int32, rows per expert of this rank's tokens
    send: list[int]               # rows sent to each rank
    recv_counts: torch.Tensor | None = None   # [W, E/W] int32
    recv: list[int] | None = None             # rows received from each rank


def route(x: torch.Tensor, logits: torch.Tensor, k: int, chunk_size: int, world: int) -> Dispatch:
    """Phase 1: route this rank's tokens over all experts."""
    r = M.moe_route_permute(logits, x, k, chunk_size)
    E = logits.shape[1]
    counts = (r.expert_offsets[1:] - r.expert_offsets[:-1]).to(torch.int32)
    return Dispatch(routing=r, counts=counts, send=send_splits(r.expert_offsets.cpu(), E, world))


def expert_compute(rows: torch.Tensor, recv_counts: torch.Tensor, w_gu: QWeightT, w_d: QWeightT,
                   chunk_size: int, adapter: torch.Tensor | None = None) -> torch.Tensor:
    """Phase 2 on the owner: received rows (source-major) -> local expert-major
    -> gate/up + SwiGLU -> down -> back to source-major order."""
    if rows.shape[0] == 0:                      # no token chose this rank's experts
        return rows.new_empty((0, w_d.N))
    xl, groups = M.moe_ep_regroup(recv_counts, rows, 0, chunk_size)
    h, _ = M.moe_grouped_qgemm_fwd(xl, w_gu, groups, M.EPI_SWIGLU, adapter=adapter)
    yl = M.moe_grouped_qgemm_fwd(h, w_d, groups, M.EPI_NONE)
    return M.moe_ep_regroup(recv_counts, yl, 1)


def combine(dsp: Dispatch, y_perm: torch.Tensor, T: int) -> torch.Tensor:
    """Phase 3: the returned per-slot rows combined per token (gates, slot order)."""
    return M.moe_unpermute_combine(y_perm, dsp.routing, dsp.routing.gates, T, mode=0)


def forward(x: torch.Tensor, logits: torch.Tensor, w_gu_local: QWeightT, w_d_local: QWeightT,
            k: int, chunk_size: int, adapter_local: torch.Tensor | None = None,
            group=None) -> torch.Tensor:
    """The layer forward with the experts split over the ranks of `group`;
    w_*_local hold this rank's E/W experts. Returns y for this rank's tokens."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    dsp = route(x, logits, k, chunk_size, world)
    dsp.recv_counts = exchange_counts(dsp.counts, world, group)
    dsp.recv = dsp.recv_counts.sum(dim=1).cpu().tolist()
    rows = exchange_rows(dsp.routing.x_perm, dsp.send, dsp.recv, group)
    out = expert_compute(rows, dsp.recv_counts, w_gu_local, w_d_local, chunk_size, adapter_local)
    y_perm = exchange_rows(out, dsp.recv, dsp.send, group)
    return combine(dsp, y_perm, x.shape[0])
