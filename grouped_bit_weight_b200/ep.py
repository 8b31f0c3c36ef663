"""Expert-parallel sharding of the grouped 4-bit expert matmul.

"grouped-nf4-gemm 0.43.0", opening lines: one launch multiplies the routed
rows of every active expert by that expert's packed weights.  Split across
ranks by expert, each rank holds the packed weights of experts
[rank * E_local, (rank + 1) * E_local) only, and a layer becomes

  dispatch  every routed row (token t, slot s, expert topk_ids[t, s]) goes to
            the rank that owns its expert: one all-to-all of the per-expert
            row counts, one of the activation rows;
  compute   one grouped launch per rank over the rows it received, sorted by
            local expert through row_to_token (the kernels gather the rows;
            nothing is copied into expert order);
  combine   the output rows go back to the ranks they came from (one
            all-to-all) and land at their (token, slot) place.

The exchange is plain `torch.distributed.all_to_all_single` (NCCL over
NVLink on GPUs; gloo on CPU for the host-side tests), each rank's kernels
touching only its own memory.  Weighting and summing the k slots of a token
(the router's combine weights) stays with the caller: it is routing, not
this path.

Row order.  The dispatch sorts a rank's routed rows by global expert id
(stable), which orders them by owner rank and, within a rank, by local
expert; the receiver's buffer is therefore source-major and expert-sorted
within each source, and one stable sort of the received rows' local expert
ids gives row_to_token and expert_offsets for the grouped call.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional

import torch


@dataclass
class Dispatch:
    """What a dispatch leaves for the local call and the combine."""
    x: torch.Tensor               # [R, K] rows received, source-major
    expert_offsets: torch.Tensor  # [E_local + 1] int32, over the expert-sorted rows
    row_to_token: torch.Tensor    # [R] int32: sorted row p reads x row row_to_token[p]
    order: torch.Tensor           # [T * k] int64: routed rows (t * k + s) in send order
    send_split: List[int]         # rows sent to each rank
    recv_split: List[int]         # rows received from each rank
    T: int
    k: int


class ExpertParallel:
    """Experts [rank * E_local, (rank + 1) * E_local) live on this rank of
    `group` (the default process group when None); E % world == 0."""

    def __init__(self, num_experts: int, group=None):
        import torch.distributed as dist
        self._dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if num_experts < 1 or num_experts % self.world:
            raise ValueError(f"ExpertParallel: {num_experts} experts do not split evenly over "
                             f"{self.world} ranks")
        self.num_experts = num_experts
        self.E_local = num_experts // self.world
        self.first_expert = self.rank * self.E_local

    def dispatch(self, x: torch.Tensor, topk_ids: torch.Tensor) -> Dispatch:
        """Send each routed row of x [T, K] (T tokens, topk_ids [T, k] global
        expert ids) to the rank that owns its expert."""
        dist = self._dist
        if x.dim() != 2 or topk_ids.dim() != 2 or topk_ids.shape[0] != x.shape[0]:
            raise ValueError("dispatch: x must be [T, K] and topk_ids [T, k]")
        T, K = x.shape
        k = topk_ids.shape[1]
        ids = topk_ids.reshape(-1).to(device=x.device, dtype=torch.int64)
        if ids.numel() and (int(ids.min()) < 0 or int(ids.max()) >= self.num_experts):
            raise ValueError(f"dispatch: expert ids must lie in [0, {self.num_experts})")
        order = torch.sort(ids, stable=True).indices
        # rows for (owner rank d, its local expert j), exchanged so that each
        # rank learns how many rows every source sends to each of its experts
        send_mat = torch.bincount(ids, minlength=self.num_experts).view(self.world, self.E_local)
        recv_mat = torch.empty_like(send_mat)
        dist.all_to_all_single(recv_mat.view(-1), send_mat.reshape(-1).contiguous(),
                               group=self.group)
        send_split = send_mat.sum(1).tolist()
        recv_split = recv_mat.sum(1).tolist()
        send_x = x.index_select(0, order // k)
        recv_x = x.new_empty((sum(recv_split), K))
        dist.all_to_all_single(recv_x, send_x, recv_split, send_split, group=self.group)
        # local expert of every received row: per source, experts in order
        local_ids = torch.repeat_interleave(
            torch.arange(self.E_local, device=x.device).repeat(self.world), recv_mat.reshape(-1))
        row_to_token = torch.sort(local_ids, stable=True).indices.to(torch.int32)
        offsets = torch.zeros(self.E_local + 1, dtype=torch.int32, device=x.device)
        offsets[1:] = torch.cumsum(recv_mat.sum(0), 0)
        return Dispatch(recv_x, offsets, row_to_token, order, send_split, recv_split, T, k)

    def combine(self, out: torch.Tensor, d: Dispatch) -> torch.Tensor:
        """Return the local call's output rows out [R, N] (expert-sorted, as
        the grouped call writes them) to their source ranks; the result is
        y [T, k, N] with y[t, s] the row of token t's slot s."""
        dist = self._dist
        R = d.row_to_token.numel()
        if out.dim() != 2 or out.shape[0] != R:
            raise ValueError(f"combine: out must be [{R}, N]")
        N = out.shape[1]
        back_in = torch.empty_like(out)  # received order
        back_in.index_copy_(0, d.row_to_token.long(), out)
        back = out.new_empty((sum(d.send_split), N))
        dist.all_to_all_single(back, back_in, d.send_split, d.recv_split, group=self.group)
        y = out.new_empty((d.T * d.k, N))
        y.index_copy_(0, d.order, back)
        return y.view(d.T, d.k, N)

    def run(self, x: torch.Tensor, topk_ids: torch.Tensor,
            local: Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]
            ) -> torch.Tensor:
        """dispatch -> local(x_recv, expert_offsets, row_to_token) -> combine."""
        d = self.dispatch(x, topk_ids)
        return self.combine(local(d.x, d.expert_offsets, d.row_to_token), d)


def ep_grouped_gemm(ep: ExpertParallel, x: torch.Tensor, topk_ids: torch.Tensor,
                    packed: torch.Tensor, scale: torch.Tensor, fmt: str = "nf4",
                    mode: str = "auto", out_features: Optional[int] = None) -> torch.Tensor:
    """Expert-parallel grouped forward: y[t, s] = x[t] @ W_{topk_ids[t, s]}^T
    with this rank's experts' packed weights (packed [E_local, N, K/2],
    scale the matching absmax or e8m0 scales).  Returns y [T, k, N] bf16."""
    from . import gmxfp4_grouped_gemm, gnf4_grouped_gemm
    if fmt not in ("nf4", "mxfp4"):
        raise ValueError(f"ep_grouped_gemm: unknown format {fmt!r}")
    if packed.dim() < 2 or packed.shape[0] != ep.E_local:
        raise ValueError(f"ep_grouped_gemm: packed must hold this rank's {ep.E_local} experts")
    if out_features is not None and packed.shape[1] != out_features:
        raise ValueError("ep_grouped_gemm: packed weights have the wrong N")
    fn = gnf4_grouped_gemm if fmt == "nf4" else gmxfp4_grouped_gemm
    return ep.run(x, topk_ids, lambda xr, off, r2t: fn(xr, packed, scale, off, r2t, mode=mode))
