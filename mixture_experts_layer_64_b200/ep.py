"""Expert-parallel LatentMoE layer over torch.distributed (one process per GPU).

The paper's deployment (LatentMoE, Section 2.2 "Communication Bottleneck";
Section 3, the paragraph after Eq. (1)) places the N experts on `world` GPUs
and exchanges routed rows in two all-to-alls per layer: the dispatch of
each token's rows to the GPUs that own its experts, and the return of the
expert outputs.  LatentMoE sends the latent rows (width l) instead of the
hidden rows (width d), so both exchanges carry d / l times fewer bytes.

Rank r owns the n = N / world experts [r n, (r + 1) n).  The compute runs in
the library (lmoe_ep_dispatch / lmoe_ep_experts / lmoe_ep_combine); this
module only moves rows between ranks with all_to_all_single (NCCL on GPUs,
gloo on CPU for the plan tests).  Received rows land in this rank's own
memory before any kernel reads them.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist


def exchange_counts(counts: torch.Tensor, world: int, group=None
                    ) -> Tuple[torch.Tensor, List[int], List[int]]:
    """counts [N] int32: rows this rank routes to each expert.  Returns the
    counts this rank receives, recv_counts [world, n] (host; row s = source
    rank s, column e = local expert e), the rows it sends to each rank
    (send_splits) and the rows it receives from each (recv_splits)."""
    N = counts.numel()
    if N % world:
        raise ValueError(f"{N} experts do not split over {world} ranks")
    n = N // world
    recv = torch.empty_like(counts)
    dist.all_to_all_single(recv, counts, group=group)
    send_splits = counts.view(world, n).sum(1).tolist()
    recv_counts = recv.view(world, n).cpu()
    recv_splits = recv_counts.sum(1).tolist()
    return recv_counts, send_splits, recv_splits


def exchange_rows(rows: torch.Tensor, send_splits: List[int], recv_splits: List[int],
                  group=None) -> torch.Tensor:
    """Sends rows[block q] to rank q (blocks in rank order, sizes send_splits)
    and returns the blocks received, sources in rank order."""
    out = torch.empty((sum(recv_splits),) + tuple(rows.shape[1:]), dtype=rows.dtype,
                      device=rows.device)
    dist.all_to_all_single(out, rows, output_split_sizes=recv_splits,
                           input_split_sizes=send_splits, group=group)
    return out


class ExpertParallelLayer:
    """One rank of an expert-parallel LatentMoE layer.  `layer` is this
    rank's LatentMoELayer (weights set, workspace reserved); max_recv_rows
    bounds the rows one rank may receive per call (at most world * T * k)."""

    def __init__(self, layer, max_recv_rows: int, group=None):
        self.layer = layer
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if layer.N % self.world:
            raise ValueError(f"{layer.N} experts do not split over {self.world} ranks")
        layer.ep_reserve(max_recv_rows)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        L = self.layer
        send_rows, send_gates, counts = L.ep_dispatch(x)
        recv_counts, send_splits, recv_splits = exchange_counts(counts, self.world, self.group)
        recv_rows = exchange_rows(send_rows, send_splits, recv_splits, self.group)
        recv_gates = exchange_rows(send_gates, send_splits, recv_splits, self.group)
        out_rows = L.ep_experts(recv_rows, recv_gates, recv_counts, self.rank, self.world)
        back = exchange_rows(out_rows, recv_splits, send_splits, self.group)
        return L.ep_combine(x, back, out)

    __call__ = forward
