"""Expert-parallel MoE layer: the experts split over torch.distributed ranks.

"Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary), section
"Training Infrastructure and Stabilization Techniques": expert parallelism,
with all-to-all communication that routes tokens to the GPU holding their
selected experts; section "Mixture-of-Experts (MoE) in Jamba: Router, Top-K,
and Load Balancing": MoE layers need all-to-all communication under expert
parallelism.

With G ranks and E experts (E % G == 0), rank g owns the E/G consecutive
experts ``g*E/G .. (g+1)*E/G - 1`` and only their INT8 weights.  Each rank
routes its own tokens (the router is replicated), then

1. ``dispatch``: the library groups the token->expert assignments by expert,
   which orders them by owner rank, and packs the token rows in that order
   (``jmoe_ep_dispatch``);
2. all-to-all: rank r receives, from every rank in rank order, the rows for
   its experts and their expert indices within r;
3. ``experts``: ``jmoe_forward`` on the received rows with the owned experts
   (one expert per row, gate 1);
4. all-to-all back, with the splits reversed;
5. ``combine``: each token's returned rows, weighted by its gates, summed in
   fp32 and rounded once (``jmoe_ep_combine``).

The exchanges are ``torch.distributed.all_to_all_single`` (NCCL over
NVLink between GPUs): rows travel as raw bytes and land in local buffers, so
no kernel reads another GPU's memory.  The split sizes come from the grouping
offsets, which the host reads once per call.
"""
from __future__ import annotations

from typing import List, Sequence

from . import (JMOE_PATH_AUTO, jmoe_ep_combine, jmoe_ep_dispatch, jmoe_forward, make_desc)


def owner_splits(offsets_host: Sequence[int], E: int, G: int) -> List[int]:
    """Rows for each rank, from the grouping offsets [E+1]: rank r owns the
    experts r*E/G .. (r+1)*E/G - 1, whose rows are contiguous."""
    if E % G:
        raise ValueError(f"{E} experts do not split over {G} ranks")
    el = E // G
    return [int(offsets_host[(r + 1) * el]) - int(offsets_host[r * el]) for r in range(G)]


def exchange_rows(send, send_splits: Sequence[int], recv_splits: Sequence[int], group=None):
    """All-to-all of row blocks: rank r's block i goes to rank i.  The rows
    move as bytes, so any dtype and row width works on any backend."""
    import torch
    import torch.distributed as dist

    send = send.contiguous()
    row_shape = tuple(send.shape[1:])
    b = send.view(torch.uint8).reshape(send.shape[0], -1)
    out = torch.empty((sum(recv_splits), b.shape[1]), dtype=torch.uint8, device=send.device)
    dist.all_to_all_single(out, b, output_split_sizes=list(recv_splits),
                           input_split_sizes=list(send_splits), group=group)
    return out.view(send.dtype).reshape((sum(recv_splits),) + row_shape)


def exchange_counts(send_splits: Sequence[int], device, group=None) -> List[int]:
    """Every rank learns how many rows each rank sends it."""
    import torch
    import torch.distributed as dist

    s = torch.tensor(list(send_splits), dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return [int(v) for v in r.cpu()]


class JmoeEpOps:
    """The per-rank compute of the expert-parallel layer, in the library's
    kernels: this rank's experts are given as slices [E/G, ...] of the
    quantised weights (w_gu, s_gu, w_d, s_d as for make_desc)."""

    def __init__(self, w_gu, s_gu, w_d, s_d, E: int, path: int = JMOE_PATH_AUTO):
        self.E = E
        self.desc = make_desc(w_gu, s_gu, w_d, s_d, top_k=1, path=path)
        self._weights = (w_gu, s_gu, w_d, s_d)  # keep alive for the descriptor

    def dispatch(self, x, ids, G: int):
        offsets, _perm, inv, x_send, local_ids = jmoe_ep_dispatch(x, ids, self.E, G)
        return offsets.cpu().tolist(), inv, x_send, local_ids

    def experts(self, x_recv, ids_recv):
        import torch

        R = x_recv.shape[0]
        if R == 0:
            return torch.empty_like(x_recv)
        ones = torch.ones((R, 1), dtype=torch.float32, device=x_recv.device)
        return jmoe_forward(self.desc, x_recv, ids_recv.reshape(R, 1).contiguous(), ones)

    def combine(self, y_back, inv, gates):
        return jmoe_ep_combine(y_back.contiguous(), inv, gates)


def ep_forward(ops, x, ids, gates, E: int, group=None):
    """One expert-parallel MoE layer forward on this rank's tokens.

    x [T, d], ids int32 [T, top_k] (global expert ids), gates fp32 [T, top_k];
    ``ops`` does the per-rank compute (JmoeEpOps on GPUs).  Returns [T, d]."""
    import torch.distributed as dist

    G = dist.get_world_size(group)
    offsets, inv, x_send, local_ids = ops.dispatch(x, ids, G)
    send = owner_splits(offsets, E, G)
    n = sum(send)
    recv = exchange_counts(send, x.device, group)
    x_recv = exchange_rows(x_send[:n], send, recv, group)
    ids_recv = exchange_rows(local_ids[:n], send, recv, group)
    y_recv = ops.experts(x_recv, ids_recv)
    y_back = exchange_rows(y_recv, recv, send, group)
    return ops.combine(y_back, inv, gates)


def local_slices(w_gu, s_gu, w_d, s_d, E: int, G: int, rank: int):
    """This rank's experts out of the full quantised weights (views)."""
    el = E // G
    sl = slice(rank * el, (rank + 1) * el)
    return w_gu[sl], s_gu[sl], w_d[sl], s_d[sl]
