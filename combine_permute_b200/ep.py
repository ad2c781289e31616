"""Expert-parallel dispatch and combine between GPUs, one process per GPU.

The exchange step of an expert-parallel MoE layer (Mooncake PR #4581:
dispatch / combine kernels across ranks over NCCL; TensorRT-LLM PR #9592:
"Alltoall comm", one rank's experts being the window local_expert_offset ..
+ num_local_experts).  R ranks each own El = E / R consecutive experts:
rank r owns experts [r*El, (r+1)*El).

ep_dispatch, on every rank:
  1. moe_prepare over all E experts, then moe_dispatch_rows: the dispatched
     rows are sorted by expert, hence by destination rank, so the rows for
     rank r are one contiguous block;
  2. the expert counts, viewed [R, El], go to their owners (all-to-all of
     El ints per pair): each rank learns what every source will send it;
  3. the row blocks cross (all-to-all with per-rank sizes) into a buffer
     holding the source blocks in source order;
  4. moe_ep_recv_layout gives the layout grouped by local expert, then
     source, then the source's order, and one row gather puts the rows
     there.  The grouped rows and their expert offsets are what the expert
     stage (a grouped GEMM) takes.

ep_combine reverses steps 4 and 3 for the expert outputs and runs
moe_combine on the source rank, which weights and sums every token's k
outputs exactly as on one GPU.

The data plane is torch.distributed.all_to_all_single on the given process
group (NCCL between GPUs; gloo between CPU processes).  The per-rank steps
come from an ``ops`` object; the default, ``CudaOps``, is this library's
kernels.  The module has no other implementation of them: a caller without
the CUDA library gets the binding's error.  Passing another ``ops`` is how a
test drives the same exchange logic on CPU ranks.

ep_dispatch_peer and ep_combine_peer are the same exchange without
all-to-alls: every source's dispatch kernel stores its rows straight into
the owners' grouped buffers (other GPUs' memory mapped into this process)
and its combine kernel reads the expert outputs straight back from them;
the only collectives are an all-gather of the expert counts and two
barriers.
"""

from __future__ import annotations

from typing import List, NamedTuple, Optional

import torch
import torch.distributed as dist

from . import (moe_combine, moe_dispatch_rows, moe_ep_combine_peer, moe_ep_dispatch_peer,
               moe_ep_peer_layout, moe_ep_recv_layout, moe_prepare)

__all__ = ["CudaOps", "EpHandle", "ep_dispatch", "ep_combine", "EpPeerHandle",
           "ep_dispatch_peer", "ep_combine_peer"]


class CudaOps:
    """The per-rank steps of the exchange on this library's CUDA kernels."""

    def prepare(self, topk_ids: torch.Tensor, num_experts: int):
        return moe_prepare(topk_ids, num_experts)

    def dispatch(self, x: torch.Tensor, top_k: int, meta):
        return moe_dispatch_rows(x, top_k, meta.input_permutation, meta.output_permutation)

    def recv_layout(self, recv_counts: torch.Tensor, num_recv: int):
        return moe_ep_recv_layout(recv_counts, num_recv)

    def gather_rows(self, rows: torch.Tensor, index: torch.Tensor) -> torch.Tensor:
        # out[g] = rows[index[g]]: the gather form of the dispatch with top-k 1
        return moe_dispatch_rows(rows, 1, input_permutation=index)

    def combine(self, y: torch.Tensor, meta, weights: torch.Tensor, out_dtype: torch.dtype):
        return moe_combine(y, meta.output_permutation, weights, out_dtype=out_dtype)


class EpHandle(NamedTuple):
    """What ep_combine needs from the matching ep_dispatch."""
    meta: object                  # this rank's prepare result (all experts)
    layout: object                # this rank's receive layout
    send_splits: List[int]        # rows sent to each rank
    recv_splits: List[int]        # rows received from each rank
    num_tokens: int
    top_k: int


def _ranks(group) -> int:
    return dist.get_world_size(group)


def ep_dispatch(x: torch.Tensor, topk_ids: torch.Tensor, num_experts: int, group=None,
                ops=None):
    """Sends every token row to the ranks owning its experts.

    x [T, H] and topk_ids [T, k] int32 (ids over all ``num_experts``) are
    this rank's tokens.  Returns (rows [N, H] grouped by this rank's local
    expert, then source rank, then the source's order; local_offsets
    [El+1] int32, the expert offsets of those rows; the handle for
    ep_combine).  Ids outside [0, num_experts) are sent nowhere.
    """
    ops = ops or CudaOps()
    R = _ranks(group)
    if num_experts % R:
        raise ValueError(f"{num_experts} experts do not split evenly over {R} ranks")
    El = num_experts // R
    T, k = topk_ids.shape
    H = x.shape[1]
    meta = ops.prepare(topk_ids, num_experts)
    xd = ops.dispatch(x, k, meta)
    # what each rank will receive from this one, and what this one receives
    send_counts = meta.expert_counts.reshape(R, El).contiguous()
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    bounds = meta.expert_offsets[::El].tolist()  # R + 1 block bounds of the dispatched rows
    send_splits = [bounds[r + 1] - bounds[r] for r in range(R)]
    recv_splits = recv_counts.sum(dim=1).tolist()
    n = int(sum(recv_splits))
    recv = x.new_empty((n, H))
    dist.all_to_all_single(recv, xd[: bounds[R]], recv_splits, send_splits, group=group)
    layout = ops.recv_layout(recv_counts, n)
    grouped = ops.gather_rows(recv, layout.local_to_recv) if n else recv
    return grouped, layout.local_offsets, EpHandle(meta, layout, send_splits, recv_splits, T, k)


def ep_combine(y: torch.Tensor, weights: torch.Tensor, handle: EpHandle, group=None, ops=None,
               out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """Returns every expert output row to its token's rank and combines.

    y [N, H] holds the expert outputs in the grouped order ep_dispatch
    returned; weights [T, k] fp32 are this rank's router weights.  Returns
    this rank's out [T, H] = sum_j weights[t, j] * output of slot (t, j),
    accumulated in fp32 in slot order (moe_combine).
    """
    ops = ops or CudaOps()
    H = y.shape[1]
    n = int(sum(handle.recv_splits))
    y_recv = ops.gather_rows(y, handle.layout.recv_to_local) if n else y
    # rows of slots with no valid expert stay unwritten; combine never reads them
    back = y.new_empty((handle.num_tokens * handle.top_k, H))
    sent = int(sum(handle.send_splits))
    dist.all_to_all_single(back[:sent], y_recv, handle.send_splits, handle.recv_splits,
                           group=group)
    return ops.combine(back, handle.meta, weights, out_dtype or y.dtype)


class EpPeerHandle(NamedTuple):
    """What ep_combine_peer needs from the matching ep_dispatch_peer."""
    layout: object                # moe_ep_peer_layout of this rank
    num_tokens: int
    top_k: int


def _barrier(group, dev):
    # a one-element all-reduce on the current stream: every rank's earlier
    # kernels (and their stores into other ranks' buffers) have finished
    # before any rank's later kernels start
    t = torch.zeros(1, dtype=torch.int32, device=dev)
    dist.all_reduce(t, group=group)


def ep_dispatch_peer(x: torch.Tensor, topk_ids: torch.Tensor, num_experts: int, recv_buffers,
                     group=None):
    """Stores every token row into the grouped buffer of the ranks owning
    its experts.

    ``recv_buffers`` are this process's views of every rank's grouped
    receive buffer, in rank order ([capacity, H] each, x's dtype; this
    rank's own is local memory, the others are other GPUs' memory mapped
    in), none of them in use by an earlier step.  Returns (this rank's
    grouped rows: a view of its own buffer, by local expert, then source,
    then the source's order; local_offsets [El+1]; the handle for
    ep_combine_peer)."""
    R = _ranks(group)
    rank = dist.get_rank(group)
    if num_experts % R:
        raise ValueError(f"{num_experts} experts do not split evenly over {R} ranks")
    if len(recv_buffers) != R:
        raise ValueError(f"{len(recv_buffers)} buffers for {R} ranks")
    T, k = topk_ids.shape
    meta = moe_prepare(topk_ids, num_experts)
    counts = torch.empty((R, num_experts), dtype=torch.int32, device=topk_ids.device)
    dist.all_gather_into_tensor(counts, meta.expert_counts, group=group)
    layout = moe_ep_peer_layout(counts, rank, topk_ids, meta)
    rows = layout.recv_rows.tolist()
    for r, b in enumerate(recv_buffers):
        if isinstance(b, torch.Tensor) and b.shape[0] < rows[r]:
            raise ValueError(f"rank {r}'s buffer holds {b.shape[0]} rows, {rows[r]} needed")
    moe_ep_dispatch_peer(x, k, layout, recv_buffers)
    _barrier(group, x.device)
    own = recv_buffers[rank]
    return own[: rows[rank]], layout.local_offsets, EpPeerHandle(layout, T, k)


def ep_combine_peer(out_buffers, y_dtype: torch.dtype, hidden: int, weights: torch.Tensor,
                    handle: EpPeerHandle, group=None, out_dtype=None) -> torch.Tensor:
    """Combines this rank's tokens from the expert outputs the owners wrote
    into their buffers (``out_buffers``: every rank's, in rank order, in the
    grouped layout).  Returns out [T, H] as moe_combine would."""
    _barrier(group, weights.device)  # every owner has written its expert outputs
    return moe_ep_combine_peer(out_buffers, y_dtype, hidden, handle.layout, weights,
                               out_dtype=out_dtype)
