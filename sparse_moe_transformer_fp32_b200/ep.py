"""Expert parallelism for the Beam MoE layer: one process per GPU, rank p owning experts
p * E / P .. (p + 1) * E / P - 1 ("Use HF Transformers" cookbook, section Parallelism).

The arithmetic runs in libbeam_moe.so (beam_moe_ep_count / _dispatch / _experts / _combine,
declared in include/beam_moe.h); this module holds the host plumbing around it:
torch.distributed gathers every rank's per-expert counts and orders the steps, and
beam_moe_ep_plan sizes the exchange.  Token rows travel by peer stores inside the dispatch
kernel and expert outputs by peer loads inside the combine kernel, so the only collectives are
the count all-gather and one-word barriers on the stream.
"""
from __future__ import annotations

import torch

from . import beam_moe as bm


def experts_of(rank: int, P: int, E: int) -> range:
    """Experts held by `rank`: a contiguous block of E / P."""
    if E % P:
        raise ValueError(f"the rank count {P} must divide the expert count {E}")
    ep = E // P
    return range(rank * ep, (rank + 1) * ep)


def gather_counts(dist, counts: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's per-expert slot counts, [P, E] int32 on the counts' device (rank-major)."""
    P = dist.get_world_size(group)
    out = torch.empty(P * counts.numel(), dtype=counts.dtype, device=counts.device)
    dist.all_gather_into_tensor(out, counts.contiguous().view(-1), group=group)
    return out.view(P, counts.numel())


def plan(all_counts: torch.Tensor, rank: int):
    """Host exchange sizes of `rank` from the gathered counts: (rows received, rows sent to
    each rank, rows received from each rank)."""
    c = all_counts.to("cpu")
    P, E = c.shape
    return bm.beam_moe_ep_plan(P, E, c.numpy(), rank)


def map_peer_buffers(dist, buf: torch.Tensor, group=None):
    """Every rank's `buf` as seen from this rank: its own tensor, and the other ranks' opened
    through CUDA IPC handles exchanged with all_gather_object (torch's own CUDA tensor
    sharing), with peer access enabled from this rank's device to each buffer's device.
    Returns (tensors, device addresses); the tensors must stay alive while the addresses are
    in use, and every rank's `buf` until all ranks are done with it.  The handles name devices
    by index, so every rank must see the node's GPUs under the same numbering (one process per
    GPU selected with torch.cuda.set_device, not a per-rank CUDA_VISIBLE_DEVICES)."""
    from torch.multiprocessing.reductions import reduce_tensor
    P = dist.get_world_size(group)
    me = dist.get_rank(group)
    handles = [None] * P
    dist.all_gather_object(handles, reduce_tensor(buf), group=group)
    peers = []
    with torch.cuda.device(buf.device):
        for p, (rebuild, args) in enumerate(handles):
            if p == me:
                peers.append(buf)
                continue
            t = rebuild(*args)
            if t.device != buf.device:
                bm.beam_moe_enable_peer_access(t.device.index)
            peers.append(t)
    return peers, [t.data_ptr() for t in peers]


def _stream_barrier(dist, device, group=None):
    """Orders this rank's stream after every rank's earlier work on theirs: an all-reduce of one
    word, enqueued on the current stream (NCCL) like the kernels around it."""
    flag = torch.ones(1, dtype=torch.int32, device=device)
    dist.all_reduce(flag, group=group)


def layer_step(dist, shape, hidden, topk_idx, topk_w, w_gate, w_up, w_down, out, xrecv_peers,
               yrecv_peers, xrecv, yrecv, recv_rows_max: int, ws, T_total: int, group=None):
    """One expert-parallel layer step on this rank (routing given in topk_idx / topk_w).

    w_gate, w_up [E/P, I, d] and w_down [E/P, d, I] are this rank's experts; xrecv / yrecv
    [recv_rows_max, d] BF16 are its receive buffers and xrecv_peers / yrecv_peers the device
    addresses of every rank's buffers as mapped on this GPU (its own included; see
    map_peer_buffers).  Not run on a multi-GPU machine in this repository's tests: there the
    same four library calls are run rank after rank on one GPU."""
    P = dist.get_world_size(group)
    rank = dist.get_rank(group)
    counts = torch.empty(shape.E, dtype=torch.int32, device=hidden.device)
    bm.beam_moe_ep_count(shape, P, topk_idx, counts, recv_rows_max, ws)
    all_counts = gather_counts(dist, counts, group)
    bm.beam_moe_ep_dispatch(shape, P, rank, hidden, topk_idx, all_counts, xrecv_peers,
                            recv_rows_max, ws)
    _stream_barrier(dist, hidden.device, group)
    bm.beam_moe_ep_experts(shape, P, rank, T_total, all_counts, w_gate, w_up, w_down, xrecv,
                           yrecv, recv_rows_max, ws)
    _stream_barrier(dist, hidden.device, group)
    bm.beam_moe_ep_combine(shape, P, topk_w, yrecv_peers, recv_rows_max, out, ws)
    # the next step writes into the receive buffers only after every rank has read them
    _stream_barrier(dist, hidden.device, group)
    return all_counts
