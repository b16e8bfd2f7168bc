"""Expert-parallel exchange sizes (beam_moe_ep_plan, host only) against a plain enumeration of
slots, the argument checks of the expert-parallel entry points, and the host plumbing on two
gloo ranks: each rank counts its own routing, the counts are all-gathered, and every rank's
plan agrees with every other rank's (rows q sends to r are the rows r receives from q)."""
import os
import socket

import numpy as np
import pytest
import torch

from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import ep


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.zeros((T, k), np.int32)
    for t in range(T):
        idx[t] = np.sort(rng.choice(E, size=k, replace=False))
    return idx


def _slots_brute(idx_per_rank, E, P):
    """send[p][q] = slots of rank p whose expert q owns (by enumeration)."""
    ep_ = E // P
    send = np.zeros((P, P), np.int64)
    for p, idx in enumerate(idx_per_rank):
        for t in range(idx.shape[0]):
            for e in idx[t]:
                send[p, e // ep_] += 1
    return send


@pytest.mark.parametrize("P,E,k,Ts", [(2, 16, 4, (50, 70)), (4, 16, 4, (0, 33, 7, 100)),
                                      (8, 256, 8, (40, 1, 0, 13, 64, 64, 2, 9))])
def test_plan_matches_slot_enumeration(P, E, k, Ts):
    idx = [_routing(T, E, k, 10 * P + p) for p, T in enumerate(Ts)]
    all_counts = np.stack([np.bincount(i.reshape(-1), minlength=E) for i in idx]).astype(np.int32)
    send = _slots_brute(idx, E, P)
    for r in range(P):
        recv, s, frm = bm.beam_moe_ep_plan(P, E, all_counts, r)
        assert np.array_equal(s, send[r])
        assert np.array_equal(frm, send[:, r])
        assert recv == send[:, r].sum()


def test_plan_and_workspace_reject_bad_arguments():
    c = np.zeros((3, 16), np.int32)
    with pytest.raises(bm.BeamError):
        bm.beam_moe_ep_plan(3, 16, c, 0)          # 3 does not divide 16
    with pytest.raises(bm.BeamError):
        bm.beam_moe_ep_plan(2, 16, c[:2], 2)      # rank out of range
    neg = np.zeros((2, 16), np.int32)
    neg[1, 3] = -1
    with pytest.raises(bm.BeamError):
        bm.beam_moe_ep_plan(2, 16, neg, 0)
    s = bm.make_shape(64, 256, 16, 4, 2, 4, 128)
    assert bm.beam_moe_ep_workspace_size(s, 3, 1000) == 0     # P does not divide E
    assert bm.beam_moe_ep_workspace_size(s, 2, 0) == 0        # no receive rows
    assert bm.beam_moe_ep_workspace_size(s, 65, 1000) == 0    # above the rank limit
    assert bm.beam_moe_ep_workspace_size(s, 4, 1000) > 1000 * 128 * 2  # holds the activation
    L = bm.lib()
    # argument errors return before any device work (no GPU needed): P that does not divide E
    import ctypes
    assert L.beam_moe_ep_count(ctypes.byref(s), 3, None, None, 1000, None, 0, None) == \
        bm.BEAM_ERR_UNSUPPORTED
    assert L.beam_moe_ep_dispatch(ctypes.byref(s), 2, 2, None, None, None, None, 1000, None, 0,
                                  None) == bm.BEAM_ERR_INVALID_ARG


def test_experts_of_partitions_contiguously():
    owners = [r for r in range(8) for _ in ep.experts_of(r, 8, 256)]
    assert owners == [e // 32 for e in range(256)]
    with pytest.raises(ValueError):
        ep.experts_of(0, 3, 256)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, E, k, Ts, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        idx = _routing(Ts[rank], E, k, 100 + rank)
        counts = torch.from_numpy(np.bincount(idx.reshape(-1), minlength=E).astype(np.int32))
        all_counts = ep.gather_counts(dist, counts)
        recv, send, frm = ep.plan(all_counts, rank)
        sends = [torch.zeros(world, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sends, torch.from_numpy(send))
        q.put((rank, all_counts.numpy().tolist(), recv, send.tolist(), frm.tolist(),
               [s.tolist() for s in sends]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_exchange():
    import torch.multiprocessing as mp
    E, k, Ts = 16, 4, (37, 90)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, E, k, Ts, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    idx = [_routing(Ts[r], E, k, 100 + r) for r in range(2)]
    brute = _slots_brute(idx, E, 2)
    for r in range(2):
        _, all_counts, recv, send, frm, sends = res[r]
        assert np.array_equal(np.array(all_counts), np.stack(
            [np.bincount(i.reshape(-1), minlength=E) for i in idx]))
        assert send == brute[r].tolist() and frm == brute[:, r].tolist()
        assert recv == int(brute[:, r].sum())
        # what every rank says it sends to r is what r expects to receive from it
        assert [sends[p][r] for p in range(2)] == frm
