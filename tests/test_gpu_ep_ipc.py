"""Expert parallelism across processes: two ranks, each its own process on the same GPU, map
each other's receive buffers with ep.map_peer_buffers (CUDA IPC handles exchanged over gloo)
and run the four library steps, the dispatch storing into and the combine loading from the
other process's memory.  The steps are ordered by host barriers after a device synchronize,
so no kernel of one rank ever waits for the other's.  Each rank's output rows must equal
beam_moe_forward over all tokens bit for bit."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest
import torch

pytestmark = pytest.mark.gpu

TOKENS = (120, 180)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, port: int, q):
    import numpy as np
    import torch.distributed as dist
    from sparse_moe_transformer_fp32_b200 import beam_moe as bm
    from sparse_moe_transformer_fp32_b200 import ep
    from sparse_moe_transformer_fp32_b200 import workloads as W
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=2, timeout=datetime.timedelta(seconds=120))
        torch.cuda.set_device(0)
        P = 2

        def step_barrier():
            torch.cuda.synchronize()
            dist.barrier()

        wl = W.WORKLOADS["tiny"].with_tokens(sum(TOKENS))
        E, d, k = wl.E, wl.d, wl.top_k
        h = W.hidden(wl).cuda()
        rw, b = W.router_weight(wl).cuda(), W.router_bias(wl).cuda()
        weights = W.expert_weights(wl, "cuda")
        ref = torch.empty(wl.T, d, dtype=torch.bfloat16, device="cuda")
        idx = torch.empty(wl.T, k, dtype=torch.int32, device="cuda")
        w = torch.empty(wl.T, k, dtype=torch.float32, device="cuda")
        ws = bm.beam_moe_forward(bm.shape_of(wl), h, rw, b, *weights, ref, idx, w)
        assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK

        t0 = sum(TOKENS[:rank])
        sl = slice(t0, t0 + TOKENS[rank])
        ep_e = E // P
        owners = idx.cpu().numpy() // ep_e
        cap = max(int((owners == r).sum()) for r in range(P))
        shape = bm.shape_of(wl, TOKENS[rank])
        wse = bm.ep_workspace(shape, P, cap)
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        bm.beam_moe_ep_count(shape, P, idx[sl], counts, cap, wse)
        torch.cuda.synchronize()
        gathered = [torch.empty(E, dtype=torch.int32) for _ in range(P)]
        dist.all_gather(gathered, counts.cpu())
        all_counts = torch.stack(gathered).cuda()

        xrecv = torch.zeros(cap, d, dtype=torch.bfloat16, device="cuda")
        yrecv = torch.zeros(cap, d, dtype=torch.bfloat16, device="cuda")
        xpeers, xaddr = ep.map_peer_buffers(dist, xrecv)
        ypeers, yaddr = ep.map_peer_buffers(dist, yrecv)
        step_barrier()

        bm.beam_moe_ep_dispatch(shape, P, rank, h[sl], idx[sl], all_counts, xaddr, cap, wse)
        step_barrier()
        e0, e1 = rank * ep_e, (rank + 1) * ep_e
        wg, wu, wd = weights
        bm.beam_moe_ep_experts(shape, P, rank, wl.T, all_counts, wg[e0:e1], wu[e0:e1],
                               wd[e0:e1], xrecv, yrecv, cap, wse)
        step_barrier()
        out = torch.empty(TOKENS[rank], d, dtype=torch.bfloat16, device="cuda")
        bm.beam_moe_ep_combine(shape, P, w[sl], yaddr, cap, out, wse)
        step_barrier()
        st = bm.beam_moe_sync_status(wse)
        same = torch.equal(out.view(torch.int16), ref[sl].view(torch.int16))
        recv_expected = int((owners == rank).sum())
        q.put((rank, st, same, recv_expected, int(np.asarray(xaddr)[rank] == xrecv.data_ptr())))
        step_barrier()  # the other rank has finished with this rank's buffers
        del xpeers, ypeers
        dist.destroy_process_group()
    except Exception as exc:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(exc), 0, 0))


def test_two_processes_exchange_through_ipc_mapped_buffers():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(2):
            r = q.get(timeout=300)
            results[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.terminate()
                p.join(timeout=30)
    for r in range(2):
        rank, st, same, recv, own = results[r]
        assert st != "error", same
        assert st == 0 and same, (rank, st, same)
        assert recv > 0 and own == 1
