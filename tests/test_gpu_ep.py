"""Expert parallelism emulated on one GPU: P ranks, each with its own slice of the tokens and
its own E / P experts, run the four library steps (count, dispatch, experts, combine) rank
after rank on one stream, with every "peer" receive buffer on the same device.  The result must
equal beam_moe_forward over the concatenated tokens bit for bit, since every m-tile and the
combine's order are the same; routing is taken from that forward's own outputs, so both sides
use the same weights.  Nothing here waits on another rank: the steps of different ranks never
run at the same time."""
import numpy as np
import pytest
import torch

from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    bm.lib()
    yield
    torch.cuda.empty_cache()


def _forward(case, weights):
    wl = case.wl
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = bm.beam_moe_forward(bm.shape_of(wl), case.h.cuda(), case.router_w.cuda(),
                             case.bias.cuda(), *weights, out, idx, w)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    return out, idx, w


def _ep_emulated(wl, h, idx, w, weights, Ts, recv_cap=None):
    """The expert-parallel step of P = len(Ts) ranks, rank p holding tokens
    sum(Ts[:p]) .. sum(Ts[:p+1]) - 1.  Returns (out, statuses of the ranks' workspaces)."""
    P = len(Ts)
    E, d, k = wl.E, wl.d, wl.top_k
    ep = E // P
    assert sum(Ts) == wl.T
    bounds = np.concatenate([[0], np.cumsum(Ts)])
    owners = idx.cpu().numpy() // ep
    need = max(int((owners == q).sum()) for q in range(P))
    cap = recv_cap if recv_cap is not None else max(need, 1)
    shapes = [bm.shape_of(wl, int(T)) for T in Ts]
    wss = [bm.ep_workspace(s, P, cap) for s in shapes]
    counts = [torch.empty(E, dtype=torch.int32, device="cuda") for _ in range(P)]
    sl = [slice(int(bounds[p]), int(bounds[p + 1])) for p in range(P)]
    for p in range(P):
        bm.beam_moe_ep_count(shapes[p], P, idx[sl[p]], counts[p], cap, wss[p])
    all_counts = torch.stack(counts)
    xrecv = [torch.empty(cap, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    yrecv = [torch.empty(cap, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for p in range(P):
        bm.beam_moe_ep_dispatch(shapes[p], P, p, h[sl[p]], idx[sl[p]], all_counts, xrecv, cap,
                                wss[p])
    wg, wu, wd = weights
    for q in range(P):
        e0, e1 = q * ep, (q + 1) * ep
        bm.beam_moe_ep_experts(shapes[q], P, q, wl.T, all_counts, wg[e0:e1], wu[e0:e1],
                               wd[e0:e1], xrecv[q], yrecv[q], cap, wss[q])
    out = torch.empty(wl.T, d, dtype=torch.bfloat16, device="cuda")
    for p in range(P):
        bm.beam_moe_ep_combine(shapes[p], P, w[sl[p]], yrecv, cap, out[sl[p]], wss[p])
    st = [bm.beam_moe_sync_status(ws) for ws in wss]
    # the host plan sees the same exchange as the device counts
    ac = all_counts.cpu().numpy()
    for q in range(P):
        recv, send, frm = bm.beam_moe_ep_plan(P, E, ac, q)
        assert recv == int((owners == q).sum())
    return out, st


@pytest.mark.parametrize("P,Ts", [
    (2, (100, 200)),
    (4, (1, 0, 150, 149)),              # a rank without tokens still runs its experts
    (16, (19,) * 15 + (15,)),           # one expert per rank
    (16, (300,) + (0,) * 15),           # one rank holds every token
])
def test_ep_equals_single_gpu_forward_tiny(P, Ts):
    wl = W.WORKLOADS["tiny"].with_tokens(300)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    ref, idx, w = _forward(case, weights)
    out, st = _ep_emulated(wl, case.h.cuda(), idx, w, weights, Ts)
    assert all(s == bm.BEAM_OK for s in st), st
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


@pytest.fixture(scope="module")
def beam_weights():
    ws = H.device_weights(W.WORKLOADS["prefill"])
    yield ws
    del ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,Ts", [
    ("prefill", (1000, 24, 512, 0, 1200, 360, 500, 500)),   # 8 ranks of 32 experts, uneven
    ("decode", (4, 4, 4, 4, 4, 4, 4, 4)),                    # weights-as-M tiles on every rank
])
def test_ep_equals_single_gpu_forward_beam(beam_weights, name, Ts):
    wl = W.WORKLOADS[name]
    case = H.make_case(wl)
    ref, idx, w = _forward(case, beam_weights)
    out, st = _ep_emulated(wl, case.h.cuda(), idx, w, beam_weights, Ts)
    assert all(s == bm.BEAM_OK for s in st), st
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_ep_receive_overflow_is_reported_and_context_survives():
    """Receive buffers too small for the routing: the rows that do not fit are not sent and
    the status says so; the GPU stays usable and a correctly sized step is exact."""
    wl = W.WORKLOADS["tiny"].with_tokens(300)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    ref, idx, w = _forward(case, weights)
    owners = idx.cpu().numpy() // (wl.E // 2)
    need = max(int((owners == q).sum()) for q in range(2))
    cap = need - 37
    cut, st = _ep_emulated(wl, case.h.cuda(), idx, w, weights, (150, 150), recv_cap=cap)
    assert bm.BEAM_ERR_DEVICE_ASSERT in st, st
    # which slots fit: an owner's rows run expert by expert, each expert's rows rank by rank,
    # each rank's in ascending token order; a row at or beyond the capacity is not sent
    ids = idx.cpu().numpy()
    sent = np.zeros_like(ids, dtype=bool)
    ep, Ts = wl.E // 2, (150, 150)
    for q in range(2):
        pos = 0
        for e in range(q * ep, (q + 1) * ep):
            for p in range(2):
                for t in range(p * 150, p * 150 + Ts[p]):
                    for j in np.nonzero(ids[t] == e)[0]:
                        sent[t, j] = pos < cap
                        pos += 1
    full = np.nonzero(sent.all(axis=1))[0]
    assert 0 < len(full) < wl.T
    # a token all of whose rows were sent is exact; the rest stay finite
    assert torch.equal(cut[full].view(torch.int16), ref[full].view(torch.int16))
    assert torch.isfinite(cut.float()).all()
    out, st = _ep_emulated(wl, case.h.cuda(), idx, w, weights, (150, 150))
    assert all(s == bm.BEAM_OK for s in st), st
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
