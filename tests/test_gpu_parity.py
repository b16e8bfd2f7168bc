"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Routing indices must match bit-exactly (inputs have near ties removed); outputs must be within
relative L2 1e-2 and max |err| 5e-2 * RMS of the oracle's.  Small cases and the T = 4096
Beam-shape layer are compared on every token; the larger Beam-shape calls on every token's
routing and on the outputs of tokens chosen from the oracle's routing so that every m-tile of
every expert is checked, in the same launch configuration the benchmark times.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
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


def _check_routing(case, idx, w):
    """Indices bit-exact.  Weights within the tolerance the FP32 logits allow: the CUDA router
    sums the d products in FP32 (|logit error| up to ~1e-5 at d = 5120), so s = sigmoid(logit)
    moves by up to ~2.5e-6 and w = S s / sum(s) by ~1e-5 relative.  The block's router reads
    its own BF16 copy of the normed input, which may sit one BF16 ulp (2^-8 relative) away from
    the oracle's in a few elements; that moves a logit by up to ~4e-4 and w by ~5e-4."""
    idx = idx.cpu().numpy()
    assert np.array_equal(idx, case.idx), np.argwhere(idx != case.idx)[:5]
    rtol = 1e-3 if case.wl.block else 1e-5
    np.testing.assert_allclose(w.cpu().numpy(), case.w, rtol=rtol, atol=1e-7)


# ------------------------------------------------------------------ small cases, every token

def test_route_tiny_with_logits():
    case = H.make_case(W.WORKLOADS["tiny"])
    wl = case.wl
    s = bm.shape_of(wl)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device="cuda")
    logits = torch.empty(wl.T, wl.E, dtype=torch.float32, device="cuda")
    ws = bm.beam_moe_route(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(), idx, w, logits)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    _check_routing(case, idx, w)
    np.testing.assert_allclose(logits.cpu().numpy(), case.logits, rtol=1e-5, atol=2e-6)


def test_forward_tiny_every_token():
    case = H.make_case(W.WORKLOADS["tiny"])
    weights = H.device_weights(case.wl)
    out, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, weights, range(case.wl.T), batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, "tiny")


@pytest.mark.parametrize("T", [1, 2, 7, 33, 129, 300])
def test_forward_ragged_token_counts(T):
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(T))
    weights = H.device_weights(case.wl)
    out, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, weights, range(T), batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, f"tiny T={T}")


def test_forward_unnormalised_weights():
    wl = W.WORKLOADS["tiny"]
    import dataclasses
    wl = dataclasses.replace(wl, norm_topk_prob=False)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    out, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, weights, range(wl.T), batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, "unnormalised")


def test_forward_deterministic_and_workspace_reuse():
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(200))
    weights = H.device_weights(case.wl)
    big = bm.workspace(bm.shape_of(case.wl.with_tokens(1000)))
    out1, _, _, _ = H.run_forward(case, weights, ws=big)
    out2, _, _, _ = H.run_forward(case, weights, ws=big)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_identical_experts_equal_scaled_dense_swiglu():
    wl = W.WORKLOADS["tiny"]
    case = H.make_case(wl)
    weights = H.device_weights(wl, identical=True)
    out, _, _, _ = H.run_forward(case, weights)
    g, u, d = (m[0].cpu() for m in weights)
    dense = (torch.nn.functional.silu((case.h.double() @ g.double().T).float().double()).float()
             * (case.h.double() @ u.double().T).float()).to(torch.bfloat16)
    ref = 2.5 * (dense.double() @ d.double().T)
    H.assert_close_out(out.float().cpu().numpy(), ref.numpy(), "identical experts")


# ------------------------------------------------------------------ Beam shapes

@pytest.fixture(scope="module")
def beam_weights():
    """One set of Beam-shape expert weights (20 GB) shared by the Beam-shape tests; each
    workload keeps its own router, bias and hidden rows."""
    wl = W.WORKLOADS["prefill"]
    ws = H.device_weights(wl)
    yield ws
    del ws
    torch.cuda.empty_cache()


def test_decode_every_token(beam_weights):
    case = H.make_case(W.WORKLOADS["decode"])
    out, idx, w, _ = H.run_forward(case, beam_weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, beam_weights, range(case.wl.T))
    H.assert_close_out(out.float().cpu().numpy(), ref, "decode")


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed"])
def test_full_size_logits_within_fp32_dot_error(name):
    """Every router logit at the Beam shapes against the oracle's (exact sum rounded once to
    FP32).  An FP32 dot product of length 5120 with h ~ N(0, 1) and W_r ~ N(0, 0.01^2) carries
    a rounding error of order sqrt(d) * 2^-24 * |partial sums| ~ 1e-6; the bound 1e-5 leaves
    room for the summation order and is the one the weight tolerance above is derived from."""
    case = H.make_case(W.WORKLOADS[name])
    wl = case.wl
    s = bm.shape_of(wl)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device="cuda")
    logits = torch.empty(wl.T, wl.E, dtype=torch.float32, device="cuda")
    ws = bm.beam_moe_route(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(), idx, w, logits)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    _check_routing(case, idx, w)
    err = np.abs(logits.cpu().numpy().astype(np.float64) - case.logits.astype(np.float64))
    assert err.max() <= 1e-5, f"{name}: max |logit error| {err.max():.3e}"


def test_full_size_prefill_every_token(beam_weights):
    """T = 4096 at Beam shapes, the benchmark's configuration: routing and output of every
    token against the oracle."""
    case = H.make_case(W.WORKLOADS["prefill"])
    out, idx, w, ws = H.run_forward(case, beam_weights)
    _check_routing(case, idx, w)
    counts = bm.beam_moe_expert_counts(bm.shape_of(case.wl), ws).numpy()
    assert np.array_equal(counts, np.bincount(case.idx.reshape(-1), minlength=case.wl.E))
    ref = H.oracle_out(case, beam_weights, range(case.wl.T))
    H.assert_close_out(out.float().cpu().numpy(), ref, "prefill")


def _expected_rows(idx, E):
    """Row of every slot in the expert-contiguous layout: experts in ascending order, each
    expert's tokens in ascending order (from the oracle's routing)."""
    rows = np.full(idx.shape, -1, np.int64)
    base = 0
    for e in range(E):
        ts, js = np.nonzero(idx == e)
        rows[ts, js] = base + np.arange(len(ts))
        base += len(ts)
    return rows


@pytest.mark.parametrize("name", ["tiny", "prefill", "skewed"])
def test_slot_rows_follow_routing_in_ascending_token_order(beam_weights, name):
    """The dispatch's row layout is the routing's function: bit-exact against the layout
    enumerated from the oracle's routing, and equal across repeated calls."""
    wl = W.WORKLOADS[name]
    case = H.make_case(wl)
    weights = beam_weights if wl.E == 256 and wl.d == 5120 else H.device_weights(wl)
    _, _, _, ws = H.run_forward(case, weights)
    s = bm.shape_of(wl)
    rows = bm.beam_moe_slot_rows(s, ws).numpy()
    assert np.array_equal(rows, _expected_rows(case.idx, wl.E))
    H.run_forward(case, weights, ws=ws)
    assert np.array_equal(bm.beam_moe_slot_rows(s, ws).numpy(), rows)


def test_full_size_skewed_routing_all_tokens_output_every_tile(beam_weights):
    """T = 16384 with a skewed load (hot experts hold up to ~14k rows, over 100 m-tiles each):
    routing of every token; outputs of the tokens holding the first and the last row of every
    m-tile of every expert."""
    case = H.make_case(W.WORKLOADS["skewed"])
    out, idx, w, ws = H.run_forward(case, beam_weights)
    _check_routing(case, idx, w)
    counts = bm.beam_moe_expert_counts(bm.shape_of(case.wl), ws).numpy()
    assert np.array_equal(counts, np.bincount(case.idx.reshape(-1), minlength=case.wl.E))
    toks = H.cover_tokens(case)
    ref = H.oracle_out(case, beam_weights, toks)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, "skewed")


def test_block_routing_all_tokens_output_every_tile(beam_weights):
    case = H.make_case(W.WORKLOADS["block"])
    x_out, idx, w, _ = H.run_block(case, beam_weights)
    _check_routing(case, idx, w)
    toks = H.cover_tokens(case)
    moe = H.oracle_out(case, beam_weights, toks)
    ref = oracle.block_tail(case.x[toks], moe, case.g_post, case.wl.eps, case.wl.k_resid)
    got = x_out[toks].cpu().numpy()
    H.assert_close_out(got, ref, "block")
    # the residual term alone is far larger than the MoE term; check the MoE part too
    cx, cf = oracle.residual_coefficients(case.wl.k_resid)
    H.assert_close_out((got - cx * case.x[toks].numpy()) / cf,
                       (ref - cx * case.x[toks].numpy()) / cf, "block moe term")


def test_block_in_place_small():
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["tiny"], block=True, T=96)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    x_out, idx, w, _ = H.run_block(case, weights, in_place=True)
    _check_routing(case, idx, w)
    moe = H.oracle_out(case, weights, range(wl.T), batch=96)
    ref = oracle.block_tail(case.x, moe, case.g_post, wl.eps, wl.k_resid)
    cx, cf = oracle.residual_coefficients(wl.k_resid)
    got = x_out.cpu().numpy()
    H.assert_close_out((got - cx * case.x.numpy()) / cf, (ref - cx * case.x.numpy()) / cf,
                       "block in place")


# ------------------------------------------------------------------ failure path

def test_wait_timeout_is_reported_and_context_survives():
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(512))
    weights = H.device_weights(case.wl)
    s = bm.shape_of(case.wl)
    out = torch.empty(case.wl.T, case.wl.d, dtype=torch.bfloat16, device="cuda")
    old = bm.beam_moe_get_wait_limit_ns()
    bm.beam_moe_set_wait_limit_ns(0)
    try:
        ws = bm.beam_moe_forward(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(),
                                 *weights, out)
        st = bm.beam_moe_sync_status(ws)
    finally:
        bm.beam_moe_set_wait_limit_ns(old)
    assert st == bm.BEAM_ERR_TIMEOUT, bm.status_string(st)
    # the context is still usable and the next call is correct
    out2, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, weights, range(0, case.wl.T, 37), batch=64)
    H.assert_close_out(out2[::37].float().cpu().numpy(), ref, "after timeout")


def test_sm_pair_wait_timeout_is_reported_and_context_survives():
    """The SM-pair GEMMs (cta_group::2) with a zero wait limit: every role gives up at its first
    open barrier and records the timeout, the leader drains both CTAs' loads, both CTAs meet at
    the cluster barrier and free TMEM; the next call is correct."""
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(1024))  # T * top_k = 256 * E: pairs
    weights = H.device_weights(case.wl)
    s = bm.shape_of(case.wl)
    out = torch.empty(case.wl.T, case.wl.d, dtype=torch.bfloat16, device="cuda")
    old = bm.beam_moe_get_wait_limit_ns()
    bm.beam_moe_set_sm_pairs(True)
    try:
        bm.beam_moe_set_wait_limit_ns(0)
        try:
            ws = bm.beam_moe_forward(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(),
                                     *weights, out)
            st = bm.beam_moe_sync_status(ws)
        finally:
            bm.beam_moe_set_wait_limit_ns(old)
        assert st == bm.BEAM_ERR_TIMEOUT, bm.status_string(st)
        out2, idx, w, _ = H.run_forward(case, weights)
    finally:
        bm.beam_moe_set_sm_pairs(False)
    _check_routing(case, idx, w)
    toks = list(range(0, case.wl.T, 37))
    ref = H.oracle_out(case, weights, toks)
    H.assert_close_out(out2[toks].float().cpu().numpy(), ref, "pairs after timeout")


# ------------------------------------------------------------------ dense SwiGLU MLP and bias update

@pytest.mark.parametrize("T,d,I", [(200, 256, 1024), (1, 512, 384), (129, 5120, 20480)])
def test_dense_mlp_every_token(T, d, I):
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["dense"], T=T, d=d, I=I)
    h = W.hidden(wl)
    mats = tuple(W.expert_weight(wl, m, 0, "cuda") for m in ("gate", "up", "down"))
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    s = bm.dense_shape(T, d, I)
    bm.beam_dense_forward(s, h.cuda(), *mats, out)
    torch.cuda.synchronize()
    toks = list(range(T)) if T <= 200 else sorted({0, T - 1, 1, T // 2, T // 3, 2 * T // 3})
    ref = oracle.dense_mlp(toks, h, *(m.cpu() for m in mats))
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"dense T={T} d={d} I={I}")


def test_bias_update_matches_oracle():
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(300))
    weights = H.device_weights(case.wl)
    _, _, _, ws = H.run_forward(case, weights)
    s = bm.shape_of(case.wl)
    bias = case.bias.cuda().clone()
    bm.beam_moe_bias_update(s, ws, bias, 1e-3)
    counts = np.bincount(case.idx.reshape(-1), minlength=case.wl.E)
    ref = oracle.bias_update(counts, case.bias, 1e-3, case.wl.R)
    assert np.array_equal(bias.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------------ other shapes and edge cases

_TINY = W.WORKLOADS["tiny"]


@pytest.mark.parametrize("name,changes", [
    ("E64_G4_Gk2_k6", dict(T=300, d=512, E=64, n_group=4, topk_group=2, top_k=6, I=256)),
    ("no_group_limit", dict(T=100, d=256, E=32, n_group=4, topk_group=4, top_k=8, I=128)),
    ("top1", dict(T=150, d=256, E=16, n_group=4, topk_group=1, top_k=1, I=128)),
    ("one_group", dict(T=90, d=256, E=16, n_group=1, topk_group=1, top_k=4, I=256)),
    ("one_expert_per_group", dict(T=77, d=256, E=8, n_group=8, topk_group=3, top_k=3, I=128)),
    ("d8192", dict(T=40, d=8192, E=8, n_group=2, topk_group=1, top_k=2, I=128)),
    ("many_tokens", dict(T=20000, d=256, E=16, n_group=4, topk_group=2, top_k=4, I=128)),
    # groups that straddle the selection's per-lane expert runs (ceil(E/32) experts a lane)
    ("E48_G8", dict(T=200, d=256, E=48, n_group=8, topk_group=3, top_k=5, I=128)),
    ("E200_G8", dict(T=130, d=256, E=200, n_group=8, topk_group=2, top_k=8, I=128)),
    ("E256_G32", dict(T=64, d=256, E=256, n_group=32, topk_group=4, top_k=8, I=128)),
    ("E20_G5", dict(T=70, d=256, E=20, n_group=5, topk_group=2, top_k=3, I=128)),
])
def test_forward_other_shapes(name, changes):
    import dataclasses
    wl = dataclasses.replace(_TINY, name=name, **changes)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    out, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    toks = list(range(wl.T)) if wl.T <= 300 else H.sample_tokens(case, 40)
    ref = H.oracle_out(case, weights, toks, batch=64)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, name)


def test_block_at_maximum_hidden_size():
    import dataclasses
    wl = dataclasses.replace(_TINY, name="block_d8192", block=True, T=33, d=8192, E=8, n_group=2,
                             topk_group=1, top_k=2, I=128)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    x_out, idx, w, _ = H.run_block(case, weights)
    _check_routing(case, idx, w)
    moe = H.oracle_out(case, weights, range(wl.T), batch=64)
    ref = oracle.block_tail(case.x, moe, case.g_post, wl.eps, wl.k_resid)
    cx, cf = oracle.residual_coefficients(wl.k_resid)
    got = x_out.cpu().numpy()
    H.assert_close_out((got - cx * case.x.numpy()) / cf, (ref - cx * case.x.numpy()) / cf,
                       "block d8192")


@pytest.mark.parametrize("T", [1, 7])
def test_beam_shape_few_tokens(beam_weights, T):
    case = H.make_case(W.WORKLOADS["decode"].with_tokens(T))
    out, idx, w, _ = H.run_forward(case, beam_weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, beam_weights, range(T))
    H.assert_close_out(out.float().cpu().numpy(), ref, f"beam T={T}")


def test_full_size_forward_is_deterministic(beam_weights):
    case = H.make_case(W.WORKLOADS["prefill"])
    out1, _, _, ws = H.run_forward(case, beam_weights)
    out2, _, _, _ = H.run_forward(case, beam_weights, ws=ws)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("T", [1024, 1500, 4000])
def test_forward_sm_pair_path(T):
    """With SM pairs on, T * top_k >= 256 * E runs the expert GEMMs on SM pairs (cta_group::2,
    256-row tiles); T = 1500 leaves experts whose last pair tile has no rows for the second SM."""
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(T))
    weights = H.device_weights(case.wl)
    bm.beam_moe_set_sm_pairs(True)
    try:
        out, idx, w, _ = H.run_forward(case, weights)
    finally:
        bm.beam_moe_set_sm_pairs(False)
    _check_routing(case, idx, w)
    toks = H.sample_tokens(case, 64)
    ref = H.oracle_out(case, weights, toks, batch=64)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"pairs T={T}")


def test_sm_pair_path_on_beam_shapes(beam_weights):
    case = H.make_case(W.WORKLOADS["prefill"].with_tokens(8192))
    bm.beam_moe_set_sm_pairs(True)
    try:
        out, idx, w, _ = H.run_forward(case, beam_weights)
    finally:
        bm.beam_moe_set_sm_pairs(False)
    _check_routing(case, idx, w)
    toks = H.cover_tokens(case, tile_rows=256)  # an SM pair's m-tile holds 256 rows
    ref = H.oracle_out(case, beam_weights, toks)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, "pairs beam")


def test_maximum_size_beam_call(beam_weights):
    """T = 65536 at Beam shapes: 524,288 slots, expert-contiguous buffers of 2.7e9 elements
    (past 32-bit element offsets).  Routing on every token; outputs of tokens that hold each
    expert's first and last row and at least one row of every m-tile."""
    case = H.make_case(W.WORKLOADS["prefill"].with_tokens(65536))
    out, idx, w, _ = H.run_forward(case, beam_weights)
    _check_routing(case, idx, w)
    toks = H.cover_tokens(case, tile_ends=False)
    ref = H.oracle_out(case, beam_weights, toks)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, "T=65536")


def test_zero_tokens_reads_nothing():
    s = bm.shape_of(W.WORKLOADS["prefill"], 0)
    L = bm.lib()
    assert L.beam_moe_forward(ctypes.byref(s), None, None, None, None, None, None, None, None,
                              None, None, 0, None) == bm.BEAM_OK


def test_forward_replays_from_a_cuda_graph():
    """The forward is launches only (no allocation, no host synchronisation), so it can be
    captured once and replayed: replays on new input contents match eager calls bit for bit."""
    wl = W.WORKLOADS["tiny"].with_tokens(300)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    fp8 = H.device_weights_fp8(weights)
    s = bm.shape_of(wl)
    dev = "cuda"
    h_static = case.h.to(dev).clone()
    rw, b = case.router_w.to(dev), case.bias.to(dev)
    out16 = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    out8 = torch.empty_like(out16)
    ws16, ws8 = bm.workspace(s), bm.fp8_workspace(s)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first calls outside the capture set up per-device state
        bm.beam_moe_forward(s, h_static, rw, b, *weights, out16, ws=ws16)
        bm.beam_moe_forward_fp8(s, h_static, rw, b, *fp8, out8, ws=ws8)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bm.beam_moe_forward(s, h_static, rw, b, *weights, out16, ws=ws16)
        bm.beam_moe_forward_fp8(s, h_static, rw, b, *fp8, out8, ws=ws8)
    for seed in (5, 6):
        h_new = W.hidden(dataclasses.replace(wl, seed=seed)).to(dev)
        h_static.copy_(h_new)
        g.replay()
        torch.cuda.synchronize()
        assert bm.beam_moe_sync_status(ws16) == bm.BEAM_OK
        ref16 = torch.empty_like(out16)
        ref8 = torch.empty_like(out8)
        bm.beam_moe_forward(s, h_new, rw, b, *weights, ref16)
        bm.beam_moe_forward_fp8(s, h_new, rw, b, *fp8, ref8)
        torch.cuda.synchronize()
        assert torch.equal(out16.view(torch.int16), ref16.view(torch.int16)), seed
        assert torch.equal(out8.view(torch.int16), ref8.view(torch.int16)), seed
    del g


def test_concurrent_forwards_on_two_streams():
    """Two forwards with their own workspaces running at the same time on two streams (kernels
    of one may share SMs with the other's) give the same bits as each run alone."""
    wl = W.WORKLOADS["tiny"].with_tokens(600)
    weights = H.device_weights(wl)
    s = bm.shape_of(wl)
    cases = [H.make_case(dataclasses.replace(wl, seed=sd)) for sd in (11, 12)]
    alone = [H.run_forward(c, weights)[0] for c in cases]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs, wss = [], []
    for c, st in zip(cases, streams):
        outs.append(torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda"))
        wss.append(bm.workspace(s))
    torch.cuda.synchronize()
    for _ in range(5):
        for c, st, o, ws in zip(cases, streams, outs, wss):
            with torch.cuda.stream(st):
                bm.beam_moe_forward(s, c.h.cuda(), c.router_w.cuda(), c.bias.cuda(), *weights, o,
                                    ws=ws)
    torch.cuda.synchronize()
    for o, a, ws in zip(outs, alone, wss):
        assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
        assert torch.equal(o.view(torch.int16), a.view(torch.int16))
