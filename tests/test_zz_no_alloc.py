"""beam_moe_route_static: the router entry point that allocates nothing.

It exists for callers that cannot allocate device memory (a serving engine whose device
memory all belongs to its own pool, or a host that forbids allocation on its request path)
and so have no workspace to pass.  Its scratch is a static per-GPU array inside the library,
which bounds T to 512 tokens.  These tests call it through the C ABI and compare it with
beam_moe_route (which uses a caller workspace) and with the oracle on consecutive calls, so
that contents left in the shared static array by one call cannot leak into the next, and check
that calls after the first leave the device's free memory unchanged.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W


@pytest.fixture(scope="module")
def L():
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    return bm.lib()


def test_static_route_rejects_more_tokens_than_its_scratch_holds(L):
    s = bm.shape_of(W.WORKLOADS["prefill"], 513)
    fake = 0x7f0000000000  # never dereferenced: the call must return before any device work
    st = L.beam_moe_route_static(ctypes.byref(s), fake, fake, fake, fake, fake, None, None)
    assert st == bm.BEAM_ERR_UNSUPPORTED
    assert "512" in bm.last_cuda_error()


def _route_both(case):
    """beam_moe_route (caller workspace) and beam_moe_route_static on the same inputs."""
    wl = case.wl
    s = bm.shape_of(wl)
    h, router_w, bias = case.h.cuda(), case.router_w.cuda(), case.bias.cuda()
    out = []
    for fn in ("workspace", "static"):
        idx = torch.full((wl.T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((wl.T, wl.top_k), -1.0, dtype=torch.float32, device="cuda")
        logits = torch.full((wl.T, wl.E), float("nan"), dtype=torch.float32, device="cuda")
        if fn == "workspace":
            ws = bm.beam_moe_route(s, h, router_w, bias, idx, w, logits)
            assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
        else:
            bm.beam_moe_route_static(s, h, router_w, bias, idx, w, logits)
            torch.cuda.synchronize()
        out.append((idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()))
    return out


@pytest.mark.gpu
def test_static_route_matches_workspace_route_and_oracle_on_consecutive_calls(L):
    """Inputs with near ties removed (so the chosen experts are unique at FP32 accuracy; the two
    entry points may split the router's K sum differently).  Both must pick the oracle's
    experts bit for bit; weights and logits agree within the FP32 dot-product error."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from tests import gpu_helpers as H
    cases = [W.WORKLOADS["prefill"].with_tokens(512),  # the largest T the static scratch holds
             W.WORKLOADS["tiny"],
             W.WORKLOADS["decode"].with_tokens(37)]
    for wl in cases:
        case = H.make_case(wl)
        (i0, w0, l0), (i1, w1, l1) = _route_both(case)
        assert np.array_equal(i0, case.idx), wl.name
        assert np.array_equal(i1, case.idx), wl.name
        np.testing.assert_allclose(w1, case.w, rtol=1e-5, atol=1e-7, err_msg=wl.name)
        np.testing.assert_allclose(w1, w0, rtol=1e-5, atol=1e-7, err_msg=wl.name)
        assert np.abs(l1.astype(np.float64) - case.logits).max() <= 1e-5, wl.name
        np.testing.assert_allclose(l1, l0, rtol=1e-5, atol=2e-6, err_msg=wl.name)
        np.testing.assert_allclose(w1.sum(axis=1), wl.scale, rtol=1e-5)


@pytest.mark.gpu
def test_static_route_allocates_no_device_memory(L):
    """After a first call (which looks up the static array's address), further calls leave the
    device's free memory unchanged."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    wl = W.WORKLOADS["decode"].with_tokens(256)
    s = bm.shape_of(wl)
    h = W.hidden(wl).cuda()
    router_w, bias = W.router_weight(wl).cuda(), W.router_bias(wl).cuda()
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device="cuda")
    bm.beam_moe_route_static(s, h, router_w, bias, idx, w)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        bm.beam_moe_route_static(s, h, router_w, bias, idx, w)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
