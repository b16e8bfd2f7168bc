"""beam_moe_route_static: the router entry point that allocates nothing.

It exists for callers that cannot allocate device memory (a serving engine whose device
memory all belongs to its own pool, or a host that forbids allocation on its request path)
and so have no workspace to pass.  Its scratch is a static per-GPU array inside the library,
which bounds T to 512 tokens.  These tests call it through the C ABI and compare it with
beam_moe_route (which uses a caller workspace) on consecutive calls, so that contents left in
the shared static array by one call cannot leak into the next.

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


def _inputs(wl):
    return (W.hidden(wl).cuda(), W.router_weight(wl).cuda(), W.router_bias(wl).cuda())


def _route_both(wl, h, router_w, bias):
    s = bm.shape_of(wl)
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
def test_static_route_matches_workspace_route_on_consecutive_calls(L):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    cases = [W.WORKLOADS["prefill"].with_tokens(512),  # the largest T the static scratch holds
             W.WORKLOADS["tiny"],
             W.WORKLOADS["decode"].with_tokens(37)]
    for wl in cases:
        h, router_w, bias = _inputs(wl)
        (i0, w0, l0), (i1, w1, l1) = _route_both(wl, h, router_w, bias)
        assert np.array_equal(i1, i0), wl.name
        np.testing.assert_allclose(w1, w0, rtol=1e-5, atol=1e-7, err_msg=wl.name)
        np.testing.assert_allclose(l1, l0, rtol=1e-5, atol=2e-6, err_msg=wl.name)
        assert np.all(np.diff(i1, axis=1) > 0)
        np.testing.assert_allclose(w1.sum(axis=1), wl.scale, rtol=1e-5)
