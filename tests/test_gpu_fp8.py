"""Parity of the FP8 (E4M3) expert-weight path (called through the C ABI) with the oracle.

The oracle quantises the seeded BF16 weights itself; the CUDA path's codes and scales must
equal the oracle's bit for bit (integer decisions taken in FP32 on both sides).  Routing is the
BF16 path's (indices bit-exact).  Outputs: relative L2 <= 1e-2 and max |err| <= 5e-2 * RMS
against the oracle's FP8 layer, which multiplies the same codes exactly in double; the GPU
accumulates in FP32 on the tensor cores, and an activation value that lands on the other side
of a BF16 or E4M3 rounding boundary moves one code of its row.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W
from tests import gpu_helpers as H
from tests.test_gpu_parity import _check_routing

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


def test_quantize_e4m3_bit_exact_with_edge_rows():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 1, (300, 512)).astype(np.float32)
    x[1] = 0.0                          # all-zero row: scale 0, codes 0
    x[2] *= 1e-30                       # tiny row (scale far below 1)
    x[3, :] = 1e-2
    x[3, 7] = 1e3                       # one outlier: the other codes subnormal (2 * 2^-9)
    x[4] = np.where(np.arange(512) % 2 == 0, 448.0, -448.0)
    x[5] *= 3e37                        # huge row
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q, s = bm.beam_moe_quantize_e4m3(xb.cuda())
    q_ref, s_ref = oracle.quantize_rows_e4m3(xb)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quantize_e4m3_bit_exact_beam_expert():
    wl = W.WORKLOADS["prefill"]
    for kind in ("gate", "down"):
        m = W.expert_weight(wl, kind, 17, "cuda")
        q, s = bm.beam_moe_quantize_e4m3(m)
        q_ref, s_ref = oracle.quantize_rows_e4m3(m.cpu())
        assert np.array_equal(s.cpu().numpy(), s_ref), kind
        assert np.array_equal(q.cpu().numpy(), q_ref), kind


def test_quantize_e4m3_rejects_bad_arguments():
    x = torch.zeros(4, 24, dtype=torch.bfloat16, device="cuda")  # 24 columns: not a multiple of 16
    with pytest.raises(bm.BeamError):
        bm.beam_moe_quantize_e4m3(x)


def test_forward_fp8_tiny_every_token():
    case = H.make_case(W.WORKLOADS["tiny"])
    weights = H.device_weights(case.wl)
    fp8 = H.device_weights_fp8(weights)
    out, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    ref = H.oracle_out_fp8(case, weights, range(case.wl.T), fp8, batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, "fp8 tiny")


@pytest.mark.parametrize("T", [1, 33, 300])
def test_forward_fp8_ragged_token_counts(T):
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(T))
    weights = H.device_weights(case.wl)
    fp8 = H.device_weights_fp8(weights)
    out, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    ref = H.oracle_out_fp8(case, weights, range(T), fp8, batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, f"fp8 tiny T={T}")


def test_forward_fp8_differs_from_bf16_by_quantisation_only():
    """Same inputs through both paths: the FP8 layer stays within a few percent of the BF16
    layer (E4M3 keeps 4 significant bits), and is not identical to it."""
    case = H.make_case(W.WORKLOADS["tiny"])
    weights = H.device_weights(case.wl)
    fp8 = H.device_weights_fp8(weights)
    out8, _, _, _ = H.run_forward_fp8(case, fp8)
    out16, _, _, _ = H.run_forward(case, weights)
    a, b = out8.float().cpu().numpy(), out16.float().cpu().numpy()
    r = H.rel_l2(a, b)
    assert 1e-3 < r < 8e-2, r


@pytest.fixture(scope="module")
def beam_fp8():
    wl = W.WORKLOADS["prefill"]
    weights = H.device_weights(wl)
    fp8 = H.device_weights_fp8(weights)
    yield weights, fp8
    del weights, fp8
    torch.cuda.empty_cache()


def test_forward_fp8_decode_every_token(beam_fp8):
    weights, fp8 = beam_fp8
    case = H.make_case(W.WORKLOADS["decode"])
    out, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    ref = H.oracle_out_fp8(case, weights, range(case.wl.T), fp8, batch=8)
    H.assert_close_out(out.float().cpu().numpy(), ref, "fp8 decode")


def test_forward_fp8_prefill_every_tile(beam_fp8):
    """T = 4096: outputs of the tokens holding the first and the last row of every m-tile."""
    weights, fp8 = beam_fp8
    case = H.make_case(W.WORKLOADS["prefill"])
    out, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    toks = H.cover_tokens(case)
    ref = H.oracle_out_fp8(case, weights, toks, fp8)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, "fp8 prefill")


@pytest.mark.parametrize("name,changes", [
    ("E48_G8", dict(T=200, d=256, E=48, n_group=8, topk_group=3, top_k=5, I=128)),
    ("d8192", dict(T=40, d=8192, E=8, n_group=2, topk_group=1, top_k=2, I=128)),
    ("one_expert_per_group", dict(T=77, d=256, E=8, n_group=8, topk_group=3, top_k=3, I=128)),
    ("many_tokens", dict(T=20000, d=256, E=16, n_group=4, topk_group=2, top_k=4, I=256)),
])
def test_forward_fp8_other_shapes(name, changes):
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["tiny"], name=name, **changes)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    fp8 = H.device_weights_fp8(weights)
    out, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    toks = list(range(wl.T)) if wl.T <= 300 else H.sample_tokens(case, 40)
    ref = H.oracle_out_fp8(case, weights, toks, fp8, batch=64)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"fp8 {name}")


def test_forward_fp8_deterministic():
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(300))
    weights = H.device_weights(case.wl)
    fp8 = H.device_weights_fp8(weights)
    out1, _, _, ws = H.run_forward_fp8(case, fp8)
    out2, _, _, _ = H.run_forward_fp8(case, fp8, ws=ws)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_forward_fp8_wait_timeout_is_reported_and_context_survives():
    """With a zero wait limit the E4M3 GEMMs give up at their first open barrier, record the
    timeout and drain; the next call is correct."""
    case = H.make_case(W.WORKLOADS["tiny"].with_tokens(512))
    weights = H.device_weights(case.wl)
    fp8 = H.device_weights_fp8(weights)
    s = bm.shape_of(case.wl)
    out = torch.empty(case.wl.T, case.wl.d, dtype=torch.bfloat16, device="cuda")
    old = bm.beam_moe_get_wait_limit_ns()
    bm.beam_moe_set_wait_limit_ns(0)
    try:
        ws = bm.beam_moe_forward_fp8(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(),
                                     *fp8, out)
        st = bm.beam_moe_sync_status(ws)
    finally:
        bm.beam_moe_set_wait_limit_ns(old)
    assert st == bm.BEAM_ERR_TIMEOUT, bm.status_string(st)
    out2, idx, w, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx, w)
    toks = list(range(0, case.wl.T, 37))
    ref = H.oracle_out_fp8(case, weights, toks, fp8, batch=64)
    H.assert_close_out(out2[toks].float().cpu().numpy(), ref, "fp8 after timeout")


def test_block_fp8_every_token():
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["tiny"], block=True, T=96)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    fp8 = H.device_weights_fp8(weights)
    s = bm.shape_of(wl)
    dev = "cuda"
    x = case.x.to(dev)
    x_out = torch.empty_like(x)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_block_fp8(s, x, case.g_pre.to(dev), case.g_post.to(dev), wl.eps, wl.k_resid,
                               case.router_w.to(dev), case.bias.to(dev), *fp8, x_out, idx, w)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    _check_routing(case, idx, w)
    moe = H.oracle_out_fp8(case, weights, range(wl.T), fp8, batch=96)
    ref = oracle.block_tail(case.x, moe, case.g_post, wl.eps, wl.k_resid)
    cx, cf = oracle.residual_coefficients(wl.k_resid)
    got = x_out.cpu().numpy()
    # the residual term dominates x'; compare the MoE contribution
    H.assert_close_out((got - cx * case.x.numpy()) / cf, (ref - cx * case.x.numpy()) / cf,
                       "fp8 block")


@pytest.mark.parametrize("T,d,I", [(200, 256, 1024), (1, 512, 384), (129, 5120, 20480)])
def test_dense_fp8_every_token(T, d, I):
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS["dense"], T=T, d=d, I=I)
    h = W.hidden(wl)
    mats = tuple(W.expert_weight(wl, m, 0, "cuda") for m in ("gate", "up", "down"))
    q = []
    for m in mats:
        q += list(bm.beam_moe_quantize_e4m3(m))
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    s = bm.dense_shape(T, d, I)
    bm.beam_dense_forward_fp8(s, h.cuda(), *q, out)
    torch.cuda.synchronize()
    ref_q = []
    for i, m in enumerate(mats):
        rq, rs = oracle.quantize_rows_e4m3(m.cpu())
        assert np.array_equal(q[2 * i].cpu().numpy(), rq) and np.array_equal(q[2 * i + 1].cpu().numpy(), rs)
        ref_q += [rq, rs]
    toks = list(range(T)) if T <= 200 else sorted({0, T - 1, 1, T // 2, T // 3, 2 * T // 3})
    ref = np.stack([oracle.expert_mlp_fp8(h[t], *ref_q) for t in toks])
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"fp8 dense T={T} d={d} I={I}")
