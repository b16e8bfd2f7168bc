"""Parity of the NVFP4 expert-weight path (called through the C ABI) with the oracle.

The oracle quantises the seeded BF16 weights itself.  The CUDA path's E2M1 codes (+-0 alike),
E4M3 block scales and FP32 row scales must equal the oracle's bit for bit, since both sides take
these integer decisions in FP32.  Routing is the BF16 path's (indices bit-exact).

Outputs are checked against the oracle's NVFP4 layer, which multiplies the same codes and block
scales exactly in double: relative L2 <= 1e-2 and max |err| <= 5e-2 * RMS.  The GPU accumulates
in FP32 on the tensor cores.  An activation value that lands on the other side of a BF16 or E2M1
rounding boundary moves one code of its row.

Shapes have I a multiple of 256 (the NVFP4 path's K stage), so the small cases use the tiny
workload with I = 256.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W
from tests import gpu_helpers as H
from tests.test_gpu_parity import _check_routing

pytestmark = pytest.mark.gpu

TINY = dataclasses.replace(W.WORKLOADS["tiny"], name="tiny_i256", I=256)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    bm.lib()
    yield
    torch.cuda.empty_cache()


def _check_quantised(x_gpu, b_gpu=None):
    """Quantises x (and b, interleaved) on the GPU and compares with the oracle row by row."""
    codes, atoms, scales = bm.beam_moe_quantize_nvfp4(x_gpu, b_gpu)
    torch.cuda.synchronize()
    G, rows, cols = x_gpu.shape
    out_rows = codes.shape[1]
    for g in range(G):
        if b_gpu is None:
            src = x_gpu[g].cpu()
        else:
            a, b = x_gpu[g].cpu(), b_gpu[g].cpu()
            src = torch.stack([a.reshape(rows // 64, 64, cols), b.reshape(rows // 64, 64, cols)],
                              dim=1).reshape(2 * rows, cols)
        q, bs, s = oracle.quantize_rows_nvfp4(src)
        gq = H.unpack_e2m1(codes[g].cpu().numpy())
        gb = H.atoms_to_rows(atoms[g].cpu().numpy(), out_rows, cols)
        assert np.array_equal(scales[g].cpu().numpy(), s), f"group {g}: row scales"
        assert np.array_equal(gb, bs), f"group {g}: block scales"
        assert np.array_equal(H.canonical_e2m1(gq), H.canonical_e2m1(q)), f"group {g}: codes"


def test_quantize_nvfp4_bit_exact_with_edge_rows():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 1, (2, 128, 512)).astype(np.float32)
    x[0, 1] = 0.0                        # all-zero row: scale 0, codes 0
    x[0, 2] *= 1e-30                     # tiny row
    x[0, 3, :] = 1e-2
    x[0, 3, 7] = 1e3                     # one outlier: the other blocks' scales underflow
    x[0, 4, 32:48] = 0.0                 # an all-zero block
    x[0, 5] = np.where(np.arange(512) % 2 == 0, 6.0, -4.0)
    x[1, 6] *= 3e37                      # huge row
    x[1, 7] = np.tile(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]), 64)  # ties
    xb = torch.from_numpy(x).to(torch.bfloat16).cuda()
    _check_quantised(xb)


def test_quantize_nvfp4_interleaves_two_matrices():
    rng = np.random.default_rng(1)
    a = torch.from_numpy(rng.normal(0, 0.02, (3, 192, 256)).astype(np.float32)).to(torch.bfloat16)
    b = torch.from_numpy(rng.normal(0, 0.5, (3, 192, 256)).astype(np.float32)).to(torch.bfloat16)
    _check_quantised(a.cuda(), b.cuda())


def test_quantize_nvfp4_bit_exact_beam_expert():
    wl = W.WORKLOADS["prefill"]
    for kind in ("gate", "down"):
        m = W.expert_weight(wl, kind, 17, "cuda")
        _check_quantised(m[None])


def test_quantize_nvfp4_rejects_bad_arguments():
    x = torch.zeros(1, 128, 320, dtype=torch.bfloat16, device="cuda")  # 320: not a multiple of 256
    with pytest.raises(bm.BeamError):
        bm.beam_moe_quantize_nvfp4(x)


def test_forward_nvfp4_small_every_token():
    case = H.make_case(TINY)
    weights = H.device_weights(case.wl)
    w4 = H.device_weights_nvfp4(weights)
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    ref = H.oracle_out_nvfp4(case, weights, range(case.wl.T), w4, batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, "nvfp4 tiny")


@pytest.mark.parametrize("T", [1, 33, 300])
def test_forward_nvfp4_ragged_token_counts(T):
    case = H.make_case(TINY.with_tokens(T))
    weights = H.device_weights(case.wl)
    w4 = H.device_weights_nvfp4(weights)
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    ref = H.oracle_out_nvfp4(case, weights, range(T), w4, batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, f"nvfp4 tiny T={T}")


def test_forward_nvfp4_differs_from_bf16_by_quantisation_only():
    """Same inputs through both paths: the NVFP4 layer stays near the BF16 layer (E2M1 keeps two
    significant bits, with a scale per 16 elements) and is not identical to it."""
    case = H.make_case(TINY)
    weights = H.device_weights(case.wl)
    w4 = H.device_weights_nvfp4(weights)
    out4, _, _, _ = H.run_forward_nvfp4(case, w4)
    out16, _, _, _ = H.run_forward(case, weights)
    r = H.rel_l2(out4.float().cpu().numpy(), out16.float().cpu().numpy())
    assert 1e-2 < r < 0.35, r


@pytest.fixture(scope="module")
def beam_nvfp4():
    wl = W.WORKLOADS["prefill"]
    weights = H.device_weights(wl)
    w4 = H.device_weights_nvfp4(weights)
    yield weights, w4
    del weights, w4
    torch.cuda.empty_cache()


def test_forward_nvfp4_decode_every_token(beam_nvfp4):
    weights, w4 = beam_nvfp4
    case = H.make_case(W.WORKLOADS["decode"])
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    ref = H.oracle_out_nvfp4(case, weights, range(case.wl.T), w4, batch=8)
    H.assert_close_out(out.float().cpu().numpy(), ref, "nvfp4 decode")


def test_forward_nvfp4_prefill_every_tile(beam_nvfp4):
    """T = 4096: outputs of the tokens holding the first and the last row of every m-tile."""
    weights, w4 = beam_nvfp4
    case = H.make_case(W.WORKLOADS["prefill"])
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    toks = H.cover_tokens(case)
    ref = H.oracle_out_nvfp4(case, weights, toks, w4)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, "nvfp4 prefill")


@pytest.mark.parametrize("name,changes", [
    ("E48_G8", dict(T=200, d=256, E=48, n_group=8, topk_group=3, top_k=5, I=256)),
    ("d8192", dict(T=40, d=8192, E=8, n_group=2, topk_group=1, top_k=2, I=256)),
    ("one_expert_per_group", dict(T=77, d=256, E=8, n_group=8, topk_group=3, top_k=3, I=512)),
    ("many_tokens", dict(T=20000, d=256, E=16, n_group=4, topk_group=2, top_k=4, I=256)),
])
def test_forward_nvfp4_other_shapes(name, changes):
    wl = dataclasses.replace(W.WORKLOADS["tiny"], name=name, **changes)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    w4 = H.device_weights_nvfp4(weights)
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    toks = list(range(wl.T)) if wl.T <= 300 else H.sample_tokens(case, 40)
    ref = H.oracle_out_nvfp4(case, weights, toks, w4, batch=64)
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"nvfp4 {name}")


def test_forward_nvfp4_deterministic():
    case = H.make_case(TINY.with_tokens(300))
    weights = H.device_weights(case.wl)
    w4 = H.device_weights_nvfp4(weights)
    out1, _, _, ws = H.run_forward_nvfp4(case, w4)
    out2, _, _, _ = H.run_forward_nvfp4(case, w4, ws=ws)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_forward_nvfp4_wait_timeout_is_reported_and_context_survives():
    """With a zero wait limit the NVFP4 GEMMs give up at their first open barrier, record the
    timeout and drain; the next call is correct."""
    case = H.make_case(TINY.with_tokens(512))
    weights = H.device_weights(case.wl)
    w4 = H.device_weights_nvfp4(weights)
    s = bm.shape_of(case.wl)
    out = torch.empty(case.wl.T, case.wl.d, dtype=torch.bfloat16, device="cuda")
    old = bm.beam_moe_get_wait_limit_ns()
    bm.beam_moe_set_wait_limit_ns(0)
    try:
        ws = bm.beam_moe_forward_nvfp4(s, case.h.cuda(), case.router_w.cuda(), case.bias.cuda(),
                                       w4[0], w4[1], out)
        st = bm.beam_moe_sync_status(ws)
    finally:
        bm.beam_moe_set_wait_limit_ns(old)
    assert st == bm.BEAM_ERR_TIMEOUT, bm.status_string(st)
    out2, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    toks = list(range(0, case.wl.T, 37))
    ref = H.oracle_out_nvfp4(case, weights, toks, w4, batch=64)
    H.assert_close_out(out2[toks].float().cpu().numpy(), ref, "nvfp4 after timeout")


def test_forward_nvfp4_replays_from_a_cuda_graph():
    """The NVFP4 forward is launches only, so it can be captured once and replayed: replays on
    new input contents match eager calls bit for bit."""
    wl = TINY.with_tokens(300)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    w4 = H.device_weights_nvfp4(weights)
    s = bm.shape_of(wl)
    dev = "cuda"
    h_static = case.h.to(dev).clone()
    rw, b = case.router_w.to(dev), case.bias.to(dev)
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    ws = bm.nvfp4_workspace(s)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # the first call sets up per-device state outside the capture
        bm.beam_moe_forward_nvfp4(s, h_static, rw, b, w4[0], w4[1], out, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bm.beam_moe_forward_nvfp4(s, h_static, rw, b, w4[0], w4[1], out, ws=ws)
    for seed in (5, 6):
        h_new = W.hidden(dataclasses.replace(wl, seed=seed)).to(dev)
        h_static.copy_(h_new)
        g.replay()
        torch.cuda.synchronize()
        assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
        ref = torch.empty_like(out)
        bm.beam_moe_forward_nvfp4(s, h_new, rw, b, w4[0], w4[1], ref)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), seed
    del g


@pytest.mark.parametrize("i", range(10))
def test_forward_nvfp4_random_shapes(i):
    """Seeded random shapes of the fuzz suite (group sizes, lane runs of the selection, ragged
    m-tiles) with I a multiple of 256."""
    from tests.test_gpu_fuzz import _shape
    shape = _shape(i)
    shape["I"] = 256 if i % 2 == 0 else 512
    wl = dataclasses.replace(W.WORKLOADS["tiny"], name=f"fuzz_nvfp4_{i}", **shape)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    w4 = H.device_weights_nvfp4(weights)
    out, idx, w, _ = H.run_forward_nvfp4(case, w4)
    _check_routing(case, idx, w)
    ref = H.oracle_out_nvfp4(case, weights, range(wl.T), w4, batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, f"nvfp4 {shape}")


def test_block_nvfp4_every_token():
    wl = dataclasses.replace(TINY, block=True, T=96)
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    w4 = H.device_weights_nvfp4(weights)
    s = bm.shape_of(wl)
    dev = "cuda"
    x = case.x.to(dev)
    x_out = torch.empty_like(x)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_block_nvfp4(s, x, case.g_pre.to(dev), case.g_post.to(dev), wl.eps,
                                 wl.k_resid, case.router_w.to(dev), case.bias.to(dev), w4[0],
                                 w4[1], x_out, idx, w)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    _check_routing(case, idx, w)
    moe = H.oracle_out_nvfp4(case, weights, range(wl.T), w4, batch=96)
    ref = oracle.block_tail(case.x, moe, case.g_post, wl.eps, wl.k_resid)
    cx, cf = oracle.residual_coefficients(wl.k_resid)
    got = x_out.cpu().numpy()
    # the residual term dominates x'; compare the MoE contribution
    H.assert_close_out((got - cx * case.x.numpy()) / cf, (ref - cx * case.x.numpy()) / cf,
                       "nvfp4 block")


@pytest.mark.parametrize("T,d,I", [(200, 256, 1024), (1, 512, 512), (129, 5120, 20480)])
def test_dense_nvfp4_every_token(T, d, I):
    wl = dataclasses.replace(W.WORKLOADS["dense"], T=T, d=d, I=I)
    h = W.hidden(wl)
    mats = tuple(W.expert_weight(wl, m, 0, "cuda") for m in ("gate", "up", "down"))
    w4 = (bm.beam_moe_quantize_nvfp4(mats[0][None], mats[1][None]),
          bm.beam_moe_quantize_nvfp4(mats[2][None]))
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    s = bm.dense_shape(T, d, I)
    ws = bm.beam_dense_forward_nvfp4(s, h.cuda(), w4[0], w4[1], out)
    assert bm.beam_moe_sync_status(ws) == bm.BEAM_OK
    ref_w = H.oracle_experts_nvfp4(tuple(m[None] for m in mats), [0], w4)[0]
    toks = list(range(T)) if T <= 200 else sorted({0, T - 1, 1, T // 2, T // 3, 2 * T // 3})
    ref = np.stack([oracle.expert_mlp_nvfp4(h[t], *ref_w) for t in toks])
    H.assert_close_out(out[toks].float().cpu().numpy(), ref, f"nvfp4 dense T={T} d={d} I={I}")
