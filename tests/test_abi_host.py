"""Host-side checks of the C ABI: the library loads without a GPU, exports every symbol the
header declares, sizes workspaces, and rejects bad arguments before launching anything.

Bad-argument calls pass fake pointer values; the library must return before touching them.
"""
import ctypes
import os
import re

import pytest
import torch

from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "beam_moe.h")


@pytest.fixture(scope="module")
def L():
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    return bm.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BEAM_API\s+[\w\s\*]+?\b(beam_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(bm.EXPORTED)
    assert L.beam_moe_abi_version() == 1


def beam(T=64, **kw):
    w = W.WORKLOADS["prefill"]
    s = bm.shape_of(w, T)
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def test_workspace_size(L):
    tiny = bm.shape_of(W.WORKLOADS["tiny"])
    assert bm.beam_moe_workspace_size(tiny) > 0
    sizes = [bm.beam_moe_workspace_size(beam(T)) for T in (1, 32, 4096, 16384)]
    assert all(b > a for a, b in zip(sizes, sizes[1:]))
    # the expert buffers dominate: Xp, act and Y at R = T * top_k rows
    R = 16384 * 8
    assert sizes[-1] >= R * (5120 + 2560 + 5120) * 2
    assert L.beam_moe_workspace_size(None) == 0
    for bad in (dict(d=100), dict(d=16384), dict(I=100), dict(E=300), dict(n_group=7),
                dict(top_k=9), dict(topk_group=9), dict(top_k=8, topk_group=1, n_group=64, E=256),
                dict(T=-1), dict(routed_scaling_factor=float("nan"))):
        assert bm.beam_moe_workspace_size(beam(**bad)) == 0, bad


FAKE = 0x7f0000000000  # 4 KB aligned, never dereferenced


def fwd(L, s, ws_bytes=None, **ptr):
    p = dict(hidden=FAKE, router_w=FAKE, bias=FAKE, w_gate=FAKE, w_up=FAKE, w_down=FAKE, out=FAKE,
             idx=None, w=None, ws=FAKE)
    p.update(ptr)
    n = bm.beam_moe_workspace_size(s) if ws_bytes is None else ws_bytes
    return L.beam_moe_forward(ctypes.byref(s), p["hidden"], p["router_w"], p["bias"], p["w_gate"],
                              p["w_up"], p["w_down"], p["out"], p["idx"], p["w"], p["ws"], n, None)


def test_forward_rejects_bad_arguments(L):
    s = beam(64)
    assert fwd(L, beam(64, d=100)) == bm.BEAM_ERR_UNSUPPORTED
    assert fwd(L, beam(64, n_group=3)) == bm.BEAM_ERR_UNSUPPORTED
    assert fwd(L, beam(-5)) == bm.BEAM_ERR_INVALID_ARG
    assert L.beam_moe_forward(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                              1 << 40, None) == bm.BEAM_ERR_INVALID_ARG
    for name in ("hidden", "router_w", "w_gate", "w_up", "w_down", "out"):
        assert fwd(L, s, **{name: None}) == bm.BEAM_ERR_INVALID_ARG, name
        assert fwd(L, s, **{name: FAKE + 8}) == bm.BEAM_ERR_INVALID_ARG, name
    assert fwd(L, s, bias=None) == bm.BEAM_ERR_INVALID_ARG
    assert fwd(L, s, idx=FAKE + 4) == bm.BEAM_ERR_INVALID_ARG
    assert fwd(L, s, ws=None) == bm.BEAM_ERR_WORKSPACE
    assert fwd(L, s, ws=FAKE + 128) == bm.BEAM_ERR_WORKSPACE
    assert fwd(L, s, ws_bytes=bm.beam_moe_workspace_size(s) - 1) == bm.BEAM_ERR_WORKSPACE
    assert fwd(L, beam(0)) == bm.BEAM_OK  # nothing to do, nothing launched
    assert fwd(L, beam(0), hidden=None, out=None, ws=None) == bm.BEAM_OK


def test_route_and_block_reject_bad_arguments(L):
    s = beam(64)
    n = bm.beam_moe_workspace_size(s)
    assert L.beam_moe_route(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, n,
                            None) == bm.BEAM_ERR_INVALID_ARG
    assert L.beam_moe_route(ctypes.byref(s), FAKE, FAKE, FAKE, None, FAKE, None, FAKE, n,
                            None) == bm.BEAM_ERR_INVALID_ARG
    assert L.beam_moe_route(ctypes.byref(beam(0)), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, n,
                            None) == bm.BEAM_OK

    def blk(eps=1e-6, k=10, x=FAKE, x_out=FAKE, shape=s):
        return L.beam_moe_block(ctypes.byref(shape), x, FAKE, FAKE, ctypes.c_float(eps), k, FAKE,
                                FAKE, FAKE, FAKE, FAKE, x_out, None, None, FAKE, n, None)
    assert blk(eps=0.0) == bm.BEAM_ERR_INVALID_ARG
    assert blk(eps=float("inf")) == bm.BEAM_ERR_INVALID_ARG
    assert blk(k=0) == bm.BEAM_ERR_INVALID_ARG
    assert blk(x_out=FAKE + 4096) == bm.BEAM_ERR_INVALID_ARG  # partial overlap with x
    assert blk(shape=beam(0)) == bm.BEAM_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error(L):
    s = beam(64)
    assert fwd(L, s) == bm.BEAM_ERR_CUDA
    assert bm.last_cuda_error() != ""


def test_status_strings_and_knobs(L):
    assert bm.status_string(bm.BEAM_ERR_TIMEOUT) == "BEAM_ERR_TIMEOUT"
    assert bm.status_string(99) == "BEAM_ERR_UNKNOWN"
    old = bm.beam_moe_get_wait_limit_ns()
    bm.beam_moe_set_wait_limit_ns(123)
    assert bm.beam_moe_get_wait_limit_ns() == 123
    bm.beam_moe_set_wait_limit_ns(old)
    names = bm.kernel_names()
    assert "expert_gemm_gate_up" in names and "router_gemm" in names
    assert bm.beam_moe_launch_count() == 0 or torch.cuda.is_available()


def test_binding_rejects_cpu_tensors(L):
    w = W.WORKLOADS["tiny"]
    s = bm.shape_of(w)
    h = torch.zeros(w.T, w.d, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bm.beam_moe_route(s, h, torch.zeros(w.E, w.d), torch.zeros(w.E),
                          torch.zeros(w.T, w.top_k, dtype=torch.int32), torch.zeros(w.T, w.top_k))


def test_fp8_entry_points_validate_before_launching(L):
    s = beam(4096)
    fp8 = bm.beam_moe_fp8_workspace_size(s)
    R = 4096 * 8
    # the BF16 layout plus Xp row scales, the E4M3 activation and its row scales
    assert fp8 >= bm.beam_moe_workspace_size(s) + R * (4 + 2560 + 4)
    assert L.beam_moe_fp8_workspace_size(None) == 0
    assert bm.beam_moe_fp8_workspace_size(beam(64, d=100)) == 0
    A = 1 << 20  # a fake, 16-byte aligned address: never dereferenced on these paths
    q = ctypes.c_void_p
    quant = L.beam_moe_quantize_e4m3
    assert quant(q(A), 0, 512, q(A + (1 << 24)), q(A), None) == bm.BEAM_OK  # no rows: no-op
    for rows, cols, x, out, sc in ((4, 24, A, A << 4, A),        # cols not a multiple of 16
                                   (4, 0, A, A << 4, A),         # no columns
                                   (-1, 64, A, A << 4, A),       # negative rows
                                   (4, 64, A + 8, A << 4, A),    # misaligned input
                                   (4, 64, A, (A << 4) + 4, A),  # misaligned codes
                                   (4, 64, A, A << 4, 0),        # no scale array
                                   (4, 64, A, A + 64, A)):       # codes overlap the input
        assert quant(q(x), rows, cols, q(out), q(sc) if sc else None, None) == \
            bm.BEAM_ERR_INVALID_ARG, (rows, cols)
    fwd = L.beam_moe_forward_fp8
    args = [q(A)] * 13
    assert fwd(ctypes.byref(beam(0)), *[None] * 13, 0, None) == bm.BEAM_OK
    assert fwd(ctypes.byref(beam(64, d=100)), *args, 1 << 30, None) == bm.BEAM_ERR_UNSUPPORTED
    misaligned = list(args)
    misaligned[5] = q(A + 4)  # up_scale
    assert fwd(ctypes.byref(beam(64)), *misaligned, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert fwd(ctypes.byref(beam(64)), *args[:12], None, 16, None) == bm.BEAM_ERR_WORKSPACE


def test_fp8_block_and_dense_validate_before_launching(L):
    A = 1 << 20
    q = ctypes.c_void_p
    s = beam(64)
    blk = L.beam_moe_block_fp8
    base = [q(A)] * 3 + [ctypes.c_float(1e-6), ctypes.c_int32(10)] + [q(A)] * 12
    assert blk(ctypes.byref(beam(0)), *[None] * 3, ctypes.c_float(1e-6), ctypes.c_int32(10),
               *[None] * 12, 0, None) == bm.BEAM_OK
    bad_eps = list(base)
    bad_eps[3] = ctypes.c_float(0.0)
    assert blk(ctypes.byref(s), *bad_eps, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    mis = list(base)
    mis[8] = q(A + 8)  # gate_scale
    assert blk(ctypes.byref(s), *mis, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    # x_out overlapping x without being x
    ov = list(base)
    ov[13] = q(A + 64)
    assert blk(ctypes.byref(s), *ov, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert blk(ctypes.byref(s), *base[:16], None, 16, None) == bm.BEAM_ERR_WORKSPACE

    ds = bm.dense_shape(256, 5120, 20480)
    assert bm.lib().beam_dense_fp8_workspace_size(ctypes.byref(ds)) > \
        bm.lib().beam_dense_workspace_size(ctypes.byref(ds)) + 256 * (5120 + 20480)
    assert bm.lib().beam_dense_fp8_workspace_size(ctypes.byref(bm.dense_shape(4, 100, 128))) == 0
    dns = L.beam_dense_forward_fp8
    args = [q(A)] * 8  # hidden, w_gate, gate_scale, w_up, up_scale, w_down, down_scale, out
    mis = list(args)
    mis[4] = q(A + 4)  # up_scale
    assert dns(ctypes.byref(ds), *mis, q(A), 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert dns(ctypes.byref(ds), *args, None, 16, None) == bm.BEAM_ERR_WORKSPACE
    assert dns(ctypes.byref(bm.dense_shape(0, 5120, 20480)), *[None] * 9, 0, None) == bm.BEAM_OK


def test_nvfp4_entry_points_validate_before_launching(L):
    s = beam(4096)
    n = bm.beam_moe_nvfp4_workspace_size(s)
    R = 4096 * 8
    mt_cap = R // 128 + 256
    # the BF16 layout plus Xp row scales and atoms, the act codes, atoms and row scales
    assert n >= bm.beam_moe_workspace_size(s) + R * (4 + 1280 + 4) + mt_cap * 128 * (320 + 160)
    assert L.beam_moe_nvfp4_workspace_size(None) == 0
    assert bm.beam_moe_nvfp4_workspace_size(beam(64, I=128)) == 0   # I not a multiple of 256
    A = 1 << 20  # a fake, 16-byte aligned address: never dereferenced on these paths
    q = ctypes.c_void_p
    quant = L.beam_moe_quantize_nvfp4
    far = A << 6
    assert quant(q(A), None, 0, 128, 256, q(far), q(far << 1), q(far << 2), None) == bm.BEAM_OK
    for b, groups, rows, cols, codes in ((None, 2, 128, 320, far),   # cols not a multiple of 256
                                         (None, 2, 64, 256, far),    # rows not a multiple of 128
                                         (A << 3, 2, 32, 256, far),  # interleaved: rows % 64
                                         (None, -1, 128, 256, far),  # negative groups
                                         (None, 2, 0, 256, far),     # no rows
                                         (None, 2, 128, 256, far + 4),  # misaligned codes
                                         (A << 3 | 8, 2, 64, 256, far),  # misaligned b
                                         (None, 2, 128, 256, A + 256)):  # codes overlap a
        assert quant(q(A), q(b) if b else None, groups, rows, cols, q(codes), q(far << 1),
                     q(far << 2), None) == bm.BEAM_ERR_INVALID_ARG, (b, groups, rows, cols)
    # block scales overlapping the second input
    assert quant(q(A), q(A << 3), 2, 64, 256, q(far), q((A << 3) + 64), q(far << 2), None) == \
        bm.BEAM_ERR_INVALID_ARG
    fwd = L.beam_moe_forward_nvfp4
    args = [q(A)] * 13  # hidden .. topk_w, ws
    assert fwd(ctypes.byref(beam(0)), *[None] * 13, 0, None) == bm.BEAM_OK
    assert fwd(ctypes.byref(beam(64, I=128)), *args, 1 << 30, None) == bm.BEAM_ERR_UNSUPPORTED
    misaligned = list(args)
    misaligned[4] = q(A + 4)  # gate_up block scales
    assert fwd(ctypes.byref(beam(64)), *misaligned, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert fwd(ctypes.byref(beam(64)), *args[:12], None, 16, None) == bm.BEAM_ERR_WORKSPACE


def test_nvfp4_block_and_dense_validate_before_launching(L):
    A = 1 << 20
    q = ctypes.c_void_p
    s = beam(64)
    blk = L.beam_moe_block_nvfp4
    base = [q(A)] * 3 + [ctypes.c_float(1e-6), ctypes.c_int32(10)] + [q(A)] * 12
    assert blk(ctypes.byref(beam(0)), *[None] * 3, ctypes.c_float(1e-6), ctypes.c_int32(10),
               *[None] * 12, 0, None) == bm.BEAM_OK
    assert blk(ctypes.byref(beam(64, I=128)), *base, 1 << 30, None) == bm.BEAM_ERR_UNSUPPORTED
    mis = list(base)
    mis[10] = q(A + 8)  # down codes
    assert blk(ctypes.byref(s), *mis, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    mis = list(base)
    mis[12] = q(A + 4)  # down row scales
    assert blk(ctypes.byref(s), *mis, 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert blk(ctypes.byref(s), *base[:16], None, 16, None) == bm.BEAM_ERR_WORKSPACE

    ds = bm.dense_shape(256, 5120, 20480)
    n = bm.lib().beam_dense_nvfp4_workspace_size(ctypes.byref(ds))
    assert n > bm.lib().beam_dense_workspace_size(ctypes.byref(ds)) + 256 * (2560 + 10240)
    assert bm.lib().beam_dense_nvfp4_workspace_size(ctypes.byref(bm.dense_shape(4, 256, 128))) == 0
    dns = L.beam_dense_forward_nvfp4
    args = [q(A)] * 8  # hidden, 3 gate|up arrays, 3 down arrays, out
    mis = list(args)
    mis[3] = q(A + 4)  # gate|up row scales
    assert dns(ctypes.byref(ds), *mis, q(A), 1 << 30, None) == bm.BEAM_ERR_INVALID_ARG
    assert dns(ctypes.byref(ds), *args, None, 16, None) == bm.BEAM_ERR_WORKSPACE
    assert dns(ctypes.byref(bm.dense_shape(0, 5120, 20480)), *[None] * 9, 0, None) == bm.BEAM_OK
    assert dns(ctypes.byref(bm.dense_shape(4, 256, 128)), *args, q(A), 1 << 30, None) == \
        bm.BEAM_ERR_UNSUPPORTED
