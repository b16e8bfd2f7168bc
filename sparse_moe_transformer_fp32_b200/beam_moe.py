"""Python binding of libbeam_moe.so (include/beam_moe.h): argument marshalling only.

Every function here checks tensor devices, dtypes, shapes and contiguity, turns tensors
into raw device pointers and the current torch stream into a cudaStream_t, and calls the C
function of the same name.  All arithmetic runs in the library's CUDA kernels; if the
library is missing this module raises instead of computing anything itself.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbeam_moe.so")

BEAM_OK = 0
BEAM_ERR_INVALID_ARG = 1
BEAM_ERR_UNSUPPORTED = 2
BEAM_ERR_WORKSPACE = 3
BEAM_ERR_CUDA = 4
BEAM_ERR_TIMEOUT = 5
BEAM_ERR_DEVICE_ASSERT = 6

EXPORTED = [
    "beam_moe_workspace_size", "beam_moe_route", "beam_moe_forward", "beam_moe_block",
    "beam_moe_sync_status", "beam_status_string", "beam_moe_last_cuda_error",
    "beam_moe_expert_counts", "beam_moe_set_wait_limit_ns", "beam_moe_get_wait_limit_ns",
    "beam_moe_launch_count", "beam_moe_profile_enable", "beam_moe_profile_reset",
    "beam_moe_kernel_count", "beam_moe_kernel_name", "beam_moe_profile_read",
    "beam_moe_abi_version", "beam_moe_route_static", "beam_dense_workspace_size",
    "beam_dense_forward", "beam_moe_bias_update", "beam_moe_set_sm_pairs",
    "beam_moe_get_sm_pairs", "beam_moe_quantize_e4m3", "beam_moe_fp8_workspace_size",
    "beam_moe_forward_fp8", "beam_moe_block_fp8", "beam_dense_fp8_workspace_size",
    "beam_dense_forward_fp8", "beam_moe_quantize_nvfp4", "beam_moe_nvfp4_workspace_size",
    "beam_moe_forward_nvfp4", "beam_moe_block_nvfp4", "beam_dense_nvfp4_workspace_size",
    "beam_dense_forward_nvfp4", "beam_moe_slot_rows", "beam_moe_ep_workspace_size",
    "beam_moe_ep_plan", "beam_moe_ep_count", "beam_moe_ep_dispatch", "beam_moe_ep_experts",
    "beam_moe_ep_combine", "beam_moe_enable_peer_access",
]


class BeamError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        detail = last_cuda_error()
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class beam_moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("I", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("norm_topk_prob", ctypes.c_int32)]

    def __repr__(self):
        return "beam_moe_shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class beam_dense_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("I", ctypes.c_int32)]


def make_shape(T, d, E, n_group, topk_group, top_k, I, routed_scaling_factor=2.5,
               norm_topk_prob=True) -> beam_moe_shape:
    return beam_moe_shape(T, d, E, n_group, topk_group, top_k, I, routed_scaling_factor,
                          1 if norm_topk_prob else 0)


def shape_of(w, T: int | None = None) -> beam_moe_shape:
    """Shape of a workloads.Workload (optionally with another token count)."""
    return make_shape(w.T if T is None else T, w.d, w.E, w.n_group, w.topk_group, w.top_k, w.I,
                      w.scale, w.norm_topk_prob)


_lib = None


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built: run "
                           "`python -m sparse_moe_transformer_fp32_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, u64, f32 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64,
                             ctypes.c_float)
    shp = ctypes.POINTER(beam_moe_shape)
    L.beam_moe_workspace_size.argtypes = [shp]
    L.beam_moe_workspace_size.restype = sz
    L.beam_moe_route.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.beam_moe_forward.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.beam_moe_block.argtypes = [shp, vp, vp, vp, f32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                 sz, vp]
    L.beam_moe_route_static.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp]
    dshp = ctypes.POINTER(beam_dense_shape)
    L.beam_dense_workspace_size.argtypes = [dshp]
    L.beam_dense_workspace_size.restype = sz
    L.beam_dense_forward.argtypes = [dshp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.beam_dense_fp8_workspace_size.argtypes = [dshp]
    L.beam_dense_fp8_workspace_size.restype = sz
    L.beam_dense_forward_fp8.argtypes = [dshp] + [vp] * 9 + [sz, vp]
    L.beam_moe_bias_update.argtypes = [shp, vp, vp, f32, vp]
    L.beam_moe_quantize_e4m3.argtypes = [vp, ctypes.c_int64, i32, vp, vp, vp]
    L.beam_moe_fp8_workspace_size.argtypes = [shp]
    L.beam_moe_fp8_workspace_size.restype = sz
    L.beam_moe_forward_fp8.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                       sz, vp]
    L.beam_moe_block_fp8.argtypes = [shp, vp, vp, vp, f32, i32] + [vp] * 12 + [sz, vp]
    L.beam_moe_quantize_nvfp4.argtypes = [vp, vp, ctypes.c_int64, i32, i32, vp, vp, vp, vp]
    L.beam_moe_nvfp4_workspace_size.argtypes = [shp]
    L.beam_moe_nvfp4_workspace_size.restype = sz
    L.beam_moe_forward_nvfp4.argtypes = [shp] + [vp] * 13 + [sz, vp]
    L.beam_moe_block_nvfp4.argtypes = [shp, vp, vp, vp, f32, i32] + [vp] * 12 + [sz, vp]
    L.beam_dense_nvfp4_workspace_size.argtypes = [dshp]
    L.beam_dense_nvfp4_workspace_size.restype = sz
    L.beam_dense_forward_nvfp4.argtypes = [dshp] + [vp] * 9 + [sz, vp]
    L.beam_moe_sync_status.argtypes = [vp, vp]
    L.beam_status_string.argtypes = [ctypes.c_int]
    L.beam_status_string.restype = ctypes.c_char_p
    L.beam_moe_last_cuda_error.restype = ctypes.c_char_p
    L.beam_moe_expert_counts.argtypes = [shp, vp, vp, vp]
    L.beam_moe_slot_rows.argtypes = [shp, vp, vp, vp]
    i64 = ctypes.c_int64
    L.beam_moe_ep_workspace_size.argtypes = [shp, i32, i64]
    L.beam_moe_ep_workspace_size.restype = sz
    L.beam_moe_ep_plan.argtypes = [i32, i32, vp, i32, vp, vp, vp]
    L.beam_moe_ep_count.argtypes = [shp, i32, vp, vp, i64, vp, sz, vp]
    L.beam_moe_ep_dispatch.argtypes = [shp, i32, i32, vp, vp, vp, vp, i64, vp, sz, vp]
    L.beam_moe_ep_experts.argtypes = [shp, i32, i32, i64, vp, vp, vp, vp, vp, vp, i64, vp, sz, vp]
    L.beam_moe_ep_combine.argtypes = [shp, i32, vp, vp, i64, vp, vp, sz, vp]
    L.beam_moe_enable_peer_access.argtypes = [i32]
    L.beam_moe_set_wait_limit_ns.argtypes = [u64]
    L.beam_moe_get_wait_limit_ns.restype = u64
    L.beam_moe_launch_count.restype = u64
    L.beam_moe_set_sm_pairs.argtypes = [ctypes.c_int]
    L.beam_moe_get_sm_pairs.restype = ctypes.c_int
    L.beam_moe_profile_enable.argtypes = [ctypes.c_int]
    L.beam_moe_kernel_name.argtypes = [ctypes.c_int]
    L.beam_moe_kernel_name.restype = ctypes.c_char_p
    L.beam_moe_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                                        ctypes.POINTER(ctypes.c_double)]
    for name in ("beam_moe_route", "beam_moe_route_static", "beam_moe_forward", "beam_moe_block",
                 "beam_moe_sync_status", "beam_dense_forward", "beam_moe_bias_update",
                 "beam_moe_expert_counts", "beam_moe_profile_read", "beam_moe_quantize_e4m3",
                 "beam_moe_forward_fp8", "beam_moe_block_fp8", "beam_dense_forward_fp8",
                 "beam_moe_quantize_nvfp4", "beam_moe_forward_nvfp4", "beam_moe_block_nvfp4",
                 "beam_dense_forward_nvfp4", "beam_moe_slot_rows", "beam_moe_ep_plan",
                 "beam_moe_ep_count", "beam_moe_ep_dispatch", "beam_moe_ep_experts",
                 "beam_moe_ep_combine", "beam_moe_enable_peer_access"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().beam_status_string(int(status)).decode()


def last_cuda_error() -> str:
    return lib().beam_moe_last_cuda_error().decode()


# ------------------------------------------------------------------ marshalling helpers

def _ptr(t, dtype, name, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def beam_moe_workspace_size(shape: beam_moe_shape) -> int:
    return int(lib().beam_moe_workspace_size(ctypes.byref(shape)))


def workspace(shape: beam_moe_shape, device="cuda") -> torch.Tensor:
    n = beam_moe_workspace_size(shape)
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _ws(shape, ws, device):
    if ws is None:
        ws = workspace(shape, device)
    _ptr(ws, torch.uint8, "ws")
    return ws


def _check(status, where):
    if status != BEAM_OK:
        raise BeamError(status, where)


# ------------------------------------------------------------------ entry points

def beam_moe_route(shape, hidden, router_w, bias, topk_idx, topk_w, logits_out=None, ws=None,
                   stream=None):
    T, d, E, k = shape.T, shape.d, shape.E, shape.top_k
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k)),
            _ptr(topk_w, torch.float32, "topk_w", (T, k)),
            _ptr(logits_out, torch.float32, "logits_out", (T, E), optional=True)]
    ws = _ws(shape, ws, hidden.device)
    _check(lib().beam_moe_route(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                _stream(stream)), "beam_moe_route")
    return ws


def beam_moe_route_static(shape, hidden, router_w, bias, topk_idx, topk_w, logits_out=None,
                          stream=None):
    """beam_moe_route without a workspace: for callers that cannot allocate device memory.
    Scratch is the library's static per-GPU array (T <= 512); calls that overlap on the GPU
    race on it.  The first call on a device must come before any stream capture."""
    T, d, E, k = shape.T, shape.d, shape.E, shape.top_k
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k)),
            _ptr(topk_w, torch.float32, "topk_w", (T, k)),
            _ptr(logits_out, torch.float32, "logits_out", (T, E), optional=True)]
    _check(lib().beam_moe_route_static(ctypes.byref(shape), *args, _stream(stream)),
           "beam_moe_route_static")


def beam_moe_forward(shape, hidden, router_w, bias, w_gate, w_up, w_down, out, topk_idx=None,
                     topk_w=None, ws=None, stream=None):
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(w_gate, torch.bfloat16, "w_gate", (E, I, d)),
            _ptr(w_up, torch.bfloat16, "w_up", (E, I, d)),
            _ptr(w_down, torch.bfloat16, "w_down", (E, d, I)),
            _ptr(out, torch.bfloat16, "out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    ws = _ws(shape, ws, hidden.device)
    _check(lib().beam_moe_forward(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                  _stream(stream)), "beam_moe_forward")
    return ws


# ------------------------------------------------------------------ FP8 (E4M3) expert weights

def beam_moe_fp8_workspace_size(shape: beam_moe_shape) -> int:
    return lib().beam_moe_fp8_workspace_size(ctypes.byref(shape))


def fp8_workspace(shape: beam_moe_shape, device="cuda") -> torch.Tensor:
    n = beam_moe_fp8_workspace_size(shape)
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_moe_fp8_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_moe_quantize_e4m3(x, q=None, scale=None, stream=None):
    """Row-wise E4M3 codes and FP32 scales of a BF16 matrix (the last dimension is the row);
    returns (q uint8 of x's shape, scale float32 of x's shape without the last dimension)."""
    if x.dim() < 2:
        raise ValueError("x must have at least two dimensions")
    cols = x.shape[-1]
    rows = x.numel() // cols
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    args = [_ptr(x, torch.bfloat16, "x", tuple(x.shape)), ctypes.c_int64(rows),
            ctypes.c_int32(cols), _ptr(q, torch.uint8, "q", tuple(x.shape)),
            _ptr(scale, torch.float32, "scale", tuple(x.shape[:-1]))]
    _check(lib().beam_moe_quantize_e4m3(*args, _stream(stream)), "beam_moe_quantize_e4m3")
    return q, scale


def beam_moe_forward_fp8(shape, hidden, router_w, bias, w_gate, gate_scale, w_up, up_scale,
                         w_down, down_scale, out, topk_idx=None, topk_w=None, ws=None,
                         stream=None):
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(w_gate, torch.uint8, "w_gate", (E, I, d)),
            _ptr(gate_scale, torch.float32, "gate_scale", (E, I)),
            _ptr(w_up, torch.uint8, "w_up", (E, I, d)),
            _ptr(up_scale, torch.float32, "up_scale", (E, I)),
            _ptr(w_down, torch.uint8, "w_down", (E, d, I)),
            _ptr(down_scale, torch.float32, "down_scale", (E, d)),
            _ptr(out, torch.bfloat16, "out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    if ws is None:
        ws = fp8_workspace(shape, hidden.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_moe_forward_fp8(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                      _stream(stream)), "beam_moe_forward_fp8")
    return ws


# ------------------------------------------------------------------ NVFP4 expert weights

def beam_moe_nvfp4_workspace_size(shape: beam_moe_shape) -> int:
    return int(lib().beam_moe_nvfp4_workspace_size(ctypes.byref(shape)))


def nvfp4_workspace(shape: beam_moe_shape, device="cuda") -> torch.Tensor:
    n = beam_moe_nvfp4_workspace_size(shape)
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_moe_nvfp4_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_moe_quantize_nvfp4(a, b=None, stream=None):
    """NVFP4 codes, block-scale atoms and row scales of BF16 weights a [groups, rows, cols]
    (with b of the same shape: a and b interleaved in 64-row chunks, 2 * rows rows per group).
    Returns (codes uint8 [groups, out_rows, cols / 2], atoms uint8 [groups, out_rows * cols / 16],
    row scales float32 [groups, out_rows])."""
    if a.dim() != 3:
        raise ValueError("a must be [groups, rows, cols]")
    groups, rows, cols = a.shape
    out_rows = 2 * rows if b is not None else rows
    codes = torch.empty((groups, out_rows, cols // 2), dtype=torch.uint8, device=a.device)
    atoms = torch.empty((groups, out_rows * (cols // 16)), dtype=torch.uint8, device=a.device)
    scales = torch.empty((groups, out_rows), dtype=torch.float32, device=a.device)
    args = [_ptr(a, torch.bfloat16, "a", tuple(a.shape)),
            _ptr(b, torch.bfloat16, "b", tuple(a.shape), optional=True),
            ctypes.c_int64(groups), ctypes.c_int32(rows), ctypes.c_int32(cols),
            codes.data_ptr(), atoms.data_ptr(), scales.data_ptr()]
    _check(lib().beam_moe_quantize_nvfp4(*args, _stream(stream)), "beam_moe_quantize_nvfp4")
    return codes, atoms, scales


def beam_moe_forward_nvfp4(shape, hidden, router_w, bias, gate_up, down, out, topk_idx=None,
                           topk_w=None, ws=None, stream=None):
    """beam_moe_forward with NVFP4 experts: gate_up = beam_moe_quantize_nvfp4(w_gate, w_up),
    down = beam_moe_quantize_nvfp4(w_down), each (codes, atoms, row scales)."""
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    gc, ga, gs = gate_up
    dc, da, ds = down
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(gc, torch.uint8, "gate_up codes", (E, 2 * I, d // 2)),
            _ptr(ga, torch.uint8, "gate_up block scales", (E, 2 * I * (d // 16))),
            _ptr(gs, torch.float32, "gate_up scales", (E, 2 * I)),
            _ptr(dc, torch.uint8, "down codes", (E, d, I // 2)),
            _ptr(da, torch.uint8, "down block scales", (E, d * (I // 16))),
            _ptr(ds, torch.float32, "down scales", (E, d)),
            _ptr(out, torch.bfloat16, "out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    if ws is None:
        ws = nvfp4_workspace(shape, hidden.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_moe_forward_nvfp4(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                        _stream(stream)), "beam_moe_forward_nvfp4")
    return ws


def beam_moe_block(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, w_gate, w_up, w_down,
                   x_out, topk_idx=None, topk_w=None, ws=None, stream=None):
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    args = [_ptr(x, torch.float32, "x", (T, d)),
            _ptr(g_pre, torch.float32, "g_pre", (d,)),
            _ptr(g_post, torch.float32, "g_post", (d,)),
            ctypes.c_float(eps), ctypes.c_int32(k_resid),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(w_gate, torch.bfloat16, "w_gate", (E, I, d)),
            _ptr(w_up, torch.bfloat16, "w_up", (E, I, d)),
            _ptr(w_down, torch.bfloat16, "w_down", (E, d, I)),
            _ptr(x_out, torch.float32, "x_out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    ws = _ws(shape, ws, x.device)
    _check(lib().beam_moe_block(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                _stream(stream)), "beam_moe_block")
    return ws


def dense_shape(T, d, I) -> beam_dense_shape:
    return beam_dense_shape(T, d, I)


def dense_workspace(shape: beam_dense_shape, device="cuda") -> torch.Tensor:
    n = int(lib().beam_dense_workspace_size(ctypes.byref(shape)))
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_dense_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_dense_forward(shape, hidden, w_gate, w_up, w_down, out, ws=None, stream=None):
    T, d, I = shape.T, shape.d, shape.I
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(w_gate, torch.bfloat16, "w_gate", (I, d)),
            _ptr(w_up, torch.bfloat16, "w_up", (I, d)),
            _ptr(w_down, torch.bfloat16, "w_down", (d, I)),
            _ptr(out, torch.bfloat16, "out", (T, d))]
    if ws is None:
        ws = dense_workspace(shape, hidden.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_dense_forward(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                    _stream(stream)), "beam_dense_forward")
    return ws


def beam_moe_block_fp8(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, w_gate, gate_scale,
                       w_up, up_scale, w_down, down_scale, x_out, topk_idx=None, topk_w=None,
                       ws=None, stream=None):
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    args = [_ptr(x, torch.float32, "x", (T, d)),
            _ptr(g_pre, torch.float32, "g_pre", (d,)),
            _ptr(g_post, torch.float32, "g_post", (d,)),
            ctypes.c_float(eps), ctypes.c_int32(k_resid),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(w_gate, torch.uint8, "w_gate", (E, I, d)),
            _ptr(gate_scale, torch.float32, "gate_scale", (E, I)),
            _ptr(w_up, torch.uint8, "w_up", (E, I, d)),
            _ptr(up_scale, torch.float32, "up_scale", (E, I)),
            _ptr(w_down, torch.uint8, "w_down", (E, d, I)),
            _ptr(down_scale, torch.float32, "down_scale", (E, d)),
            _ptr(x_out, torch.float32, "x_out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    if ws is None:
        ws = fp8_workspace(shape, x.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_moe_block_fp8(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                    _stream(stream)), "beam_moe_block_fp8")
    return ws


def dense_fp8_workspace(shape: beam_dense_shape, device="cuda") -> torch.Tensor:
    n = int(lib().beam_dense_fp8_workspace_size(ctypes.byref(shape)))
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_dense_fp8_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_dense_forward_fp8(shape, hidden, w_gate, gate_scale, w_up, up_scale, w_down, down_scale,
                           out, ws=None, stream=None):
    T, d, I = shape.T, shape.d, shape.I
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(w_gate, torch.uint8, "w_gate", (I, d)),
            _ptr(gate_scale, torch.float32, "gate_scale", (I,)),
            _ptr(w_up, torch.uint8, "w_up", (I, d)),
            _ptr(up_scale, torch.float32, "up_scale", (I,)),
            _ptr(w_down, torch.uint8, "w_down", (d, I)),
            _ptr(down_scale, torch.float32, "down_scale", (d,)),
            _ptr(out, torch.bfloat16, "out", (T, d))]
    if ws is None:
        ws = dense_fp8_workspace(shape, hidden.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_dense_forward_fp8(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                        _stream(stream)), "beam_dense_forward_fp8")
    return ws


def beam_moe_bias_update(shape, ws, bias, gamma: float, stream=None) -> None:
    """bias += gamma * sign(mean load - load) from the loads of the last forward on ``ws``."""
    _check(lib().beam_moe_bias_update(ctypes.byref(shape), _ptr(ws, torch.uint8, "ws"),
                                      _ptr(bias, torch.float32, "bias", (shape.E,)),
                                      ctypes.c_float(gamma), _stream(stream)),
           "beam_moe_bias_update")


def beam_moe_sync_status(ws, stream=None) -> int:
    """Synchronises and returns the device status code of the latest call on ``ws``."""
    return int(lib().beam_moe_sync_status(_ptr(ws, torch.uint8, "ws"), _stream(stream)))


def beam_moe_expert_counts(shape, ws, stream=None) -> torch.Tensor:
    out = torch.empty(shape.E, dtype=torch.int32)
    _check(lib().beam_moe_expert_counts(ctypes.byref(shape), _ptr(ws, torch.uint8, "ws"),
                                        out.data_ptr(), _stream(stream)), "beam_moe_expert_counts")
    return out


def beam_moe_slot_rows(shape, ws, stream=None) -> torch.Tensor:
    out = torch.empty(shape.T, shape.top_k, dtype=torch.int32)
    _check(lib().beam_moe_slot_rows(ctypes.byref(shape), _ptr(ws, torch.uint8, "ws"),
                                    out.data_ptr(), _stream(stream)), "beam_moe_slot_rows")
    return out


# ------------------------------------------------------------------ expert parallelism

def beam_moe_ep_workspace_size(shape, P: int, recv_rows_max: int) -> int:
    return int(lib().beam_moe_ep_workspace_size(ctypes.byref(shape), int(P), int(recv_rows_max)))


def ep_workspace(shape, P: int, recv_rows_max: int, device="cuda") -> torch.Tensor:
    n = beam_moe_ep_workspace_size(shape, P, recv_rows_max)
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_moe_ep_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_moe_ep_plan(P: int, E: int, all_counts, rank: int):
    """Host-only exchange sizes from the gathered counts [P, E] (CPU): (rows this rank receives,
    rows it sends to each rank [P], rows it receives from each rank [P])."""
    import numpy as np
    c = np.ascontiguousarray(np.asarray(all_counts, dtype=np.int32).reshape(P, E))
    recv = ctypes.c_int64(0)
    send = np.zeros(P, np.int64)
    frm = np.zeros(P, np.int64)
    _check(lib().beam_moe_ep_plan(int(P), int(E), c.ctypes.data, int(rank), ctypes.byref(recv),
                                  send.ctypes.data, frm.ctypes.data), "beam_moe_ep_plan")
    return int(recv.value), send, frm


def beam_moe_enable_peer_access(peer_device: int):
    """Lets kernels on the current device access memory of `peer_device` (a no-op when it is
    the current device or access is already enabled)."""
    _check(lib().beam_moe_enable_peer_access(int(peer_device)), "beam_moe_enable_peer_access")


def _peer_array(ptrs, P: int, name: str):
    if len(ptrs) != P:
        raise ValueError(f"{name} must hold {P} device pointers")
    vals = [p.data_ptr() if isinstance(p, torch.Tensor) else int(p) for p in ptrs]
    return (ctypes.c_void_p * P)(*vals)


def beam_moe_ep_count(shape, P: int, topk_idx, counts, recv_rows_max: int, ws, stream=None):
    T, E, k = shape.T, shape.E, shape.top_k
    _check(lib().beam_moe_ep_count(ctypes.byref(shape), int(P),
                                   _ptr(topk_idx, torch.int32, "topk_idx", (T, k)),
                                   _ptr(counts, torch.int32, "counts", (E,)), int(recv_rows_max),
                                   _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)),
           "beam_moe_ep_count")


def beam_moe_ep_dispatch(shape, P: int, rank: int, hidden, topk_idx, all_counts, xrecv_peers,
                         recv_rows_max: int, ws, stream=None):
    T, d, E, k = shape.T, shape.d, shape.E, shape.top_k
    _check(lib().beam_moe_ep_dispatch(ctypes.byref(shape), int(P), int(rank),
                                      _ptr(hidden, torch.bfloat16, "hidden", (T, d)),
                                      _ptr(topk_idx, torch.int32, "topk_idx", (T, k)),
                                      _ptr(all_counts, torch.int32, "all_counts", (P, E)),
                                      _peer_array(xrecv_peers, P, "xrecv_peers"),
                                      int(recv_rows_max), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                      _stream(stream)), "beam_moe_ep_dispatch")


def beam_moe_ep_experts(shape, P: int, rank: int, T_total: int, all_counts, w_gate, w_up, w_down,
                        xrecv, yrecv, recv_rows_max: int, ws, stream=None):
    d, E, I = shape.d, shape.E, shape.I
    ep = E // P
    _check(lib().beam_moe_ep_experts(ctypes.byref(shape), int(P), int(rank), int(T_total),
                                     _ptr(all_counts, torch.int32, "all_counts", (P, E)),
                                     _ptr(w_gate, torch.bfloat16, "w_gate", (ep, I, d)),
                                     _ptr(w_up, torch.bfloat16, "w_up", (ep, I, d)),
                                     _ptr(w_down, torch.bfloat16, "w_down", (ep, d, I)),
                                     _ptr(xrecv, torch.bfloat16, "xrecv", (recv_rows_max, d)),
                                     _ptr(yrecv, torch.bfloat16, "yrecv", (recv_rows_max, d)),
                                     int(recv_rows_max), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                     _stream(stream)), "beam_moe_ep_experts")


def beam_moe_ep_combine(shape, P: int, topk_w, yrecv_peers, recv_rows_max: int, out, ws,
                        stream=None):
    T, d, k = shape.T, shape.d, shape.top_k
    _check(lib().beam_moe_ep_combine(ctypes.byref(shape), int(P),
                                     _ptr(topk_w, torch.float32, "topk_w", (T, k)),
                                     _peer_array(yrecv_peers, P, "yrecv_peers"),
                                     int(recv_rows_max), _ptr(out, torch.bfloat16, "out", (T, d)),
                                     _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)),
           "beam_moe_ep_combine")


def beam_moe_set_wait_limit_ns(ns: int) -> None:
    lib().beam_moe_set_wait_limit_ns(int(ns))


def beam_moe_get_wait_limit_ns() -> int:
    return int(lib().beam_moe_get_wait_limit_ns())


def beam_moe_set_sm_pairs(enable: bool) -> None:
    lib().beam_moe_set_sm_pairs(1 if enable else 0)


def beam_moe_get_sm_pairs() -> bool:
    return bool(lib().beam_moe_get_sm_pairs())


def beam_moe_launch_count() -> int:
    return int(lib().beam_moe_launch_count())


def beam_moe_profile_enable(on: bool) -> None:
    lib().beam_moe_profile_enable(1 if on else 0)


def beam_moe_profile_reset() -> None:
    lib().beam_moe_profile_reset()


def kernel_names():
    L = lib()
    return [L.beam_moe_kernel_name(i).decode() for i in range(L.beam_moe_kernel_count())]


def beam_moe_profile_read():
    """{kernel name: (launches, total ms)} since the last reset."""
    L = lib()
    out = {}
    for i, name in enumerate(kernel_names()):
        n, ms = ctypes.c_int64(), ctypes.c_double()
        _check(L.beam_moe_profile_read(i, ctypes.byref(n), ctypes.byref(ms)), "beam_moe_profile_read")
        out[name] = (n.value, ms.value)
    return out


def beam_moe_block_nvfp4(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, gate_up, down,
                         x_out, topk_idx=None, topk_w=None, ws=None, stream=None):
    """beam_moe_block with NVFP4 experts (gate_up, down as for beam_moe_forward_nvfp4)."""
    T, d, E, k, I = shape.T, shape.d, shape.E, shape.top_k, shape.I
    gc, ga, gs = gate_up
    dc, da, ds = down
    args = [_ptr(x, torch.float32, "x", (T, d)),
            _ptr(g_pre, torch.float32, "g_pre", (d,)),
            _ptr(g_post, torch.float32, "g_post", (d,)),
            ctypes.c_float(eps), ctypes.c_int32(k_resid),
            _ptr(router_w, torch.float32, "router_w", (E, d)),
            _ptr(bias, torch.float32, "bias", (E,)),
            _ptr(gc, torch.uint8, "gate_up codes", (E, 2 * I, d // 2)),
            _ptr(ga, torch.uint8, "gate_up block scales", (E, 2 * I * (d // 16))),
            _ptr(gs, torch.float32, "gate_up scales", (E, 2 * I)),
            _ptr(dc, torch.uint8, "down codes", (E, d, I // 2)),
            _ptr(da, torch.uint8, "down block scales", (E, d * (I // 16))),
            _ptr(ds, torch.float32, "down scales", (E, d)),
            _ptr(x_out, torch.float32, "x_out", (T, d)),
            _ptr(topk_idx, torch.int32, "topk_idx", (T, k), optional=True),
            _ptr(topk_w, torch.float32, "topk_w", (T, k), optional=True)]
    if ws is None:
        ws = nvfp4_workspace(shape, x.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_moe_block_nvfp4(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                      _stream(stream)), "beam_moe_block_nvfp4")
    return ws


def dense_nvfp4_workspace(shape: beam_dense_shape, device="cuda") -> torch.Tensor:
    n = int(lib().beam_dense_nvfp4_workspace_size(ctypes.byref(shape)))
    if n == 0:
        raise BeamError(BEAM_ERR_UNSUPPORTED, "beam_dense_nvfp4_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def beam_dense_forward_nvfp4(shape, hidden, gate_up, down, out, ws=None, stream=None):
    """beam_dense_forward with NVFP4 weights: gate_up = beam_moe_quantize_nvfp4(w_gate[None],
    w_up[None]), down = beam_moe_quantize_nvfp4(w_down[None])."""
    T, d, I = shape.T, shape.d, shape.I
    gc, ga, gs = gate_up
    dc, da, ds = down
    args = [_ptr(hidden, torch.bfloat16, "hidden", (T, d)),
            _ptr(gc, torch.uint8, "gate_up codes", (1, 2 * I, d // 2)),
            _ptr(ga, torch.uint8, "gate_up block scales", (1, 2 * I * (d // 16))),
            _ptr(gs, torch.float32, "gate_up scales", (1, 2 * I)),
            _ptr(dc, torch.uint8, "down codes", (1, d, I // 2)),
            _ptr(da, torch.uint8, "down block scales", (1, d * (I // 16))),
            _ptr(ds, torch.float32, "down scales", (1, d)),
            _ptr(out, torch.bfloat16, "out", (T, d))]
    if ws is None:
        ws = dense_nvfp4_workspace(shape, hidden.device)
    _ptr(ws, torch.uint8, "ws")
    _check(lib().beam_dense_forward_nvfp4(ctypes.byref(shape), *args, ws.data_ptr(), ws.numel(),
                                          _stream(stream)), "beam_dense_forward_nvfp4")
    return ws
