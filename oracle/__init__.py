"""Python side of the CPU oracle for the Beam sparse-MoE layer.

TEST INFRASTRUCTURE, not part of the product: only the tests, the smoke check
and the benchmark's CPU-baseline / reference leg may import this package.  It
loads ``libbeam_moe_oracle.so`` (plain C++ built from ``beam_moe_oracle.cpp``
by :func:`build`) and marshals numpy / torch CPU arrays into it.  It shares no
code with the CUDA path.

The layer the oracle computes (see the C++ source for the step-by-step
citations): FP32 sigmoid router with a selection-only bias, group-limited
top-k (group score = sum of the top-2 biased scores), normalised weights times
routed_scaling_factor, SwiGLU experts, a combine in ascending expert order,
and for the block form the sandwich RMSNorms and the depth-scaled residual.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "beam_moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libbeam_moe_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compiles the oracle with g++ (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-pthread", "-o", _LIB + ".tmp", _SRC]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, i32, f32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        L.oracle_hardware_threads.restype = i32
        L.oracle_f32_to_bf16.argtypes = [i64, vp, vp]
        L.oracle_bf16_to_f32.argtypes = [i64, vp, vp]
        L.oracle_router_logits.argtypes = [i64, i64, i64, vp, vp, vp, i32]
        L.oracle_route.argtypes = [i64, i32, i32, i32, i32, f32, i32, vp, vp, vp, vp, vp, vp, i32]
        L.oracle_route.restype = i32
        L.oracle_expert_mlp.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_tokens.argtypes = [i64, vp, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, i32]
        L.oracle_moe_tokens.restype = i32
        L.oracle_rmsnorm.argtypes = [i64, i64, vp, vp, f32, vp, i32]
        L.oracle_residual.argtypes = [i64, vp, vp, i32, vp]
        L.oracle_residual_coefficients.argtypes = [i32, ctypes.POINTER(ctypes.c_double),
                                                   ctypes.POINTER(ctypes.c_double)]
        L.oracle_bias_update.argtypes = [i32, vp, i64, vp, f32, vp]
        L.oracle_f32_to_e4m3.argtypes = [i64, vp, vp]
        L.oracle_e4m3_to_f32.argtypes = [i64, vp, vp]
        L.oracle_quantize_rows_e4m3.argtypes = [i64, i64, vp, vp, vp, i32]
        L.oracle_linear_fp8.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, i32]
        L.oracle_expert_mlp_fp8.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_tokens_fp8.argtypes = [i64, vp, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp,
                                            vp, vp, vp, i32]
        L.oracle_moe_tokens_fp8.restype = i32
        L.oracle_f32_to_e2m1.argtypes = [i64, vp, vp]
        L.oracle_e2m1_to_f32.argtypes = [i64, vp, vp]
        L.oracle_quantize_rows_nvfp4.argtypes = [i64, i64, vp, vp, vp, vp, i32]
        L.oracle_linear_nvfp4.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, i32]
        L.oracle_expert_mlp_nvfp4.argtypes = [i64, i64] + [vp] * 12
        L.oracle_moe_tokens_nvfp4.argtypes = [i64, vp, i64, i64, i32, vp, vp, vp] + [vp] * 10 + [i32]
        L.oracle_moe_tokens_nvfp4.restype = i32
        _lib = L
    return _lib


def hardware_threads() -> int:
    return lib().oracle_hardware_threads()


# ---------------------------------------------------------------- marshalling helpers

def _np(x, dtype):
    """Contiguous numpy view of a CPU tensor / array with the given numpy dtype."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        x = x.numpy()
    x = np.ascontiguousarray(x)
    if x.dtype != dtype:
        if dtype == np.uint16 and x.dtype == np.int16:
            x = x.view(np.uint16)
        else:
            x = x.astype(dtype)
    return x


def _check_tokens(tokens: np.ndarray, n: int) -> None:
    """Token ids index rows of h, idx and w: they must lie in [0, n)."""
    if tokens.size and (tokens.min() < 0 or tokens.max() >= n):
        raise ValueError(f"token ids must lie in [0, {n}); got {tokens.min()}..{tokens.max()}")


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def bf16_bits(x) -> np.ndarray:
    """BF16 tensor (or uint16 array) -> uint16 bit pattern array."""
    return _np(x, np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def f32_to_bf16(x) -> np.ndarray:
    x = _np(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_bf16(x.size, _p(x), _p(out))
    return out


def bf16_to_f32(bits) -> np.ndarray:
    b = _np(bits, np.uint16)
    out = np.empty(b.shape, np.float32)
    lib().oracle_bf16_to_f32(b.size, _p(b), _p(out))
    return out


# ---------------------------------------------------------------- layer steps

def router_logits(h, router_w, nthreads: int = 0) -> np.ndarray:
    """FP32 [T, E] router logits from BF16 h [T, d] and FP32 W_r [E, d]."""
    hb = bf16_bits(h)
    W = _np(router_w, np.float32)
    T, d = hb.shape
    E = W.shape[0]
    out = np.empty((T, E), np.float32)
    lib().oracle_router_logits(T, d, E, _p(hb), _p(W), _p(out), nthreads)
    return out


def route(logits, bias, n_group: int, topk_group: int, top_k: int, scale: float = 2.5,
          norm_topk_prob: bool = True, nthreads: int = 0):
    """Selection from logits.  Returns (idx int32 [T,k] ascending, w fp32 [T,k],
    expert margin [T], group margin [T])."""
    L = _np(logits, np.float32)
    b = _np(bias, np.float32)
    T, E = L.shape
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    me = np.empty(T, np.float32)
    mg = np.empty(T, np.float32)
    rc = lib().oracle_route(T, E, n_group, topk_group, top_k, scale, int(norm_topk_prob),
                            _p(L), _p(b), _p(idx), _p(w), _p(me), _p(mg), nthreads)
    if rc != 0:
        raise ValueError("oracle_route: invalid shape")
    return idx, w, me, mg


def expert_mlp(x, wg, wu, wd, return_act: bool = False):
    """One SwiGLU expert on one BF16 row x [d]; returns y fp32 [d] (and a bf16 bits [I])."""
    xb = bf16_bits(x).reshape(-1)
    g = bf16_bits(wg)
    u = bf16_bits(wu)
    dn = bf16_bits(wd)
    I, d = g.shape
    y = np.empty(d, np.float32)
    a = np.empty(I, np.uint16)
    lib().oracle_expert_mlp(d, I, _p(xb), _p(g), _p(u), _p(dn), _p(y), _p(a))
    return (y, a) if return_act else y


def moe_tokens(tokens, h, idx, w, experts, nthreads: int = 0) -> np.ndarray:
    """MoE output (FP32, before any BF16 rounding) for the listed tokens.

    ``experts`` maps expert id -> (w_gate [I,d], w_up [I,d], w_down [d,I]) BF16
    CPU tensors; only experts used by the listed tokens need to be present.
    """
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
    hb = bf16_bits(h)
    ix = _np(idx, np.int32)
    ww = _np(w, np.float32)
    T, d = hb.shape
    _check_tokens(tok, min(T, ix.shape[0], ww.shape[0]))
    k = ix.shape[1]
    E = int(max(experts.keys())) + 1 if experts else 1
    E = max(E, int(ix.max()) + 1)
    keep = []
    arrs = [[None] * E for _ in range(3)]
    for e, mats in experts.items():
        for m in range(3):
            a = bf16_bits(mats[m])
            keep.append(a)
            arrs[m][e] = a.ctypes.data
    I = next(iter(experts.values()))[0].shape[0]
    ptr_t = ctypes.c_void_p * E
    pg, pu, pd = (ptr_t(*[p if p is not None else None for p in arrs[m]]) for m in range(3))
    out = np.empty((len(tok), d), np.float32)
    rc = lib().oracle_moe_tokens(len(tok), _p(tok), d, I, k, _p(hb), _p(ix), _p(ww),
                                 ctypes.cast(pg, ctypes.c_void_p), ctypes.cast(pu, ctypes.c_void_p),
                                 ctypes.cast(pd, ctypes.c_void_p), _p(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_moe_tokens: an expert the tokens use was not supplied")
    del keep
    return out


def rmsnorm(x, g, eps: float, nthreads: int = 0) -> np.ndarray:
    X = _np(x, np.float32)
    G = _np(g, np.float32)
    T, d = X.shape
    y = np.empty_like(X)
    lib().oracle_rmsnorm(T, d, _p(X), _p(G), eps, _p(y), nthreads)
    return y


def residual(x, f, k: int) -> np.ndarray:
    X = _np(x, np.float32)
    F = _np(f, np.float32)
    out = np.empty_like(X)
    lib().oracle_residual(X.size, _p(X), _p(F), k, _p(out))
    return out


def residual_coefficients(k: int):
    cx, cf = ctypes.c_double(), ctypes.c_double()
    lib().oracle_residual_coefficients(k, ctypes.byref(cx), ctypes.byref(cf))
    return cx.value, cf.value


def bias_update(counts, bias, gamma: float, slots: int) -> np.ndarray:
    """bias + gamma * sign(slots / E - counts) (FP32)."""
    c = _np(counts, np.int32)
    b = _np(bias, np.float32)
    out = np.empty_like(b)
    lib().oracle_bias_update(b.size, _p(c), int(slots), _p(b), gamma, _p(out))
    return out


def dense_mlp(tokens, h, w_gate, w_up, w_down, nthreads: int = 0) -> np.ndarray:
    """Dense SwiGLU MLP (FP32 out) for the listed tokens: one expert, weight 1."""
    hb = bf16_bits(h)
    idx = np.zeros((hb.shape[0], 1), np.int32)
    w = np.ones((hb.shape[0], 1), np.float32)
    return moe_tokens(tokens, hb, idx, w, {0: (w_gate, w_up, w_down)}, nthreads)


# ---------------------------------------------------------------- whole layer / block

def layer_routing(h, router_w, bias, wl, nthreads: int = 0):
    """Oracle routing of a workload ``wl`` (a workloads.Workload-like object)."""
    logits = router_logits(h, router_w, nthreads)
    return (logits,) + route(logits, bias, wl.n_group, wl.topk_group, wl.top_k, wl.scale,
                             wl.norm_topk_prob, nthreads)


def block_prenorm(x, g_pre, eps: float, nthreads: int = 0) -> np.ndarray:
    """h = bf16(rmsnorm(x) * g_pre) as uint16 bits."""
    return f32_to_bf16(rmsnorm(x, g_pre, eps, nthreads))


def block_tail(x_rows, moe_out_rows, g_post, eps: float, k_resid: int, nthreads: int = 0):
    """x' = x*sqrt((k-1)/k) + rmsnorm(out)*g_post / sqrt(k) for the given rows."""
    o = rmsnorm(moe_out_rows, g_post, eps, nthreads)
    return residual(x_rows, o, k_resid)


# ------------------------------------------------------------------ FP8 (E4M3) expert weights

def f32_to_e4m3(x) -> np.ndarray:
    """E4M3 codes (uint8) of FP32 values: round to nearest even, saturate to +-448."""
    a = np.ascontiguousarray(_np(x, np.float32))
    out = np.empty(a.shape, np.uint8)
    lib().oracle_f32_to_e4m3(a.size, _p(a), _p(out))
    return out


def e4m3_to_f32(codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, np.uint8))
    out = np.empty(c.shape, np.float32)
    lib().oracle_e4m3_to_f32(c.size, _p(c), _p(out))
    return out


def quantize_rows_e4m3(x, nthreads: int = 0):
    """Row-wise E4M3 quantisation of a BF16 matrix [rows, cols] -> (codes uint8, scales f32)."""
    b = np.ascontiguousarray(bf16_bits(x))
    rows, cols = b.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(rows, np.float32)
    lib().oracle_quantize_rows_e4m3(rows, cols, _p(b), _p(q), _p(s), nthreads)
    return q, s


def linear_fp8(xq, sx, wq, sw, nthreads: int = 0) -> np.ndarray:
    """y[r, c] = fl32(sx_r * sw_c * sum_j xq[r, j] wq[c, j]) on decoded E4M3 codes."""
    xq = np.ascontiguousarray(np.asarray(xq, np.uint8))
    wq = np.ascontiguousarray(np.asarray(wq, np.uint8))
    sx = np.ascontiguousarray(np.asarray(sx, np.float32))
    sw = np.ascontiguousarray(np.asarray(sw, np.float32))
    rows, K = xq.shape
    n_out = wq.shape[0]
    y = np.empty((rows, n_out), np.float32)
    lib().oracle_linear_fp8(rows, n_out, K, _p(xq), _p(sx), _p(wq), _p(sw), _p(y), nthreads)
    return y


def expert_mlp_fp8(x, gq, sg, uq, su, dq, sd, return_act: bool = False):
    """One E4M3 SwiGLU expert on one BF16 row x [d]; weights as (codes, row scales)."""
    xb = np.ascontiguousarray(bf16_bits(x).reshape(-1))
    d = xb.size
    I = gq.shape[0]
    arrs = [_np(a, t) for a, t in
            ((gq, np.uint8), (sg, np.float32), (uq, np.uint8), (su, np.float32),
             (dq, np.uint8), (sd, np.float32))]
    y = np.empty(d, np.float32)
    a = np.empty(I, np.uint16)
    lib().oracle_expert_mlp_fp8(d, I, _p(xb), *[_p(v) for v in arrs], _p(y), _p(a))
    return (y, a) if return_act else y


def moe_tokens_fp8(tokens, h, idx, w, experts, nthreads: int = 0) -> np.ndarray:
    """MoE output rows for `tokens` with E4M3 experts; experts maps e -> (gq, sg, uq, su, dq, sd)
    (codes uint8 [I, d] / [d, I], row scales f32)."""
    tokens = np.ascontiguousarray(np.asarray(tokens, np.int64))
    hb = np.ascontiguousarray(bf16_bits(h))
    T, d = hb.shape
    idx = _np(idx, np.int32)
    w = _np(w, np.float32)
    _check_tokens(tokens, min(T, idx.shape[0], w.shape[0]))
    k = idx.shape[1]
    E = int(idx.max()) + 1 if idx.size else 0
    E = max([E] + [int(e) + 1 for e in experts])
    keep = []
    ptrs = [(ctypes.c_void_p * E)() for _ in range(6)]
    I = None
    for e, parts in experts.items():
        dt = (np.uint8, np.float32) * 3
        arrs = [_np(a, t) for a, t in zip(parts, dt)]
        keep.append(arrs)
        I = arrs[0].shape[0]
        for i, a in enumerate(arrs):
            ptrs[i][e] = a.ctypes.data
    out = np.empty((tokens.size, d), np.float32)
    r = lib().oracle_moe_tokens_fp8(tokens.size, _p(tokens), d, I, k, _p(hb), _p(idx), _p(w),
                                    *[ctypes.cast(p, ctypes.c_void_p) for p in ptrs], _p(out),
                                    nthreads)
    if r != 0:
        raise ValueError("moe_tokens_fp8: a token uses an expert that was not supplied")
    return out


# ------------------------------------------------------------------ NVFP4 expert weights

def f32_to_e2m1(x) -> np.ndarray:
    """E2M1 codes (uint8, low 4 bits) of FP32 values: round to nearest even, saturate to +-6."""
    a = np.ascontiguousarray(_np(x, np.float32))
    out = np.empty(a.shape, np.uint8)
    lib().oracle_f32_to_e2m1(a.size, _p(a), _p(out))
    return out


def e2m1_to_f32(codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, np.uint8))
    out = np.empty(c.shape, np.float32)
    lib().oracle_e2m1_to_f32(c.size, _p(c), _p(out))
    return out


def quantize_rows_nvfp4(x, nthreads: int = 0):
    """NVFP4 quantisation of a BF16 matrix [rows, cols] (cols a multiple of 16) ->
    (codes uint8 [rows, cols], E4M3 block scales uint8 [rows, cols / 16], row scales f32)."""
    b = np.ascontiguousarray(bf16_bits(x))
    rows, cols = b.shape
    if cols % 16:
        raise ValueError("quantize_rows_nvfp4: cols must be a multiple of 16")
    q = np.empty((rows, cols), np.uint8)
    bs = np.empty((rows, cols // 16), np.uint8)
    s = np.empty(rows, np.float32)
    lib().oracle_quantize_rows_nvfp4(rows, cols, _p(b), _p(q), _p(bs), _p(s), nthreads)
    return q, bs, s


def linear_nvfp4(xq, xbs, sx, wq, wbs, sw, nthreads: int = 0) -> np.ndarray:
    """y[r, c] = fl32(sx_r * sw_c * sum_b xbs[r, b] wbs[c, b] sum_{j in b} xq[r, j] wq[c, j])
    on decoded codes (blocks of 16 along K)."""
    xq, wq, xbs, wbs = (np.ascontiguousarray(np.asarray(a, np.uint8)) for a in (xq, wq, xbs, wbs))
    sx = np.ascontiguousarray(np.asarray(sx, np.float32))
    sw = np.ascontiguousarray(np.asarray(sw, np.float32))
    rows, K = xq.shape
    n_out = wq.shape[0]
    y = np.empty((rows, n_out), np.float32)
    lib().oracle_linear_nvfp4(rows, n_out, K, _p(xq), _p(xbs), _p(sx), _p(wq), _p(wbs), _p(sw),
                              _p(y), nthreads)
    return y


_NVFP4_PARTS = (np.uint8, np.uint8, np.float32) * 3


def expert_mlp_nvfp4(x, gate, up, down, return_act: bool = False):
    """One NVFP4 SwiGLU expert on one BF16 row x [d]; gate, up, down are each
    (codes, block scales, row scales) as returned by quantize_rows_nvfp4."""
    xb = np.ascontiguousarray(bf16_bits(x).reshape(-1))
    d = xb.size
    I = gate[0].shape[0]
    arrs = [_np(a, t) for a, t in zip((*gate, *up, *down), _NVFP4_PARTS)]
    y = np.empty(d, np.float32)
    a = np.empty(I, np.uint16)
    lib().oracle_expert_mlp_nvfp4(d, I, _p(xb), *[_p(v) for v in arrs], _p(y), _p(a))
    return (y, a) if return_act else y


def moe_tokens_nvfp4(tokens, h, idx, w, experts, nthreads: int = 0) -> np.ndarray:
    """MoE output rows for `tokens` with NVFP4 experts; experts maps e -> (gate, up, down), each
    (codes, block scales, row scales) as returned by quantize_rows_nvfp4."""
    tokens = np.ascontiguousarray(np.asarray(tokens, np.int64))
    hb = np.ascontiguousarray(bf16_bits(h))
    T, d = hb.shape
    idx = _np(idx, np.int32)
    w = _np(w, np.float32)
    _check_tokens(tokens, min(T, idx.shape[0], w.shape[0]))
    k = idx.shape[1]
    E = int(idx.max()) + 1 if idx.size else 0
    E = max([E] + [int(e) + 1 for e in experts])
    keep = []
    ptrs = [(ctypes.c_void_p * E)() for _ in range(9)]
    I = None
    for e, (gate, up, down) in experts.items():
        arrs = [_np(a, t) for a, t in zip((*gate, *up, *down), _NVFP4_PARTS)]
        keep.append(arrs)
        I = arrs[0].shape[0]
        for i, a in enumerate(arrs):
            ptrs[i][e] = a.ctypes.data
    out = np.empty((tokens.size, d), np.float32)
    r = lib().oracle_moe_tokens_nvfp4(tokens.size, _p(tokens), d, I, k, _p(hb), _p(idx), _p(w),
                                      *[ctypes.cast(p, ctypes.c_void_p) for p in ptrs], _p(out),
                                      nthreads)
    if r != 0:
        raise ValueError("moe_tokens_nvfp4: a token uses an expert that was not supplied")
    return out
