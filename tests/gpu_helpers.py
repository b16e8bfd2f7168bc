"""Shared pieces of the GPU parity tests: inputs with near ties removed (decided by the
oracle), runs of the CUDA path through the C ABI, and oracle references for sampled tokens.

Nothing here feeds a value computed by the CUDA path into the oracle: inputs come from
sparse_moe_transformer_fp32_b200.workloads (weights drawn on the GPU and copied to the host
byte for byte), and every expected value is computed by the oracle from those inputs.
"""
from __future__ import annotations

import dataclasses
import weakref

import numpy as np
import torch

import oracle
from sparse_moe_transformer_fp32_b200 import beam_moe as bm
from sparse_moe_transformer_fp32_b200 import workloads as W

# Near-tie margin in biased-score units.  The CUDA router sums FP32 products in another order
# than the oracle's double sum (|difference| ~1e-6 in a logit for d = 5120); a selection whose
# margin is below DELTA is re-drawn so that the chosen set is unique at FP32 accuracy.
DELTA = 1e-4
DELTA_BLOCK = 1e-3  # the block's BF16 rounding of the normed input may differ by one ulp


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_close_out(got, ref, what=""):
    """Output tolerance: relative L2 <= 1e-2 and max |err| <= 5e-2 * RMS(ref)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref ** 2)))
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref)))
    assert r <= 1e-2, f"{what}: relative L2 {r:.3e} > 1e-2"
    assert m <= 5e-2 * rms, f"{what}: max abs {m:.3e} > 5e-2 * RMS {rms:.3e}"
    return r, m / rms


@dataclasses.dataclass
class Case:
    wl: W.Workload
    h: torch.Tensor          # BF16 [T, d] CPU (layer) -- oracle's normed input for the block
    router_w: torch.Tensor   # FP32 [E, d] CPU
    bias: torch.Tensor       # FP32 [E] CPU
    idx: np.ndarray          # oracle routing
    w: np.ndarray
    logits: np.ndarray
    resampled: int
    x: torch.Tensor | None = None       # FP32 [T, d] CPU (block)
    g_pre: torch.Tensor | None = None
    g_post: torch.Tensor | None = None


def make_case(wl: W.Workload, max_attempts: int = 64) -> Case:
    """Inputs of workload ``wl`` with every near-tie token re-drawn (counter attempt+1)."""
    router_w = W.router_weight(wl)
    bias = W.router_bias(wl)
    x = g_pre = g_post = None
    if wl.block:
        x = W.residual_x(wl)
        g_pre, g_post = W.norm_gains(wl)
        h = torch.from_numpy(oracle.block_prenorm(x, g_pre, wl.eps).view(np.int16)).view(torch.bfloat16)
        delta = DELTA_BLOCK
    else:
        h = W.hidden(wl)
        delta = DELTA
    resampled = 0
    rows = np.arange(wl.T)
    logits = np.empty((wl.T, wl.E), np.float32)
    idx = np.empty((wl.T, wl.top_k), np.int32)
    w = np.empty((wl.T, wl.top_k), np.float32)
    attempt = np.zeros(wl.T, np.int64)
    for _ in range(max_attempts + 1):
        L, ix, ww, me, mg = oracle.layer_routing(h[rows], router_w, bias, wl)
        logits[rows], idx[rows], w[rows] = L, ix, ww
        bad = rows[(me < delta) | (mg < delta)]
        if len(bad) == 0:
            break
        resampled += len(bad)
        for t in bad:
            attempt[t] += 1
            if wl.block:
                x[t] = W.residual_row(wl, int(t), int(attempt[t]))
                nb = oracle.block_prenorm(x[t:t + 1], g_pre, wl.eps).view(np.int16)
                h[t] = torch.from_numpy(nb[0]).view(torch.bfloat16)
            else:
                h[t] = W.hidden_row(wl, int(t), int(attempt[t]))
        rows = bad
    else:
        raise RuntimeError("could not remove near ties")
    return Case(wl, h, router_w, bias, idx, w, logits, resampled, x, g_pre, g_post)


def device_weights(wl: W.Workload, identical: bool = False):
    """Expert weights drawn on the GPU (bytes shared with the oracle by copying to host)."""
    if identical:
        g = W.expert_weight(wl, "gate", 0, "cuda")
        u = W.expert_weight(wl, "up", 0, "cuda")
        d = W.expert_weight(wl, "down", 0, "cuda")
        return (g.expand(wl.E, -1, -1).contiguous(), u.expand(wl.E, -1, -1).contiguous(),
                d.expand(wl.E, -1, -1).contiguous())
    return W.expert_weights(wl, "cuda")


def run_forward(case: Case, weights, ws=None):
    wl = case.wl
    s = bm.shape_of(wl)
    dev = "cuda"
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_forward(s, case.h.to(dev), case.router_w.to(dev), case.bias.to(dev),
                             *weights, out, idx, w, ws=ws)
    st = bm.beam_moe_sync_status(ws)
    assert st == bm.BEAM_OK, bm.status_string(st)
    return out, idx, w, ws


def run_block(case: Case, weights, in_place=False):
    wl = case.wl
    s = bm.shape_of(wl)
    dev = "cuda"
    x = case.x.to(dev)
    x_out = x if in_place else torch.empty_like(x)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_block(s, x, case.g_pre.to(dev), case.g_post.to(dev), wl.eps, wl.k_resid,
                           case.router_w.to(dev), case.bias.to(dev), *weights, x_out, idx, w)
    st = bm.beam_moe_sync_status(ws)
    assert st == bm.BEAM_OK, bm.status_string(st)
    return x_out, idx, w, ws


class _HostExperts:
    """Host copies of device expert weights (and the oracle's own quantisations of them), made
    once per expert and kept while the device tensors they came from are alive."""

    def __init__(self):
        self._store = {}

    def get(self, weights, kind: str, e: int, make):
        key = (id(weights[0]), kind, e)
        hit = self._store.get(key)
        if hit is not None and hit[0]() is weights[0]:
            return hit[1]
        # drop entries of device weights that no longer exist before adding more
        self._store = {k: v for k, v in self._store.items() if v[0]() is not None}
        val = make()
        self._store[key] = (weakref.ref(weights[0]), val)
        return val


_HOST = _HostExperts()


def host_expert(weights, e: int):
    """(gate, up, down) of expert e as CPU tensors (copied from the device once)."""
    return _HOST.get(weights, "bf16", e, lambda: tuple(m[e].cpu() for m in weights))


def _experts_of(case: Case, tokens):
    return sorted({int(e) for t in tokens for e in case.idx[t]})


def oracle_out(case: Case, weights, tokens, batch: int = 256):
    """Oracle MoE output (FP32) for ``tokens``; the experts they use are copied to the host
    once, and the oracle runs on ``batch`` tokens at a time."""
    tokens = list(tokens)
    experts = {e: host_expert(weights, e) for e in _experts_of(case, tokens)}
    out = np.empty((len(tokens), case.wl.d), np.float32)
    for b0 in range(0, len(tokens), batch):
        tb = tokens[b0:b0 + batch]
        out[b0:b0 + len(tb)] = oracle.moe_tokens(tb, case.h, case.idx, case.w, experts)
    return out


def cover_tokens(case: Case, tile_rows: int = 128, tile_ends: bool = True):
    """Tokens whose outputs, compared with the oracle's, check every m-tile of the expert GEMMs.

    The CUDA path lays out each expert's rows in ascending token order and cuts them into
    m-tiles of ``tile_rows`` rows, so the m-tile holding each (token, expert) slot follows from
    the oracle's routing alone.  The selection always holds each expert's first and last row;
    with ``tile_ends`` it holds the first and last row of every m-tile, otherwise at least one
    row of every m-tile (tokens chosen greedily, each covering up to top_k m-tiles)."""
    idx = case.idx
    T, k = idx.shape
    E = case.wl.E
    mt_of = np.empty((T, k), np.int64)       # global m-tile id of every slot
    picks = set()
    n_tiles = 0
    for e in range(E):
        ts, js = np.nonzero(idx == e)         # ascending token order
        n = len(ts)
        if n == 0:
            continue
        tiles = np.arange(n) // tile_rows
        mt_of[ts, js] = n_tiles + tiles
        picks.update((int(ts[0]), int(ts[-1])))
        if tile_ends:
            for r0 in range(0, n, tile_rows):
                picks.update((int(ts[r0]), int(ts[min(r0 + tile_rows, n) - 1])))
        n_tiles += int(tiles[-1]) + 1
    covered = np.zeros(n_tiles, bool)
    if picks:
        covered[mt_of[sorted(picks)].reshape(-1)] = True
    while not covered.all():
        gain = (~covered[mt_of]).sum(axis=1)
        t = int(np.argmax(gain))
        picks.add(t)
        covered[mt_of[t]] = True
    return sorted(picks)


def sample_tokens(case: Case, n: int, seed: int = 0):
    """First, last and random tokens, plus tokens of the most loaded expert."""
    T = case.wl.T
    rng = np.random.default_rng(seed)
    picks = {0, T - 1}
    counts = np.bincount(case.idx.reshape(-1), minlength=case.wl.E)
    hot = int(np.argmax(counts))
    hot_tokens = np.nonzero((case.idx == hot).any(axis=1))[0]
    if len(hot_tokens):
        picks.update(rng.choice(hot_tokens, size=min(2, len(hot_tokens)), replace=False).tolist())
    while len(picks) < min(n, T):
        picks.add(int(rng.integers(0, T)))
    return sorted(picks)


# ------------------------------------------------------------------ FP8 (E4M3) expert weights

def device_weights_fp8(weights):
    """E4M3 codes and row scales of BF16 expert weights, quantised by the CUDA path:
    (gate codes, gate scales, up codes, up scales, down codes, down scales)."""
    out = []
    for m in weights:
        q, s = bm.beam_moe_quantize_e4m3(m)
        out += [q, s]
    torch.cuda.synchronize()
    return tuple(out)


def oracle_experts_fp8(weights, experts, gpu_fp8=None):
    """The oracle's own E4M3 quantisation of the listed experts (from the BF16 weights); when
    the CUDA path's codes are given, they must equal the oracle's bit for bit."""
    res = {}
    for e in experts:
        parts = _HOST.get(weights, "e4m3", e, lambda: tuple(
            p for m in host_expert(weights, e) for p in oracle.quantize_rows_e4m3(m)))
        if gpu_fp8 is not None:
            for m_i in range(3):
                q, s = parts[2 * m_i], parts[2 * m_i + 1]
                gq = gpu_fp8[2 * m_i][e].cpu().numpy()
                gs = gpu_fp8[2 * m_i + 1][e].cpu().numpy()
                assert np.array_equal(gq, q), f"expert {e} matrix {m_i}: E4M3 codes differ"
                assert np.array_equal(gs, s), f"expert {e} matrix {m_i}: scales differ"
        res[e] = parts
    return res


def run_forward_fp8(case: Case, fp8, ws=None):
    wl = case.wl
    s = bm.shape_of(wl)
    dev = "cuda"
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_forward_fp8(s, case.h.to(dev), case.router_w.to(dev), case.bias.to(dev),
                                 *fp8, out, idx, w, ws=ws)
    st = bm.beam_moe_sync_status(ws)
    assert st == bm.BEAM_OK, bm.status_string(st)
    return out, idx, w, ws


def oracle_out_fp8(case: Case, weights, tokens, gpu_fp8=None, batch: int = 256):
    """Oracle MoE output (FP32) of the E4M3 path for ``tokens``; the oracle quantises the BF16
    weights of the experts the tokens use (and checks the CUDA path's codes against its own)."""
    tokens = list(tokens)
    experts = oracle_experts_fp8(weights, _experts_of(case, tokens), gpu_fp8)
    out = np.empty((len(tokens), case.wl.d), np.float32)
    for b0 in range(0, len(tokens), batch):
        tb = tokens[b0:b0 + batch]
        out[b0:b0 + len(tb)] = oracle.moe_tokens_fp8(tb, case.h, case.idx, case.w, experts)
    return out


# ------------------------------------------------------------------ NVFP4 expert weights

def device_weights_nvfp4(weights):
    """NVFP4 form of BF16 expert weights, quantised by the CUDA path: ((gate|up interleaved
    codes, atoms, row scales), (down codes, atoms, row scales))."""
    wg, wu, wd = weights
    gu = bm.beam_moe_quantize_nvfp4(wg, wu)
    dn = bm.beam_moe_quantize_nvfp4(wd)
    torch.cuda.synchronize()
    return gu, dn


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """[..., n / 2] bytes -> [..., n] codes (element 2i in the low nibble of byte i)."""
    lo, hi = packed & 0xF, packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)


def atoms_to_rows(atoms: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Block-scale atoms of `rows` (a multiple of 128) x `cols` -> [rows, cols / 16] codes:
    byte (r % 32) * 16 + (r / 32) * 4 + (j % 4) of atom j / 4 of row group r / 128."""
    a = atoms.reshape(rows // 128, cols // 64, 32, 4, 4)      # group, atom, m0, m1, block
    return a.transpose(0, 3, 2, 1, 4).reshape(rows, cols // 16)


def canonical_e2m1(q: np.ndarray) -> np.ndarray:
    """Codes with -0 written as +0 (both are zero)."""
    return np.where((q & 7) == 0, 0, q).astype(np.uint8)


def nvfp4_expert_from_device(w4, e: int, I: int, d: int):
    """The CUDA path's NVFP4 matrices of expert e in the oracle's layout: (gate, up, down),
    each (codes [rows, cols], block scales [rows, cols / 16], row scales [rows])."""
    (gc, ga, gs), (dc, da, ds) = w4
    q = unpack_e2m1(gc[e].cpu().numpy())                       # [2I, d]
    b = atoms_to_rows(ga[e].cpu().numpy(), 2 * I, d)           # [2I, d / 16]
    s = gs[e].cpu().numpy()
    def split(x):
        x = x.reshape(I // 64, 2, 64, *x.shape[1:])
        return x[:, 0].reshape(I, *x.shape[3:]), x[:, 1].reshape(I, *x.shape[3:])
    (qg, qu), (bg, bu), (sg, su) = split(q), split(b), split(s)
    qd = unpack_e2m1(dc[e].cpu().numpy())
    bd = atoms_to_rows(da[e].cpu().numpy(), d, I)
    sd = ds[e].cpu().numpy()
    return (qg, bg, sg), (qu, bu, su), (qd, bd, sd)


def oracle_experts_nvfp4(weights, experts, w4=None):
    """The oracle's own NVFP4 quantisation of the listed experts (from the BF16 weights); when
    the CUDA path's weights are given, they must equal the oracle's bit for bit (+-0 alike)."""
    res = {}
    for e in experts:
        parts = _HOST.get(weights, "nvfp4", e, lambda: tuple(
            oracle.quantize_rows_nvfp4(m) for m in host_expert(weights, e)))
        if w4 is not None:
            I, d = weights[0].shape[1], weights[0].shape[2]
            got = nvfp4_expert_from_device(w4, e, I, d)
            for name, (q, b, s), (gq, gb, gs) in zip(("gate", "up", "down"), parts, got):
                assert np.array_equal(canonical_e2m1(gq), canonical_e2m1(q)), f"{e} {name} codes"
                assert np.array_equal(gb, b), f"expert {e} {name}: block scales differ"
                assert np.array_equal(gs, s), f"expert {e} {name}: row scales differ"
        res[e] = parts
    return res


def run_forward_nvfp4(case: Case, w4, ws=None):
    wl = case.wl
    s = bm.shape_of(wl)
    dev = "cuda"
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.beam_moe_forward_nvfp4(s, case.h.to(dev), case.router_w.to(dev), case.bias.to(dev),
                                   w4[0], w4[1], out, idx, w, ws=ws)
    st = bm.beam_moe_sync_status(ws)
    assert st == bm.BEAM_OK, bm.status_string(st)
    return out, idx, w, ws


def oracle_out_nvfp4(case: Case, weights, tokens, w4=None, batch: int = 256):
    """Oracle MoE output (FP32) of the NVFP4 path for ``tokens``; the oracle quantises the BF16
    weights of the experts the tokens use (and checks the CUDA path's weights against them)."""
    tokens = list(tokens)
    experts = oracle_experts_nvfp4(weights, _experts_of(case, tokens), w4)
    out = np.empty((len(tokens), case.wl.d), np.float32)
    for b0 in range(0, len(tokens), batch):
        tb = tokens[b0:b0 + batch]
        out[b0:b0 + len(tb)] = oracle.moe_tokens_nvfp4(tb, case.h, case.idx, case.w, experts)
    return out
