#!/usr/bin/env python
"""Throughput of the Beam sparse-MoE layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill] [--impl cuda|reference]

One step is one whole layer forward (router, dispatch, gate/up GEMM + SwiGLU, down GEMM,
combine; the block workload adds the two RMSNorms and the residual) over one batch of
synthetic tokens, through the C ABI.  With N > 1 (launched by torch.distributed.run) every
rank runs an independent replica of the layer on its own GPU and its own tokens: the layer is
data parallel over tokens and has no exchange step, so there is no collective on the data
path; the barrier and the max-over-ranks of the timed region are the only cross-rank calls.

``--impl reference`` times the CPU oracle (the plain C++ reference of the same layer) on the
host cores on a bounded sample of the same workload, and prints the same JSON line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import contextlib
import dataclasses
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_moe_transformer_fp32_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s at Beam shape T=4096 BF16; % BF16 tensor peak / % HBM BW"
METRIC_FP8 = "MoE-layer tokens/s at Beam shape with FP8 E4M3 expert weights; % FP8 tensor peak / % HBM BW"
METRIC_NVFP4 = ("MoE-layer tokens/s at Beam shape with NVFP4 expert weights; % FP4 tensor peak / "
                "% HBM BW")
NVFP4_BYTES = 0.5 + 1.0 / 16  # one E2M1 code and a sixteenth of an E4M3 block scale per element
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0, "source": "fallback"}
N_SMS = 148
FFMA_PER_SM_PER_CLK = 128


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="prefill", choices=sorted(W.WORKLOADS))
    p.add_argument("--tokens", type=int, default=None,
                   help="override T (profiling-size runs; the JSON names the reduced workload)")
    p.add_argument("--experts", type=int, default=None,
                   help="override E, keeping n_group and topk_group (profiling-size runs)")
    p.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    p.add_argument("--cpu-sample-tokens", type=int, default=128,
                   help="tokens in the oracle's bounded sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--sm-pairs", action="store_true",
                   help="enable the SM-pair (cta_group::2) expert GEMMs for calls with >= 256 "
                        "rows per expert (off by default)")
    p.add_argument("--fp8", action="store_true",
                   help="E4M3 expert weights (beam_moe_forward_fp8); layer workloads only")
    p.add_argument("--nvfp4", action="store_true",
                   help="NVFP4 expert weights (beam_moe_forward_nvfp4, _block_nvfp4, "
                        "beam_dense_forward_nvfp4)")
    p.add_argument("--route-only", action="store_true",
                   help="time beam_moe_route alone (router profiling; not the layer metric)")
    p.add_argument("--ep-ranks", type=int, default=0,
                   help="time the expert-parallel layer step of this many ranks, emulated on one "
                        "GPU rank after rank (their receive buffers all on this GPU; not the "
                        "layer metric)")
    p.add_argument("--dry-run", action="store_true",
                   help="exercise the launch/aggregation logic on CPU (gloo); measures nothing")
    args = p.parse_args(argv)
    if args.warmup < 3 and not args.dry_run:
        p.error("--warmup must be >= 3")
    if args.nvfp4 and args.fp8:
        p.error("--nvfp4 and --fp8 are exclusive")
    return args


def selected_workload(args):
    wl = W.WORKLOADS[args.workload]
    changes = {}
    if args.tokens is not None:
        changes["T"] = args.tokens
    if args.experts is not None:
        changes["E"] = args.experts
    if changes:
        wl = dataclasses.replace(wl, name=wl.name + "-reduced", **changes)
        if wl.E % wl.n_group or wl.top_k > wl.topk_group * (wl.E // wl.n_group):
            raise SystemExit("bench.py: --experts must keep E % n_group == 0 and "
                             "top_k <= topk_group * E / n_group")
    return wl


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


@contextlib.contextmanager
def process_group(world, backend):
    if world <= 1:
        yield None
        return
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    try:
        yield dist
    finally:
        dist.destroy_process_group()


def barrier(dist, device=None):
    if dist is None:
        return
    if device is not None and device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


def max_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ peaks and clocks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def _gpu_selector(device_index: int) -> str:
    """nvidia-smi -i selector of torch's device: its PCI bus id, else its visible index."""
    try:
        p = torch.cuda.get_device_properties(device_index)
        return "%08X:%02X:%02X.0" % (int(p.pci_domain_id), int(p.pci_bus_id), int(p.pci_device_id))
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if device_index < len(ids):
            return str(ids[device_index])
    return str(device_index)


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int, period_ms: int = 50):
        self.sel = _gpu_selector(device_index)
        self.period_ms = period_ms
        self.samples = []
        self.proc = None
        self.window = None

    def start(self):
        cmd = ["nvidia-smi", "-i", self.sel, "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", str(self.period_ms)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True, bufsize=1)
        except (OSError, TypeError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5.0:
            time.sleep(0.01)

    def _reader(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.samples.append((time.time(), parts))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        rows = self.samples
        if self.window:
            inside = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
            rows = inside or rows
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = sorted(v for v in (num(r[1][1]) for r in rows) if v is not None)
        mx = [v for v in (num(r[1][2]) for r in rows) if v is not None]
        pw = [v for v in (num(r[1][3]) for r in rows) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[1][5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ algorithmic work

def kernel_work(wl, touched: int, fp8: bool = False, nvfp4: bool = False):
    """Algorithmic bytes and FLOPs per launch of each kernel (the minimum each must move).
    With fp8 the weights and the GEMM inputs are one-byte E4M3 codes (row scales ignored); with
    nvfp4 they are half-byte E2M1 codes plus one E4M3 block scale per 16 elements."""
    T, d, E, k, I = wl.T, wl.d, wl.E, wl.top_k, wl.I
    R = T * k
    bf, f4 = 2, 4
    if nvfp4:
        q = NVFP4_BYTES
        return {
            "router_transpose": {"flops": 0, "bytes": 2 * E * d * f4},
            "dispatch_scan": {"flops": 0, "bytes": E * 16},
            "router_gemm": {"flops": 2 * T * d * E, "bytes": T * d * bf + E * d * f4 + T * E * f4},
            "router_select": {"flops": 0, "bytes": T * E * f4 + 2 * R * f4},
            "permute": {"flops": 0, "bytes": T * d * bf + R * d * q},
            "expert_gemm_gate_up": {"flops": 4 * R * d * I,
                                    "bytes": touched * 2 * I * d * q + R * d * q + R * I * bf},
            "quantize_nvfp4": {"flops": 0, "bytes": R * I * bf + R * I * q},
            "expert_gemm_down": {"flops": 2 * R * d * I,
                                 "bytes": touched * d * I * q + R * I * q + R * d * bf},
            "combine": {"flops": 2 * R * d, "bytes": R * d * bf + T * d * bf},
            "combine_block": {"flops": 2 * R * d, "bytes": R * d * bf + 3 * T * d * f4},
            "prenorm": {"flops": 3 * T * d, "bytes": T * d * f4 + T * d * bf},
            "dense_tiles": {"flops": 0, "bytes": 16 * (T // 128 + 1)},
        }
    if fp8:
        q = 1
        return {
            "router_transpose": {"flops": 0, "bytes": 2 * E * d * f4},
            "dispatch_scan": {"flops": 0, "bytes": E * 16},
            "router_gemm": {"flops": 2 * T * d * E, "bytes": T * d * bf + E * d * f4 + T * E * f4},
            "router_select": {"flops": 0, "bytes": T * E * f4 + 2 * R * f4},
            "permute": {"flops": 0, "bytes": T * d * bf + R * d * q},
            "expert_gemm_gate_up": {"flops": 4 * R * d * I,
                                    "bytes": touched * 2 * I * d * q + R * d * q + R * I * bf},
            "quantize_e4m3": {"flops": 0, "bytes": R * I * bf + R * I * q},
            "expert_gemm_down": {"flops": 2 * R * d * I,
                                 "bytes": touched * d * I * q + R * I * q + R * d * bf},
            "combine": {"flops": 2 * R * d, "bytes": R * d * bf + T * d * bf},
            "combine_block": {"flops": 2 * R * d, "bytes": R * d * bf + 3 * T * d * f4},
            "prenorm": {"flops": 3 * T * d, "bytes": T * d * f4 + T * d * bf},
            "dense_tiles": {"flops": 0, "bytes": 16 * (T // 128 + 1)},
        }
    w_gu = touched * 2 * I * d * bf
    w_dn = touched * d * I * bf
    return {
        "router_transpose": {"flops": 0, "bytes": 2 * E * d * f4},
        "dispatch_scan": {"flops": 0, "bytes": E * 16},
        "router_gemm": {"flops": 2 * T * d * E, "bytes": T * d * bf + E * d * f4 + T * E * f4},
        "router_select": {"flops": 0, "bytes": T * E * f4 + 2 * R * f4},
        "permute": {"flops": 0, "bytes": T * d * bf + R * d * bf},
        "expert_gemm_gate_up": {"flops": 4 * R * d * I, "bytes": w_gu + R * d * bf + R * I * bf},
        "expert_gemm_down": {"flops": 2 * R * d * I, "bytes": w_dn + R * I * bf + R * d * bf},
        "combine": {"flops": 2 * R * d, "bytes": R * d * bf + T * d * bf},
        "combine_block": {"flops": 2 * R * d, "bytes": R * d * bf + 3 * T * d * f4},
        "prenorm": {"flops": 3 * T * d, "bytes": T * d * f4 + T * d * bf},
    }


def layer_min_bytes(wl, touched: int, fp8: bool = False, nvfp4: bool = False):
    T, d, I = wl.T, wl.d, wl.I
    b = touched * 3 * d * I * (NVFP4_BYTES if nvfp4 else 1 if fp8 else 2) + T * d * 2 * 2
    if wl.block:
        b += 2 * T * d * 4
    return b


GEMM_SOURCES = ("expert_gemm.cu", "beam_moe_internal.cuh")
NVFP4_SOURCES = ("nvfp4.cu", "beam_moe_nvfp4.cuh", "beam_moe_internal.cuh")


def traffic_from_profile(kernel: str, workload: str, sources=GEMM_SOURCES):
    """dram bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (the sha256 of `sources`, in order; else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{16,64})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "sparse_moe_transformer_fp32_b200", "csrc")
    cur = hashlib.sha256()
    for name in sources:
        with open(os.path.join(src, name), "rb") as f:
            cur.update(f.read())
    if not cur.hexdigest().startswith(h.group(1)):
        return None
    return float(m.group(1))


# ------------------------------------------------------------------ oracle (CPU) timing

def oracle_sample_rate(wl, router_w, bias, hidden_cpu, weights_dev, n_tokens: int, repeats=1,
                       nthreads: int = 0):
    """Tokens/s of the CPU oracle on the first n tokens (full layer: logits, routing, experts,
    combine), expert weights copied from the device (not timed); nthreads 0 = all cores."""
    import numpy as np
    import oracle
    oracle.build()
    n_tokens = min(n_tokens, wl.T)
    h = hidden_cpu[:n_tokens]
    sample = wl.with_tokens(n_tokens)
    _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample)
    ex = sorted({int(e) for e in idx.reshape(-1)})
    experts = {e: tuple(m[e].cpu() for m in weights_dev) for e in ex}
    t0 = time.perf_counter()
    for _ in range(repeats):
        _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample, nthreads=nthreads)
        oracle.moe_tokens(np.arange(n_tokens), h, idx, w, experts, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return n_tokens * repeats / dt, dt, nthreads or oracle.hardware_threads()


def oracle_fp8_sample_rate(wl, router_w, bias, hidden_cpu, weights_dev, n_tokens: int):
    """Tokens/s of the CPU oracle's E4M3 layer on the first n tokens; the oracle converts the
    experts those tokens use from the BF16 weights first (not timed: a one-off conversion)."""
    import numpy as np
    import oracle
    oracle.build()
    n_tokens = min(n_tokens, wl.T)
    h = hidden_cpu[:n_tokens]
    sample = wl.with_tokens(n_tokens)
    _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample)
    experts = {}
    for e in sorted({int(e) for e in idx.reshape(-1)}):
        parts = []
        for m in weights_dev:
            parts += list(oracle.quantize_rows_e4m3(m[e].cpu()))
        experts[e] = tuple(parts)
    t0 = time.perf_counter()
    _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample)
    oracle.moe_tokens_fp8(np.arange(n_tokens), h, idx, w, experts)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, oracle.hardware_threads()


def oracle_nvfp4_sample_rate(wl, router_w, bias, hidden_cpu, weights_dev, n_tokens: int):
    """Tokens/s of the CPU oracle's NVFP4 layer on the first n tokens; the oracle converts the
    experts those tokens use from the BF16 weights first (not timed: a one-off conversion)."""
    import numpy as np
    import oracle
    oracle.build()
    n_tokens = min(n_tokens, wl.T)
    h = hidden_cpu[:n_tokens]
    sample = wl.with_tokens(n_tokens)
    _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample)
    experts = {e: tuple(oracle.quantize_rows_nvfp4(m[e].cpu()) for m in weights_dev)
               for e in sorted({int(e) for e in idx.reshape(-1)})}
    t0 = time.perf_counter()
    _, idx, w, _, _ = oracle.layer_routing(h, router_w, bias, sample)
    oracle.moe_tokens_nvfp4(np.arange(n_tokens), h, idx, w, experts)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, oracle.hardware_threads()


def oracle_dense_rate(wl, hidden_cpu, weights_dev, n_tokens: int):
    import oracle
    oracle.build()
    n = min(n_tokens, wl.T)
    mats = tuple(m[0].cpu() for m in weights_dev)
    t0 = time.perf_counter()
    oracle.dense_mlp(range(n), hidden_cpu[:n], *mats)
    dt = time.perf_counter() - t0
    return n / dt, dt, oracle.hardware_threads()


# ------------------------------------------------------------------ the CUDA arm

def replica_workload(wl, rank):
    # every replica holds the same layer weights and processes its own tokens
    return dataclasses.replace(wl, seed=W.seed_for(wl.seed, 1000 + rank)) if rank else wl


def run_cuda(args, rank, world, local):
    from sparse_moe_transformer_fp32_b200 import beam_moe as bm
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device; the CUDA path has no CPU fallback")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    bm.lib()  # fails loudly if the extension is missing
    bm.beam_moe_set_sm_pairs(bool(args.sm_pairs))
    wl = selected_workload(args)
    peaks = load_peaks()
    with process_group(world, "nccl") as dist:
        s = bm.shape_of(wl)
        router_w = W.router_weight(wl).to(dev)
        bias = W.router_bias(wl).to(dev)
        weights = W.expert_weights(wl, dev)
        mine = replica_workload(wl, rank)
        if wl.dense:
            ds = bm.dense_shape(wl.T, wl.d, wl.I)
        if wl.block:
            x_cpu = W.residual_x(mine)
            g_pre, g_post = (g.to(dev) for g in W.norm_gains(wl))
            x = x_cpu.to(dev)
            x_out = torch.empty_like(x)
            inp_cpu, inp, res = x_cpu, x, x_out
        else:
            h_cpu = W.hidden(mine)
            h = h_cpu.to(dev)
            out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
            inp_cpu, inp, res = h_cpu, h, out
        fp8 = None
        fp4 = None
        if args.nvfp4:
            fp4 = (bm.beam_moe_quantize_nvfp4(weights[0], weights[1]),
                   bm.beam_moe_quantize_nvfp4(weights[2]))
            torch.cuda.synchronize(dev)
        if args.fp8:
            fp8 = []
            for m in weights:
                fp8 += list(bm.beam_moe_quantize_e4m3(m[0] if wl.dense else m))
            torch.cuda.synchronize(dev)
        if wl.dense and not fp4:
            ws = bm.dense_fp8_workspace(ds, dev) if fp8 else bm.dense_workspace(ds, dev)
        elif fp4:
            ws = bm.dense_nvfp4_workspace(ds, dev) if wl.dense else bm.nvfp4_workspace(s, dev)
        else:
            ws = bm.fp8_workspace(s, dev) if fp8 else bm.workspace(s, dev)
        stream = torch.cuda.current_stream(dev)

        def step(src=None, dst=None):
            src = inp if src is None else src
            dst = res if dst is None else dst
            if wl.dense and fp4:
                bm.beam_dense_forward_nvfp4(ds, src, fp4[0], fp4[1], dst, ws=ws)
            elif wl.block and fp4:
                bm.beam_moe_block_nvfp4(s, src, g_pre, g_post, wl.eps, wl.k_resid, router_w, bias,
                                        fp4[0], fp4[1], dst, ws=ws)
            elif wl.dense and fp8:
                bm.beam_dense_forward_fp8(ds, src, *fp8, dst, ws=ws)
            elif wl.dense:
                bm.beam_dense_forward(ds, src, weights[0][0], weights[1][0], weights[2][0], dst,
                                      ws=ws)
            elif wl.block and fp8:
                bm.beam_moe_block_fp8(s, src, g_pre, g_post, wl.eps, wl.k_resid, router_w, bias,
                                      *fp8, dst, ws=ws)
            elif wl.block:
                bm.beam_moe_block(s, src, g_pre, g_post, wl.eps, wl.k_resid, router_w, bias,
                                  *weights, dst, ws=ws)
            elif fp4:
                bm.beam_moe_forward_nvfp4(s, src, router_w, bias, fp4[0], fp4[1], dst, ws=ws)
            elif fp8:
                bm.beam_moe_forward_fp8(s, src, router_w, bias, *fp8, dst, ws=ws)
            else:
                bm.beam_moe_forward(s, src, router_w, bias, *weights, dst, ws=ws)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        st = bm.beam_moe_sync_status(ws)
        if st != bm.BEAM_OK:
            raise SystemExit(f"bench.py: device status {bm.status_string(st)}")
        counts = (torch.tensor([wl.T], dtype=torch.int32) if wl.dense
                  else bm.beam_moe_expert_counts(s, ws))
        touched = int((counts > 0).sum())

        # ---- timed region (device time, max over ranks)
        clocks = ClockSampler(dev.index)
        clocks.start()
        bm.beam_moe_profile_reset()
        bm.beam_moe_profile_enable(True)
        launches0 = bm.beam_moe_launch_count()
        barrier(dist, dev)
        torch.cuda.synchronize(dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.time()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        w1 = time.time()
        barrier(dist, dev)
        bm.beam_moe_profile_enable(False)
        clocks.mark(w0, w1)
        clocks.stop()
        gpu_launches = bm.beam_moe_launch_count() - launches0
        ms_local = ev0.elapsed_time(ev1)
        ms_total = max_over_ranks(dist, ms_local, dev)
        prof = bm.beam_moe_profile_read()
        st = bm.beam_moe_sync_status(ws)
        if st != bm.BEAM_OK:
            raise SystemExit(f"bench.py: device status {bm.status_string(st)}")
        tokens_all = sum_over_ranks(dist, float(wl.T * args.steps), dev)
        value = tokens_all / (ms_total / 1e3)
        ms_per_step = ms_total / args.steps

        # ---- end to end: pinned host input -> device -> layer -> host result, every step.
        # Copies run on their own streams with two buffers each, so step i's upload and
        # step i-1's download overlap step i's layer; events order every reuse of a buffer.
        e2e = None
        if not args.no_e2e:
            host_in = inp_cpu.pin_memory()
            host_out = [torch.empty(res.shape, dtype=res.dtype).pin_memory() for _ in range(2)]
            dev_in = [torch.empty_like(inp) for _ in range(2)]
            dev_out = [torch.empty_like(res) for _ in range(2)]
            s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            mk = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
            in_done, comp_done, out_done = mk(), mk(), mk()

            def pipelined(n):
                for i in range(n):
                    b = i % 2
                    if i >= 2:
                        s_in.wait_event(comp_done[b])      # step i-2 finished reading dev_in[b]
                    with torch.cuda.stream(s_in):
                        dev_in[b].copy_(host_in, non_blocking=True)
                    in_done[b].record(s_in)
                    stream.wait_event(in_done[b])
                    if i >= 2:
                        stream.wait_event(out_done[b])     # dev_out[b] of step i-2 copied out
                    step(dev_in[b], dev_out[b])
                    comp_done[b].record(stream)
                    s_out.wait_event(comp_done[b])
                    with torch.cuda.stream(s_out):
                        host_out[b].copy_(dev_out[b], non_blocking=True)
                    out_done[b].record(s_out)
                for b in range(2):
                    stream.wait_event(out_done[b])

            pipelined(3)
            barrier(dist, dev)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            s_in.wait_event(e0)
            s_out.wait_event(e0)
            pipelined(args.steps)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(dist, dev)
            e_ms = max_over_ranks(dist, e0.elapsed_time(e1), dev)
            e2e = {"value": tokens_all / (e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": host_in.numel() * host_in.element_size(),
                   "d2h_bytes_per_step": host_out[0].numel() * host_out[0].element_size(),
                   "overlap": "uploads and downloads on their own streams, double-buffered"}

        result = None
        if rank == 0:
            work = kernel_work(wl, touched, fp8=bool(fp8), nvfp4=bool(fp4))
            per_kernel = {k: {"launches": n, "ms_per_launch": (ms / n if n else None)}
                          for k, (n, ms) in prof.items() if n}
            dom = max((k for k in per_kernel if k in work), key=lambda k: prof[k][1])
            n_dom, ms_dom = prof[dom]
            avg_s = ms_dom / n_dom / 1e3
            wk = work[dom]
            hbm_t = wk["bytes"] / (peaks["hbm_gbs"] * 1e9)
            ten_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
            if fp8:
                ten_peak *= 2  # FP8 dense tensor rate: the measured BF16 rate x the nominal 2
            if fp4:
                ten_peak *= 4  # FP4 dense tensor rate: the measured BF16 rate x the nominal 4
            if dom == "router_gemm":
                clk = float(peaks.get("sm_max_mhz", 1965.0))
                alu_peak = N_SMS * FFMA_PER_SM_PER_CLK * 2 * clk * 1e6 / 1e12
                roof = {"bound": "alu", "achieved": wk["flops"] / avg_s / 1e12, "peak": alu_peak,
                        "unit": "TFLOP/s"}
            elif wk["flops"] / (ten_peak * 1e12) > hbm_t:
                roof = {"bound": "tensor", "achieved": wk["flops"] / avg_s / 1e12,
                        "peak": ten_peak, "unit": "TFLOP/s"}
            else:
                roof = {"bound": "hbm", "achieved": wk["bytes"] / avg_s / 1e9,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s"}
            roof["frac"] = roof["achieved"] / roof["peak"]
            roof["kernel"] = dom
            roof["peak_source"] = peaks.get("source", "measured")
            if fp8 and roof["bound"] == "tensor":
                roof["peak_source"] += " bf16 x 2 (nominal FP8:BF16 ratio)"
            if fp4 and roof["bound"] == "tensor":
                roof["peak_source"] += " bf16 x 4 (nominal FP4:BF16 ratio)"
            if fp4:
                roof["traffic"] = traffic_from_profile(dom, wl.name + "-nvfp4", NVFP4_SOURCES)
            else:
                roof["traffic"] = traffic_from_profile(dom, wl.name + ("-fp8" if fp8 else ""))
            roof["algorithmic_per_launch"] = wk["bytes"] if roof["bound"] == "hbm" else wk["flops"]
            roof["tensor_frac_of_sustained"] = (wk["flops"] / avg_s / 1e12) / ten_peak
            roof["hbm_frac"] = (wk["bytes"] / avg_s / 1e9) / peaks["hbm_gbs"]

            step_s = ms_per_step / 1e3
            flops_step = 6 * wl.T * wl.top_k * wl.d * wl.I  # top_k = 1 for the dense MLP
            bytes_step = layer_min_bytes(wl, touched, fp8=bool(fp8), nvfp4=bool(fp4))
            cpu = None
            result_extra = {}
            if fp4 and not args.no_cpu_baseline and world == 1 and not (wl.dense or wl.block):
                n_cpu = min(args.cpu_sample_tokens, 16)
                rate, secs, cores = oracle_nvfp4_sample_rate(
                    wl, W.router_weight(wl), W.router_bias(wl), inp_cpu, weights, n_cpu)
                cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                       "sample": f"first {n_cpu} tokens of the {wl.name} workload, full NVFP4 "
                                 f"layer (router logits, routing, {wl.top_k} NVFP4 SwiGLU experts "
                                 f"each, combine) in double-accumulating C++; {secs:.2f} s"}
            elif fp4:
                pass
            elif fp8 and (wl.dense or wl.block):
                pass  # the E4M3 CPU baseline is timed on the layer workloads only
            elif not args.no_cpu_baseline and world == 1 and fp8:
                n_cpu = min(args.cpu_sample_tokens, 16)
                rate, secs, cores = oracle_fp8_sample_rate(
                    wl, W.router_weight(wl), W.router_bias(wl), inp_cpu, weights, n_cpu)
                cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                       "sample": f"first {n_cpu} tokens of the {wl.name} workload, full E4M3 "
                                 f"layer (router logits, routing, {wl.top_k} E4M3 SwiGLU experts "
                                 f"each, combine) in double-accumulating C++; {secs:.2f} s"}
            elif not args.no_cpu_baseline and world == 1 and wl.dense:
                rate, secs, cores = oracle_dense_rate(wl, inp_cpu, weights, args.cpu_sample_tokens)
                cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                       "sample": f"first {args.cpu_sample_tokens} tokens of the dense workload, "
                                 f"SwiGLU MLP in double-accumulating C++; {secs:.2f} s"}
            elif not args.no_cpu_baseline and world == 1:
                rate, secs, cores = oracle_sample_rate(
                    wl, W.router_weight(wl), W.router_bias(wl),
                    inp_cpu if not wl.block else _block_h(wl, mine, g_pre), weights,
                    args.cpu_sample_tokens)
                cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                       "sample": f"first {min(args.cpu_sample_tokens, wl.T)} tokens of the "
                                 f"{wl.name} workload, "
                                 f"full layer (router logits, routing, {wl.top_k} SwiGLU experts "
                                 f"each, combine) in double-accumulating C++; {secs:.2f} s"}
                if wl.name in ("tiny", "decode"):  # the small configurations also on one core
                    n1 = min(args.cpu_sample_tokens, wl.T)
                    rate1, secs1, _ = oracle_sample_rate(
                        wl, W.router_weight(wl), W.router_bias(wl), inp_cpu, weights, n1,
                        nthreads=1)
                    result_extra["cpu_baseline_1core"] = {
                        "value": rate1, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                        "sample": f"first {n1} tokens, one host thread; {secs1:.2f} s"}
            result = {
                "metric": METRIC_NVFP4 if fp4 else METRIC_FP8 if fp8 else METRIC,
                "value": value, "unit": "tokens/s",
                "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e2m1" if fp4 else "e4m3" if fp8 else "bf16", "data": "synthetic",
                "config": {"workload": f"{wl.name}{'-fp8' if fp8 else ''}"
                                       f"{'-nvfp4' if fp4 else ''}"
                                       f"{'-smpairs' if args.sm_pairs else ''}: T={wl.T} d={wl.d} "
                                       f"E={wl.E} n_group={wl.n_group} "
                                       f"topk_group={wl.topk_group} top_k={wl.top_k} I={wl.I}"
                                       + (" block" if wl.block else ""),
                           "tokens_per_gpu": wl.T, "global_tokens": wl.T * world,
                           "parallelism": f"replicas x{world} (data parallel over tokens)",
                           "l2": "inputs larger than L2: every step streams the touched experts' "
                                 f"weights ({touched} of {wl.E} experts, "
                                 f"{layer_min_bytes(wl, touched, bool(fp8), bool(fp4)) / 1e9:.2f}"
                                 " GB with the activations) "
                                 "from HBM",
                           "touched_experts": touched,
                           "max_expert_load": int(counts.max()),
                           "top16_share": float(counts.sort(descending=True).values[:16].sum()
                                                / counts.sum())},
                "tflops": flops_step / step_s / 1e12,
                "hbm_gbs_layer_min_bytes": bytes_step / step_s / 1e9,
                "roofline": roof,
                "kernels": per_kernel,
                "gpu_launches": gpu_launches,
                "clocks": clocks.summary(),
                "e2e": e2e,
                "cpu_baseline": cpu,
                **result_extra,
            }
        barrier(dist, dev)
        del weights, fp8, fp4
    return result


def _block_h(wl, mine, g_pre):
    import numpy as np
    import oracle
    x = W.residual_x(mine)
    bits = oracle.block_prenorm(x, g_pre.cpu(), wl.eps)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


# ------------------------------------------------------------------ the reference arm (oracle)

def run_reference(args, rank, world, local):
    """The oracle on the host cores, one bounded sample of the workload per step.  The sample
    size is chosen from a one-token calibration so that warm-up plus timed steps take about
    two minutes."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    oracle.build()
    wl = selected_workload(args)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    router_w, bias = W.router_weight(wl), W.router_bias(wl)
    if wl.block:
        g_pre, _ = W.norm_gains(wl)
        h = _block_h(wl, wl, g_pre)
    else:
        h = W.hidden(wl)

    def prepare(n):
        sample = wl.with_tokens(n)
        _, idx, _, _, _ = oracle.layer_routing(h[:n], router_w, bias, sample)
        ex = sorted({int(e) for e in idx.reshape(-1)})
        experts = {e: tuple(W.expert_weight(wl, m, e, dev).cpu() for m in ("gate", "up", "down"))
                   for e in ex}
        if args.fp8:  # the oracle converts the experts itself (a one-off, not timed)
            experts = {e: tuple(p for m in mats for p in oracle.quantize_rows_e4m3(m))
                       for e, mats in experts.items()}
        if args.nvfp4:
            experts = {e: tuple(oracle.quantize_rows_nvfp4(m) for m in mats)
                       for e, mats in experts.items()}
        return sample, experts

    def one_step(n, sample, experts):
        _, ix, ww, _, _ = oracle.layer_routing(h[:n], router_w, bias, sample)
        if args.nvfp4:
            oracle.moe_tokens_nvfp4(np.arange(n), h[:n], ix, ww, experts)
        elif args.fp8:
            oracle.moe_tokens_fp8(np.arange(n), h[:n], ix, ww, experts)
        else:
            oracle.moe_tokens(np.arange(n), h[:n], ix, ww, experts)

    sample1, experts1 = prepare(1)
    t0 = time.perf_counter()
    one_step(1, sample1, experts1)
    t_tok = time.perf_counter() - t0
    budget_s = 120.0
    n = int(budget_s / max(1e-6, (args.steps + args.warmup) * t_tok))
    n = max(1, min(n, args.cpu_sample_tokens, wl.T))
    sample, experts = prepare(n)
    for _ in range(args.warmup):
        one_step(n, sample, experts)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step(n, sample, experts)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    cores = oracle.hardware_threads()
    kind = "NVFP4 " if args.nvfp4 else "E4M3 " if args.fp8 else ""
    desc = (f"first {n} tokens of the {wl.name} workload per step, full {kind}layer (router "
            f"logits, routing, {wl.top_k} {kind}SwiGLU experts per token, combine) in "
            f"double-accumulating C++ on {cores} host threads")
    metric = METRIC_NVFP4 if args.nvfp4 else METRIC_FP8 if args.fp8 else METRIC
    return {"impl": "reference", "metric": metric, "value": value,
            "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{wl.name}: T={wl.T} d={wl.d} E={wl.E} top_k={wl.top_k} "
                                   f"I={wl.I} (sample of {n} tokens per step)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ expert parallelism, emulated

def run_ep_emulated(args, rank, world, local):
    """The expert-parallel step of P ranks (each with T / P tokens and E / P experts) run rank
    after rank on one GPU: count, dispatch, experts and combine of every rank per step, the
    receive buffers all on this GPU, so the exchange is local stores and loads instead of NVLink
    ones.  Routing comes from one beam_moe_forward of the whole batch, made before timing."""
    from sparse_moe_transformer_fp32_b200 import beam_moe as bm
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = selected_workload(args)
    P = args.ep_ranks
    if wl.E % P or wl.T % P:
        raise SystemExit("bench.py: --ep-ranks must divide E and T")
    ep, Tp = wl.E // P, wl.T // P
    weights = W.expert_weights(wl, dev)
    h = W.hidden(wl).to(dev)
    s = bm.shape_of(wl)
    out_ref = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    bm.beam_moe_forward(s, h, W.router_weight(wl).to(dev), W.router_bias(wl).to(dev), *weights,
                        out_ref, idx, w)
    torch.cuda.synchronize(dev)
    owners = (idx // ep).cpu()
    cap = max(int((owners == q).sum()) for q in range(P))
    sp = bm.shape_of(wl, Tp)
    wss = [bm.ep_workspace(sp, P, cap, dev) for _ in range(P)]
    counts = [torch.empty(wl.E, dtype=torch.int32, device=dev) for _ in range(P)]
    all_counts = torch.empty(P, wl.E, dtype=torch.int32, device=dev)
    xrecv = [torch.empty(cap, wl.d, dtype=torch.bfloat16, device=dev) for _ in range(P)]
    yrecv = [torch.empty(cap, wl.d, dtype=torch.bfloat16, device=dev) for _ in range(P)]
    out = torch.empty_like(out_ref)
    sl = [slice(p * Tp, (p + 1) * Tp) for p in range(P)]
    wg, wu, wd = weights

    def step():
        for p in range(P):
            bm.beam_moe_ep_count(sp, P, idx[sl[p]], counts[p], cap, wss[p])
        for p in range(P):  # the all-gather, here one device copy per rank
            all_counts[p].copy_(counts[p])
        for p in range(P):
            bm.beam_moe_ep_dispatch(sp, P, p, h[sl[p]], idx[sl[p]], all_counts, xrecv, cap, wss[p])
        for q in range(P):
            e0, e1 = q * ep, (q + 1) * ep
            bm.beam_moe_ep_experts(sp, P, q, wl.T, all_counts, wg[e0:e1], wu[e0:e1], wd[e0:e1],
                                   xrecv[q], yrecv[q], cap, wss[q])
        for p in range(P):
            bm.beam_moe_ep_combine(sp, P, w[sl[p]], yrecv, cap, out[sl[p]], wss[p])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    for ws in wss:
        st = bm.beam_moe_sync_status(ws)
        if st != bm.BEAM_OK:
            raise SystemExit(f"bench.py: device status {bm.status_string(st)}")
    exact = bool(torch.equal(out.view(torch.int16), out_ref.view(torch.int16)))
    bm.beam_moe_profile_reset()
    bm.beam_moe_profile_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        step()
    ev1.record()
    torch.cuda.synchronize(dev)
    bm.beam_moe_profile_enable(False)
    ms = ev0.elapsed_time(ev1) / args.steps
    prof = bm.beam_moe_profile_read()
    R = wl.T * wl.top_k
    row = wl.d * 2
    kernels = {k: {"launches": n, "ms_per_launch": ms_ / n} for k, (n, ms_) in prof.items() if n}
    # bytes each exchange kernel must move in one step, all ranks together
    ex = {"ep_push": wl.T * row + R * row, "ep_combine": R * row + wl.T * row}
    peaks = load_peaks()
    exchange = {}
    for k, b in ex.items():
        if k in prof and prof[k][0]:
            t_step = prof[k][1] / args.steps / 1e3
            exchange[k] = {"ms_per_step": t_step * 1e3, "gbs": b / t_step / 1e9,
                           "hbm_frac": b / t_step / 1e9 / peaks["hbm_gbs"]}
    return {"metric": "expert-parallel layer step tokens/s, ranks emulated on one GPU "
                      "(not the layer metric)",
            "value": wl.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps,
            "warmup": args.warmup, "ep_ranks": P, "recv_rows_max": cap,
            "bit_equal_to_single_gpu_forward": exact,
            "config": {"workload": f"{wl.name}: T={wl.T} d={wl.d} E={wl.E} top_k={wl.top_k} "
                                   f"I={wl.I}, {P} ranks of {Tp} tokens and {ep} experts"},
            "exchange": exchange, "kernels": kernels}


# ------------------------------------------------------------------ router alone (profiling)

def run_route_only(args, rank, world, local):
    from sparse_moe_transformer_fp32_b200 import beam_moe as bm
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = selected_workload(args)
    s = bm.shape_of(wl)
    h = W.hidden(wl).to(dev)
    router_w, bias = W.router_weight(wl).to(dev), W.router_bias(wl).to(dev)
    idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.top_k, dtype=torch.float32, device=dev)
    ws = bm.workspace(s, dev)
    for _ in range(args.warmup):
        bm.beam_moe_route(s, h, router_w, bias, idx, w, ws=ws)
    torch.cuda.synchronize(dev)
    bm.beam_moe_profile_reset()
    bm.beam_moe_profile_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        bm.beam_moe_route(s, h, router_w, bias, idx, w, ws=ws)
    ev1.record()
    torch.cuda.synchronize(dev)
    bm.beam_moe_profile_enable(False)
    ms = ev0.elapsed_time(ev1) / args.steps
    prof = bm.beam_moe_profile_read()
    st = bm.beam_moe_sync_status(ws)
    if st != bm.BEAM_OK:
        raise SystemExit(f"bench.py: device status {bm.status_string(st)}")
    flops = 2.0 * wl.T * wl.d * wl.E
    return {"metric": "router tokens/s (beam_moe_route alone)", "value": wl.T / (ms / 1e3),
            "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
            "router_fp32_tflops": flops / (ms / 1e3) / 1e12,
            "config": {"workload": f"{wl.name}: T={wl.T} d={wl.d} E={wl.E}"},
            "kernels": {k: {"launches": n, "ms_per_launch": ms_ / n} for k, (n, ms_) in prof.items() if n}}


# ------------------------------------------------------------------ dry run (host logic only)

def run_dry(args, rank, world, local):
    """Exercises rank setup, barriers and the max/sum aggregation on CPU ranks (gloo)."""
    with process_group(world, "gloo") as dist:
        dev = torch.device("cpu")
        barrier(dist)
        local_ms = 10.0 * (rank + 1)
        ms = max_over_ranks(dist, local_ms, dev)
        tokens = sum_over_ranks(dist, float(W.WORKLOADS[args.workload].T * args.steps), dev)
        barrier(dist)
    if rank != 0:
        return None
    return {"dry_run": True, "n_gpus": world, "steps": args.steps, "max_ms": ms,
            "tokens_all_ranks": tokens, "value_if_measured": tokens / (ms / 1e3)}


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if world != args.gpus and not args.dry_run:
        if world == 1 and args.gpus > 1:
            raise SystemExit("bench.py: --gpus N > 1 must be launched with torch.distributed.run")
    if args.dry_run:
        res = run_dry(args, rank, world, local)
    elif args.route_only:
        res = run_route_only(args, rank, world, local)
    elif args.ep_ranks:
        res = run_ep_emulated(args, rank, world, local)
    elif args.impl == "reference":
        res = run_reference(args, rank, world, local)
    else:
        res = run_cuda(args, rank, world, local)
    if res is not None and rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
