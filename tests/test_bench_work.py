"""bench.py's algorithmic work per launch (the roofline numerators), against the figures the
profile summaries quote for one T = 4096 gate/up launch with all 256 experts touched."""
import importlib.util
import os

from sparse_moe_transformer_fp32_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_gate_up_work_matches_the_profiles():
    b = _bench()
    wl = W.WORKLOADS["prefill"]
    R = wl.T * wl.top_k
    flops = 4 * R * wl.d * wl.I
    for fmt, gbytes in (("bf16", 13.925), ("fp8", 7.046), ("nvfp4", 4.037)):
        work = b.kernel_work(wl, 256, fp8=fmt == "fp8", nvfp4=fmt == "nvfp4")
        gu = work["expert_gemm_gate_up"]
        assert gu["flops"] == flops == 1717986918400
        assert round(gu["bytes"] / 1e9, 3) == gbytes, fmt
    # weights dominate: halving the bytes per weight element roughly halves the launch's bytes
    bf = b.layer_min_bytes(wl, 256)
    f8 = b.layer_min_bytes(wl, 256, fp8=True)
    f4 = b.layer_min_bytes(wl, 256, nvfp4=True)
    assert f4 < f8 < bf and abs(f8 / bf - 0.5) < 0.01 and abs(f4 / bf - 0.28) < 0.01


def test_every_launched_kernel_has_work_for_each_format():
    """The dominant kernel is chosen among the kernels with a work entry: every kernel a layer
    forward launches must have one."""
    b = _bench()
    wl = W.WORKLOADS["prefill"]
    layer = {"router_transpose", "router_gemm", "router_select", "dispatch_scan", "permute",
             "expert_gemm_gate_up", "expert_gemm_down", "combine"}
    assert layer <= set(b.kernel_work(wl, 256))
    assert layer | {"quantize_e4m3"} <= set(b.kernel_work(wl, 256, fp8=True))
    assert layer | {"quantize_nvfp4"} <= set(b.kernel_work(wl, 256, nvfp4=True))
