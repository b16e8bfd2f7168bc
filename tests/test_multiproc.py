"""The N > 1 launch path on CPU: two gloo ranks run bench.py's rank setup, barriers and
max/sum-over-ranks aggregation (bench.py --dry-run), and only rank 0 prints one JSON line."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_dry_run_aggregates_on_rank0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--steps", "4"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    r = json.loads(lines[0])
    assert r["dry_run"] and r["n_gpus"] == 2
    assert r["max_ms"] == 20.0                      # the slower rank's time
    assert r["tokens_all_ranks"] == 2 * 4096 * 4    # every rank's tokens


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def _reference_line(*extra):
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3",
                        "--cpu-sample-tokens", "4", *extra],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    return json.loads(lines[0])


def test_reference_arm_line_carries_the_contract_keys():
    for extra, metric_word in (((), "BF16"), (("--fp8",), "E4M3"), (("--nvfp4",), "NVFP4")):
        r = _reference_line(*extra)
        assert r["impl"] == "reference" and metric_word in r["metric"]
        assert r["unit"] == "tokens/s" and r["value"] > 0 and r["higher_is_better"] is True
        assert r["steps"] == 3 and r["warmup"] == 3 and r["n_gpus"] == 1
        assert r["dtype"] == "f64" and r["data"] == "synthetic"
        assert r["config"]["workload"].startswith("tiny")
        cb = r["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1
        assert "4 tokens" in cb["sample"]
        assert r["e2e"] == {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}
