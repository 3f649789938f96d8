"""bench.py's host-side contract, on the CPU: the reference arm's JSON line
(the oracle timed on the host cores), its behaviour under torchrun with two
ranks (rank 0 alone prints, the other exits without work), and the guard that
reports ncu DRAM traffic only for the kernel source it was captured from."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def _check_reference_line(d, n_gpus):
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == n_gpus and d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith(bench.WORKLOAD_NAME)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = _json_lines(out.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0], 1)          # a warm-up below 3 is raised to 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = _json_lines(out.stdout)
    assert len(lines) == 1                      # rank 0 alone prints
    _check_reference_line(lines[0], 2)


def test_traffic_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    good = tmp_path / "good.md"
    good.write_text(f"kernel_source_sha256: {bench.kernel_source_hash()}\ncaptured_launch_M: 1\n"
                    "dram_bytes_per_launch: 50443776\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(good))
    assert bench.profiled_traffic() == {"bytes": 50443776, "M": 1}
    stale = tmp_path / "stale.md"
    stale.write_text("kernel_source_sha256: 0000000000000000\ncaptured_launch_M: 1\n"
                     "dram_bytes_per_launch: 50443776\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(stale))
    assert bench.profiled_traffic() is None
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(tmp_path / "absent.md"))
    assert bench.profiled_traffic() is None


def test_algorithmic_bytes():
    # packed weights, fp16 scales, fp16 activations of one launch
    assert bench.algo_bytes(1, 8192, 8192) == 0.75 * 8192 * 8192 + 2 * 8192 + 2 * 8192
    assert bench.algo_bytes(16, 8192, 8192, 0.5) == 0.5 * 8192 * 8192 + 2 * 8192 + 2 * 16 * 8192


_MAX_CHILD = r"""
import os, sys, datetime
sys.path.insert(0, os.environ["REPO"])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank = dist.get_rank()
bench.barrier(2)
t = bench.max_over_ranks(1.5 + rank, 2)          # rank 1 is the slower one
assert t == 2.5, t
assert bench.max_over_ranks(7.0, 1) == 7.0       # one rank: no collective
dist.destroy_process_group()
open(os.path.join(os.environ["OUT"], f"ok{rank}"), "w").close()
"""


def test_step_time_is_the_max_over_two_ranks(tmp_path):
    """The timing of an N-rank run is the slowest rank's (gloo ranks on the CPU)."""
    script = tmp_path / "max_child.py"
    script.write_text(_MAX_CHILD)
    env = dict(os.environ, REPO=ROOT, OUT=str(tmp_path))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), str(script)]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert (tmp_path / "ok0").exists() and (tmp_path / "ok1").exists()
