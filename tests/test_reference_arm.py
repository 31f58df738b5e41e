"""bench.py's reference arm (the fp64 oracle on the host cores) keeps the bench contract on CPU:
one JSON line from rank 0 with the GPU arm's metric, unit and config, and under torchrun with two
ranks the other rank exits 0 without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["bench.py", "--impl", "reference", "--workload", "32k", "--steps", "1", "--warmup", "0",
        "--ref-seconds", "0.5"]


def _json_lines(out: str) -> list[dict]:
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_line(d: dict, n: int) -> None:
    import bench
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["n_gpus"] == n and d["steps"] == 1 and d["warmup"] == 0 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"] == "prefill_32k" and d["config"]["L"] == 32768


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, *ARGS, "--gpus", "1"], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1)


def test_reference_arm_two_ranks_under_torchrun():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), *ARGS, "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1                      # rank 0 alone prints
    _check_line(lines[0], 2)
    assert lines[0]["config"]["parallelism"].startswith("dp2")
