"""bench.py's reference arm (the fp64 oracle on the host cores) keeps the JSON-line contract.

Runs on the CPU: the reference arm needs no GPU.  Under torchrun only rank 0 times and prints;
the other ranks exit 0 without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, env=None):
    r = subprocess.run([sys.executable] + args, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="2", **(env or {})))
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(line) for line in r.stdout.splitlines() if line.startswith("{")]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_decode_reference_line():
    sys.path.insert(0, ROOT)
    import bench
    (line,) = _run(["bench.py", "--impl", "reference", "--workload", "gta_tiny", "--steps", "2", "--warmup", "3"])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is False and line["value"] > 0 and line["steps"] == 2
    assert line["warmup"] >= 3 and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "GTA" in line["config"]["workload"]


def test_append_reference_line():
    (line,) = _run(["bench.py", "--impl", "reference", "--workload", "append_gta", "--tokens", "256"])
    assert KEYS <= set(line) and line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_reference_under_torchrun_prints_once():
    lines = _run(["-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
                  "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference", "--gpus", "2",
                  "--workload", "gta_tiny", "--steps", "1", "--warmup", "3"])
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
