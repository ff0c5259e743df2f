"""The bench's command-line contract, checked without a GPU: the reference arm (the fp64 oracle
on the host cores) prints one JSON line with every key the contract names, the warm-up floor
of three steps is enforced, and our arm fails loudly instead of falling back to the CPU when
no GPU is present."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = run_bench("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    for key in ("metric", "unit", "config", "data", "dtype", "scaling"):
        assert isinstance(line[key], (str, dict)) and line[key], key
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 1, 3)
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["data"] == "synthetic" and line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["unit"] == line["unit"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("impl", ["ours", "reference"])
def test_fewer_than_three_warmup_steps_are_refused(impl):
    r = run_bench("--impl", impl, "--steps", "1", "--warmup", "2", timeout=120)
    assert r.returncode != 0 and not r.stdout.strip()
    assert "--warmup" in r.stderr


def test_our_arm_fails_loudly_without_a_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the bench itself runs there")
    r = run_bench("--steps", "1", "--warmup", "3", "--cpu-seconds", "0", "--no-e2e", timeout=300)
    assert r.returncode != 0
    assert not r.stdout.strip(), "no JSON line may come out of a run without the GPU path"


def test_reference_arm_under_two_ranks_prints_once():
    # launched the way the scaling run launches every arm; rank 0 alone runs the oracle
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["cpu_baseline"]["cores"] >= 1
