"""The benchmark's reference arm (the CPU oracle) prints one JSON line with the
keys the benchmark contract names, alone and under a two-process launch."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"]


def _json_lines(out: str):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_line(d: dict, n_gpus: int):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["n_gpus"] == n_gpus and d["steps"] == 1 and d["warmup"] >= 3
    assert d["unit"] == "tok/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "decode_7b_ctx16384_b8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["sample"]
    assert cb["cores"] == len(os.sched_getaffinity(0))
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_one_process():
    r = subprocess.run([sys.executable] + ARGS, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1)


def test_reference_arm_two_processes():
    """Rank 0 alone prints the line (on every core); rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29531"] + ARGS[:1] + ["--gpus", "2"] + ARGS[1:]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 2)


def test_packed_step_inputs_share_one_buffer():
    """The end-to-end decode line moves a step's inputs in one copy: the views
    that `_packed_inputs` returns hold the given values, sit at 256-byte-aligned
    offsets of one flat buffer, and a copy of the whole buffer moves them all."""
    import torch

    sys.path.insert(0, ROOT)
    import bench

    g = torch.Generator().manual_seed(3)
    src = {"q": torch.randn(8, 1, 28, 128, generator=g).to(torch.bfloat16),
           "w": torch.rand(8, 1, 8, generator=g),
           "gate": torch.randn(8, 1, 28, generator=g).to(torch.bfloat16)}
    flat, views = bench._packed_inputs(src, lambda nb: torch.zeros(nb, dtype=torch.uint8))
    base = flat.data_ptr()
    for k, t in src.items():
        v = views[k]
        assert v.dtype == t.dtype and v.shape == t.shape and torch.equal(v, t)
        assert (v.data_ptr() - base) % 256 == 0
        assert base <= v.data_ptr() and v.data_ptr() + v.numel() * v.element_size() <= base + flat.numel()
    flat2, views2 = bench._packed_inputs({k: torch.zeros_like(t) for k, t in src.items()},
                                         lambda nb: torch.zeros(nb, dtype=torch.uint8))
    assert flat2.numel() == flat.numel()
    flat2.copy_(flat)
    for k, t in src.items():
        assert torch.equal(views2[k], t)
