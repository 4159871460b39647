"""The benchmark's host-side contract, checked on CPU: the reference arm (the oracle timed on the host) prints
one JSON line with the keys the driver reads, and the algorithmic work model is consistent."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from approximate_long_context_b200 import workload as wl  # noqa: E402


@pytest.mark.parametrize("sampling", ["uniform", "rownorm"])
def test_reference_arm_prints_one_json_line(sampling):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_fp32_n1024", "--steps", "2", "--warmup", "3", "--sampling", sampling],
                         capture_output=True, text=True, check=True, timeout=300, cwd=ROOT).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["steps"] == 2
    assert rec["config"]["workload"] == "tiny_fp32_n1024"
    assert rec["e2e"]["value"] == rec["value"] and rec["e2e"]["h2d_bytes_per_step"] == 0
    assert (rec["config"].get("sampling") == "rownorm") == (sampling == "rownorm")


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_fp32_n1024", "--steps", "1", "--warmup", "2"], capture_output=True, text=True,
                       timeout=120, cwd=ROOT)
    assert r.returncode != 0


def test_work_model():
    w = wl.WORKLOADS[wl.HEADLINE]
    _, f_u = bench.algorithmic(w, "attn")
    _, f_r = bench.algorithmic(w, "attn", "rownorm")
    # 4 d FLOPs per (query, key) pair for the block and the samples; row-norm adds 2 d per uniform sample
    assert f_u == w.bh * 4.0 * w.n * w.d * (w.block + w.m)
    assert f_r == f_u + w.bh * 2.0 * w.n * w.d * w.m
    b, f = bench.algorithmic(w, "hash")
    assert f == 0 and b == w.bh * 2 * w.n * (w.d * 2 + 3)
    assert bench.nlev_of(w) == 0
    assert bench.nlev_of(wl.WORKLOADS["prefill_causal_bf16_n32768"]) == 3


def test_step_work_model():
    """The whole-step work behind `roofline_step`: the headline step is HBM-bound (0.51 ms of bytes against
    0.33 ms of flops at the measured peaks), and the causal model adds the exact leaves and the level parts."""
    w = wl.WORKLOADS[wl.HEADLINE]
    b, f = bench.step_work(w)
    n, d, bh = w.n, w.d, w.bh
    # hash reads Q, K; attention reads Q, K, V and writes O (2-byte elements); ranks and permutations 32 B per row
    assert b == bh * (6.0 * n * d * 2 + 32.0 * n)
    assert f == bh * 4.0 * n * d * (w.block + w.m)
    assert f == bench.algorithmic(w, "attn")[1]
    c = wl.WORKLOADS["prefill_causal_bf16_n32768"]
    L = bench.nlev_of(c)
    bc, fc = bench.step_work(c)
    assert fc == c.bh * 2.0 * c.n * c.d * (c.base + L * (c.block + c.m))
    assert bc == c.bh * ((6.0 * c.n * c.d + 1.5 * L * c.n * c.d) * 2 + 32.0 * c.n * (L + 1))
    # fp32 inputs double the element bytes
    t = wl.WORKLOADS["tiny_fp32_n1024"]
    bt, _ = bench.step_work(t)
    assert bt == t.bh * (6.0 * t.n * t.d * 4 + 32.0 * t.n)


def test_traffic_entries_name_existing_sources():
    """Every recorded ncu traffic figure names a source file of the library and a 64-hex-digit hash."""
    for key, tr in bench.TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, "approximate_long_context_b200", "csrc", tr["file"])), key
        assert len(tr["sha256"]) == 64 and tr["bytes"] > 0, key
