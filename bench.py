#!/usr/bin/env python
"""Benchmark of the HyperAttention forward pass (one JSON line on rank 0).

Metric: forward throughput in Mqueries*heads/s (batch * heads * n / time) on the n = 131072 single-layer
workload (32 heads, d = 64, block 256, m = 256, r = 8, bf16), with the achieved fraction of the roofline of
the dominant kernel class. A step is one full forward pass (hash, sort, attention with gather and merge)
over the resident inputs. Multi-GPU runs are weak scaling: every rank runs its own full workload (the
problems are independent, no collective on the data path); value = all ranks' queries*heads / max time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from approximate_long_context_b200 import workload as wl  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x 2 flop/FMA x max SM clock
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch of a kernel class from an ncu capture, valid only while the source file it was
# taken from is unchanged (sha256 of the file at capture time).
TRAFFIC = {
    # 4-head captures of the 32-head workloads (the full ones are too large for a multi-pass capture), scaled x8
    # by the rows processed: attention (level kernel of ha_attn_pp.cu) 205.8 MB read + 46.5 MB written per 4-head
    # launch at n = 131072, d = 64, and 111.2 + 15.8 MB at n = 32768, d = 128; hash 134.3 + 6.5 MB.
    ("attn", "long_bf16_n131072", "tc"): {
        "file": "ha_attn_pp.cu",
        "sha256": "136d222295ffc01aedb9edce94d2b595377c094757c4b9293213988f423f0523",
        "bytes": 8 * (205_786_880 + 46_522_880)},
    ("attn", "mid_bf16_n32768", "tc"): {
        "file": "ha_attn_pp.cu",
        "sha256": "136d222295ffc01aedb9edce94d2b595377c094757c4b9293213988f423f0523",
        "bytes": 8 * (111_241_728 + 15_828_736)},
    # row-norm sampling (--sampling rownorm; kernel of ha_attn_tc.cu), 4-head capture scaled x8: 206.0 MB read +
    # 44.6 MB written (taken before that file last changed, so it is not reported)
    ("attn", "long_bf16_n131072", "tc", "rownorm"): {
        "file": "ha_attn_tc.cu",
        "sha256": "6650df5df3dc9d8021e437523ad21193b7fced4b1f61325e8162791b32184d18",
        "bytes": 8 * (206_016_256 + 44_589_056)},
    ("hash", "long_bf16_n131072", "tc"): {
        "file": "ha_hash.cu",
        "sha256": "1a375171594e17545bd7d5900ce2a4c678af7fe092264fc5a71b71c3c81842b5",
        "bytes": 8 * (134_257_152 + 6_460_160)},
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"])}, "measured"
    return FALLBACK_PEAKS, "fallback"


def nlev_of(w: wl.Workload) -> int:
    """Causal levels of a workload (0 for non-causal)."""
    return int(round(np.log2(w.n // w.base))) if (w.causal and w.n > w.base) else 0


def algorithmic(w: wl.Workload, cls: str, sampling: str = "uniform"):
    """Algorithmic work per launch of a kernel class: (bytes, flops)."""
    e = 2 if w.dtype == "bf16" else 4
    bh, n, d = w.bh, w.n, w.d
    levels = 0
    if w.causal and w.n > w.base:
        levels = int(round(np.log2(w.n // w.base)))
    if cls == "hash":
        return bh * 2 * n * (d * e + 3), 0.0                    # read Q, K rows; write rank (2 B) + flag (1 B)
    if cls == "sort":
        rows = bh * 2 * n if not w.causal else bh * n            # rows sorted per level
        return rows * (2 + 2 + 4 + 4), 0.0                       # rank read twice, perm + inverse written
    if cls == "attn":
        N = n if not w.causal else n // 2                        # query rows per level launch
        flops = bh * 4.0 * N * d * (min(w.block, N if not w.causal else n) + w.m)
        if sampling == "rownorm":                                # uniform samples: scores only; draws: both
            flops += bh * 2.0 * N * d * w.m
        byts = bh * N * (3 * d * e + d * (e if not w.causal else 4) + 8)
        return byts, flops
    if cls == "causal_base":
        flops = bh * 2.0 * n * d * w.base
        byts = bh * n * (3 * d * e + d * e) + bh * n * levels * (d * 4 + 4) / 2
        return byts, flops
    if cls == "draws":                                           # V read; norms written, read twice; cdf written
        sets_rows = n if not w.causal else levels * n // 2
        return bh * n * (d * e + 4) + bh * sets_rows * (4 * 2 + 8) + bh * w.m * 8, 0.0
    raise KeyError(cls)


def step_work(w: wl.Workload):
    """The method's algorithmic work of one whole forward pass (all heads): (bytes, flops). Non-causal per head:
    reads of Q and K for the hash, of Q, K and V for the attention, the write of O, and 32 bytes per row of ranks and
    permutations; 4 n d (b + m) flops for the two contractions. Causal per head: the exact leaves (2 n d c flops) plus
    L levels of the non-causal problem on half the rows, each with its part written and read back once."""
    e = 2 if w.dtype == "bf16" else 4
    n, d, bh = w.n, w.d, w.bh
    if not w.causal:
        return bh * (6.0 * n * d * e + 32.0 * n), bh * 4.0 * n * d * (min(w.block, n) + w.m)
    L = nlev_of(w)
    c = min(w.base, n)
    flops = bh * 2.0 * n * d * (c + L * (w.block + w.m))
    byts = bh * ((6.0 * n * d + 1.5 * L * n * d) * e + 32.0 * n * (L + 1))
    return byts, flops


class ClockSampler:
    """Samples SM clock, power and clock-event reasons of one GPU with NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.02):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            import torch
            props = torch.cuda.get_device_properties(torch_device_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            if bus is not None:
                busid = f"{dom:08X}:{bus:02X}:{dev:02X}.0"
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(busid)
            else:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # clocks are reported as unavailable rather than guessed
            self.error = str(exc)
            self.handle = None

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.handle is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable: " + getattr(self, "error", "")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sms = [s for s, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(sms)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_oracle_rate(w: wl.Workload, heads, sampling="uniform"):
    """Oracle time on full heads (all rows): returns (Mqueries*heads/s, seconds, threads)."""
    import oracle
    oracle.build()
    Qh, Kh, Vh = wl.workload_inputs(w, heads=heads)
    t0 = time.perf_counter()
    for i, h in enumerate(heads):
        oracle.forward(wl.as_f32(Qh[i]), wl.as_f32(Kh[i]), wl.as_f32(Vh[i]), block=w.block, m=w.m, r=w.r,
                       causal=w.causal, base=w.base, seed=w.algo_seed, bh=h, sampling=sampling)
    dt = time.perf_counter() - t0
    return len(heads) * w.n / dt / 1e6, dt, oracle.num_threads()


def parity_spot(w: wl.Workload, out_head0, sampling="uniform", nrows: int = 64, seed: int = 11):
    """The oracle on seeded rows of head 0, against the timed run's output of those rows (part of the CPU-baseline
    leg, after the timed region). The output has the input's type, so a bf16 output adds its own rounding (2^-9
    relative) to the parity tolerance (2e-3 for bf16 inputs, 1e-4 for fp32)."""
    import oracle
    oracle.build()
    Qh, Kh, Vh = wl.workload_inputs(w, heads=[0])
    rows = np.sort(np.random.default_rng(seed).choice(w.n, size=min(nrows, w.n), replace=False))
    ref = oracle.forward(wl.as_f32(Qh[0]), wl.as_f32(Kh[0]), wl.as_f32(Vh[0]), block=w.block, m=w.m, r=w.r,
                         causal=w.causal, base=w.base, seed=w.algo_seed, bh=0, rows=rows, sampling=sampling)["O"]
    got = out_head0[rows]
    err = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    tol = 2e-3 + 2.0 ** -9 if w.dtype == "bf16" else 1e-4
    return {"rows": int(len(rows)), "head": 0, "rel_l2": err, "tol": tol, "pass": bool(err < tol),
            "vs": "oracle on the same seeded inputs and draws (timed run's output)"}


def run_reference(args, w: wl.Workload):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    import oracle
    oracle.build()
    head = [0]
    Qh, Kh, Vh = wl.workload_inputs(w, heads=head)
    Qf, Kf, Vf = wl.as_f32(Qh[0]), wl.as_f32(Kh[0]), wl.as_f32(Vh[0])

    def step():
        oracle.forward(Qf, Kf, Vf, block=w.block, m=w.m, r=w.r, causal=w.causal, base=w.base, seed=w.algo_seed, bh=0,
                       sampling=args.sampling)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = w.n / dt / 1e6
    sample = f"1 of {w.bh} heads per step, all {w.n} query rows (hash, sort and attention of that head)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.sampling),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "HyperAttention fwd Mqueries\u00b7heads/s at n=131k; % of BF16 tensor/HBM roofline"
UNIT = "Mqueries\u00b7heads/s"


def approx_error(Qf, Kf, Vf, Of, causal: bool, nrows: int = 256, seed: int = 7):
    """Relative L2 error of the forward output against exact softmax attention, on seeded query rows of one
    head: float64 numpy, straight from the definition softmax(q K^T) V (causal: keys up to the query)."""
    n = Qf.shape[0]
    rows = np.sort(np.random.default_rng(seed).choice(n, size=min(nrows, n), replace=False))
    exact = np.empty((len(rows), Vf.shape[1]))
    for i0 in range(0, len(rows), 32):
        rr = rows[i0:i0 + 32]
        s = Qf[rr] @ Kf.T
        if causal:
            s[np.arange(n)[None, :] > rr[:, None]] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        exact[i0:i0 + 32] = (p @ Vf) / p.sum(axis=1, keepdims=True)
    diff = Of[rows] - exact
    per_row = np.linalg.norm(diff, axis=1) / np.linalg.norm(exact, axis=1)
    return {"rel_l2": float(np.linalg.norm(diff) / np.linalg.norm(exact)), "median_row_rel_l2": float(np.median(per_row)),
            "rows": int(len(rows)), "head": 0, "vs": "exact softmax attention (float64 numpy, sampled rows)"}


def config_of(w: wl.Workload, sampling: str = "uniform"):
    c = {"workload": w.name, "batch": w.batch, "heads": w.heads, "n": w.n, "d": w.d, "block": w.block, "m": w.m,
         "r": w.r, "causal": w.causal, "causal_base": w.base if w.causal else None, "input_dtype": w.dtype,
         "parallelism": "independent (batch, head) problems per GPU; no collective",
         "l2": "inputs larger than L2, no flush" if 3 * w.bh * w.n * w.d * 2 > 2 * L2_BYTES else "L2 flushed"}
    if sampling != "uniform":
        c["sampling"] = sampling
    return c


def run_ours(args, w: wl.Workload):
    import torch
    import torch.distributed as dist
    from approximate_long_context_b200 import binding
    from approximate_long_context_b200.shard import max_over_ranks, weak_shard

    world, rank, local = dist_setup()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    esz = 2 if w.dtype == "bf16" else 4
    # weak scaling: rank i holds problems [i*bh, (i+1)*bh) of a job of world*bh independent problems
    sh = weak_shard(w.bh, world, rank)
    Qh, Kh, Vh = wl.workload_inputs(w, heads=range(sh.offset, sh.offset + sh.count))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        p = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        p.copy_(t)
        return p.view(tdt) if w.dtype == "bf16" else p

    hQ, hK, hV = pinned(Qh), pinned(Kh), pinned(Vh)
    del Qh, Kh, Vh
    hO = torch.empty(hQ.shape, dtype=tdt, pin_memory=True)
    Q, K, V = hQ.to(dev), hK.to(dev), hV.to(dev)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)
    flush = None if 3 * Q.numel() * esz > 2 * L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    ha = binding.HyperAttention(local)
    ha.set_options(dtype=w.dtype, batch=w.batch, causal_base=w.base or 4096, stream=stream.cuda_stream,
                   kernel=args.kernel, bh_offset=sh.offset, sampling=args.sampling)
    kw = dict(n=w.n, d=w.d, heads=w.heads, block=w.block, m=w.m, r=w.r, causal=w.causal, seed=w.algo_seed)

    def step():
        if flush is not None:
            flush.zero_()
        ha.forward(Q, K, V, O, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    launches_per_step = ha.last_launch_count()
    ha.profile_read()          # drop anything recorded during warm-up
    ha.profile(True)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ha.profile(False)
    prof = ha.profile_read()
    assert ha.status() == 0, ha.last_error()
    out_head0 = O[0].float().cpu().numpy().astype(np.float64) if rank == 0 else None   # for the spot check
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)
    units = world * w.bh * w.n
    value = units / (ms_max * 1e-3) / 1e6

    # end to end through the host-buffer entry point: H2D of Q, K, V and D2H of O inside the timed region
    for _ in range(1):
        ha.forward_host(hQ, hK, hV, hO, **kw)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        ha.forward_host(hQ, hK, hV, hO, **kw)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    e2e_value = units / (e2e_ms * 1e-3) / 1e6

    # same-box comparison with exact softmax attention (the tensor-core exact kernel) on the same inputs
    vs_exact = None
    if not args.no_exact and w.dtype == "bf16" and w.n % 128 == 0:
        O2 = torch.empty_like(O)
        ha.set_options(dtype=w.dtype, batch=w.batch, causal_base=w.base or 4096, stream=stream.cuda_stream,
                       kernel=args.kernel, bh_offset=sh.offset)
        ha.exact(Q, K, V, O2, n=w.n, d=w.d, heads=w.heads, causal=w.causal)   # warm-up
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        x0.record(stream)
        for _ in range(2):
            ha.exact(Q, K, V, O2, n=w.n, d=w.d, heads=w.heads, causal=w.causal)
        x1.record(stream)
        torch.cuda.synchronize(dev)
        assert ha.status() == 0, ha.last_error()
        ex_ms = x0.elapsed_time(x1) / 2
        ex_flops = w.bh * 4.0 * w.n * w.n * w.d * (0.5 if w.causal else 1.0)
        vs_exact = {"exact_ms_per_step": ex_ms, "speedup": ex_ms / ms_max,
                    "exact_tflops": ex_flops / (ex_ms * 1e-3) / 1e12, "exact_kernel": "tcgen05",
                    "note": "exact softmax attention on the same inputs and GPU; causal counts half the pairs"}
        del O2

    # optional: hardness diagnostics on the first rows of head 0 (every entry of A is visited, so a slice; the
    # non-causal matrix of the slice, also for causal workloads)
    diag = None
    if args.diagnostics and rank == 0:
        nd = min(w.n, 4096)
        Qs, Ks = Q[:1, :nd].contiguous(), K[:1, :nd].contiguous()
        ha.set_options(dtype=w.dtype, batch=1, causal_base=w.base or 4096, stream=stream.cuda_stream, kernel=args.kernel)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        a0, k0 = ha.diagnostics(Qs, Ks, n=nd, d=w.d, heads=1, block=w.block, r=w.r, seed=w.algo_seed)
        g1.record(stream)
        torch.cuda.synchronize(dev)
        a32, _ = ha.diagnostics(Qs, Ks, n=nd, d=w.d, heads=1, block=w.block, r=w.r, seed=w.algo_seed, first_col=32)
        diag = {"rows": nd, "head": 0, "alpha": float(a0[0]), "alpha_without_first_32": float(a32[0]),
                "kappa": float(k0[0]), "ms": g0.elapsed_time(g1)}

    # optional: the backward pass (gradients of sum(dO * O); recomputes the forward) on the same inputs
    bwd = None
    if args.backward:
        gen = torch.Generator(device=dev).manual_seed(5)
        dO = torch.randn(Q.shape, generator=gen, device=dev, dtype=torch.float32).to(Q.dtype)
        grads = [torch.empty(Q.shape, dtype=torch.float32, device=dev) for _ in range(3)]
        ha.set_options(dtype=w.dtype, batch=w.batch, causal_base=w.base or 4096, stream=stream.cuda_stream,
                       kernel=args.kernel, bh_offset=sh.offset, sampling=args.sampling)
        ha.backward(Q, K, V, dO, *grads, **kw)   # warm-up
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        b0.record(stream)
        for _ in range(args.backward):
            ha.backward(Q, K, V, dO, *grads, **kw)
        b1.record(stream)
        torch.cuda.synchronize(dev)
        assert ha.status() == 0, ha.last_error()
        bms = max_over_ranks(b0.elapsed_time(b1) / args.backward, dev)
        # algorithmic FLOPs of the gradient kernels: per (query, key) term the score, dO.v, and the dQ, dK, dV
        # updates, 2d each; terms per query as in the forward (uniform samples count once with row-norm
        # sampling plus the draws), plus the exact causal leaves (c/2 keys per query on average)
        terms = w.bh * (w.n if not w.causal else (w.n // 2) * nlev_of(w)) * (
            min(w.block, w.n if not w.causal else w.n // 2) + w.m * (2 if args.sampling == "rownorm" else 1))
        if w.causal:
            terms += w.bh * w.n * min(w.base, w.n) / 2
        bflops = 10.0 * w.d * terms
        bwd = {"ms_per_step": bms, "value": units / (bms * 1e-3) / 1e6, "unit": UNIT, "steps": args.backward,
               "kernels": "forward recompute, then SIMT fp32 gradient kernels (dK, dV by atomic adds)",
               "roofline": {"bound": "alu", "achieved": bflops / (bms * 1e-3) / 1e12, "peak": FP32_SIMT_PEAK_TFLOPS,
                            "unit": "TFLOP/s", "frac": bflops / (bms * 1e-3) / 1e12 / FP32_SIMT_PEAK_TFLOPS,
                            "note": "whole backward call (forward recompute included) against the FP32 ALU peak"}}
        del dO, grads

    # roofline of the dominant kernel class; sort and attention launch once per level
    peaks, peak_src = load_peaks()
    family = ha.last_kernel()
    dom = max(prof, key=lambda k: prof[k][0])
    dom_ms = prof[dom][0]
    nlev = int(round(np.log2(w.n // w.base))) if (w.causal and w.n > w.base) else (0 if w.causal else 1)
    groups = nlev if dom in ("sort", "attn") else 1
    avg_ms = dom_ms / (args.steps * groups)
    byts, flops = algorithmic(w, dom, args.sampling)
    if flops > 0 and dom in ("attn", "causal_base"):
        # the binding roof is the one with the larger ideal time: algorithmic bytes at HBM peak or FLOPs at the
        # compute peak (tensor for the tcgen05 kernels, FP32 ALU for the SIMT ones)
        cpeak = peaks["bf16_tflops"] if family == "tc" else FP32_SIMT_PEAK_TFLOPS
        t_compute = flops / (cpeak * 1e12)
        t_memory = byts / (peaks["hbm_gbs"] * 1e9)
        if t_compute >= t_memory:
            bound, peak, unit = ("tensor" if family == "tc" else "alu"), cpeak, "TFLOP/s"
            achieved = flops / (avg_ms * 1e-3) / 1e12
        else:
            bound, peak, unit = "hbm", peaks["hbm_gbs"], "GB/s"
            achieved = byts / (avg_ms * 1e-3) / 1e9
    else:
        bound, peak, unit = "hbm", peaks["hbm_gbs"], "GB/s"
        achieved = byts / (avg_ms * 1e-3) / 1e9
    traffic = None
    tr = TRAFFIC.get((dom, w.name, family) + ((args.sampling,) if args.sampling != "uniform" else ()))
    if tr is not None:
        src = os.path.join(ROOT, "approximate_long_context_b200", "csrc", tr["file"])
        if os.path.exists(src) and hashlib.sha256(open(src, "rb").read()).hexdigest() == tr["sha256"]:
            traffic = tr["bytes"]

    sbytes, sflops = step_work(w)
    cpk = peaks["bf16_tflops"] if family == "tc" else FP32_SIMT_PEAK_TFLOPS
    t_hbm = sbytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    t_cmp = sflops / (cpk * 1e12) * 1e3
    roof_step = {"t_roof_ms": max(t_hbm, t_cmp), "frac": max(t_hbm, t_cmp) / ms_max,
                 "bound": ("hbm" if t_hbm >= t_cmp else ("tensor" if family == "tc" else "alu")),
                 "bytes": sbytes, "flops": sflops, "t_hbm_ms": t_hbm, "t_compute_ms": t_cmp,
                 "peak_source": peak_src + (" burst" if family == "tc" else ""),
                 "note": "whole forward step (all kernels) against the method's algorithmic bytes and flops"}

    err = None
    if rank == 0:
        f64 = lambda t: t.float().numpy().astype(np.float64)
        err = approx_error(f64(hQ[0]), f64(hK[0]), f64(hV[0]), f64(hO[0]), w.causal)

    cpu = None
    spot = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads = list(range(min(args.cpu_heads, w.bh)))
        rate, secs, cores = cpu_oracle_rate(w, heads, args.sampling)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{len(heads)} of {w.bh} heads, all {w.n} query rows ({secs:.1f} s)"}
        spot = parity_spot(w, out_head0, args.sampling)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded Gaussian Q/K/V, planted heavy keys)",
            "config": config_of(w, args.sampling),
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic, "kernel": dom,
                         # against the bf16 peak sustained for seconds under the power cap (context)
                         "frac_sustained": (achieved / peaks["bf16_tflops_sustained"]) if bound == "tensor" else None,
                         "kernel_ms_per_launch": avg_ms, "peak_source": peak_src + (" burst" if bound == "tensor" else ""),
                         "kernel_family": "tcgen05" if family == "tc" else "simt"},
            "roofline_step": roof_step,
            "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items()},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 3 * Q.numel() * esz,
                    "d2h_bytes_per_step": O.numel() * esz},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "parity_spot": spot,
            "approx_error": err,
            "vs_exact": vs_exact,
        }
        if diag is not None:
            line["diagnostics"] = diag
        if bwd is not None:
            line["backward"] = bwd
        print(json.dumps(line), flush=True)
    ha.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=wl.HEADLINE, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--sampling", default="uniform", choices=["uniform", "rownorm"],
                    help="samples of the product with V: the uniform ones, or rows of V by squared norm")
    ap.add_argument("--cpu-heads", type=int, default=32)
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads instead of its own (small profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-exact", action="store_true", help="skip the same-box exact-attention comparison")
    ap.add_argument("--backward", type=int, default=0, metavar="STEPS",
                    help="also time the backward pass over this many steps (after one warm-up)")
    ap.add_argument("--diagnostics", action="store_true",
                    help="also report the hardness diagnostics (alpha, kappa) of the first 4096 rows of head 0")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = wl.WORKLOADS[args.workload]
    if args.heads > 0:
        import dataclasses
        w = dataclasses.replace(w, heads=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
