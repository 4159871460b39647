"""Seeded synthetic inputs for the HyperAttention forward pass.

This module only makes data: it holds none of the method's arithmetic, and both the CUDA path's tests
and benchmark and the CPU oracle read the arrays it returns.

The workloads follow the shapes of the pages' experiments ("HyperAttention: Long-context Attention in
Near-Linear Time", research-map summary, "Key results": a single attention layer at n = 131k, causal and
non-causal; ChatGLM2-6B-32k at 32k context). The pages' real inputs (LongBench prompts, ImageNet, model
activations) are not available, so Gaussian stand-ins with the structure those pages describe are used:

* Q, K, V ~ N(0, 1) in fp32; Q and K multiplied by d^-1/4, so q.k carries the usual 1/sqrt(d) softmax scale;
* planted heavy entries: a fraction of the key rows of each head (distinct rows, chosen uniformly) is
  replaced by a uniformly chosen query row plus N(0, 0.1^2) noise, added after the scaling;
* sink-like columns (the summary's "Surprising findings": the first columns of the normalised attention in
  ChatGLM2 hold heavy entries): optionally the first 32 key rows are multiplied by 4 after planting;
* bf16 workloads round the fp32 values once, to nearest even, on the host.

Every head is generated independently from numpy's Philox bit generator keyed by (data seed, head index),
so one head can be regenerated on its own.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    n: int
    d: int
    block: int
    m: int
    r: int
    causal: bool
    base: int            # exact-causal leaf size (causal only)
    dtype: str           # "fp32" or "bf16"
    planted: float       # fraction of key rows replaced by noisy query copies
    sinks: bool          # first 32 key rows scaled by 4
    data_seed: int
    algo_seed: int

    @property
    def bh(self) -> int:
        return self.batch * self.heads


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32_n1024", 1, 1, 1024, 64, 64, 64, 6, False, 0, "fp32", 0.05, False,
                 0xC0FFEE00, 1234),
        Workload("mid_bf16_n32768", 1, 32, 32768, 128, 256, 256, 7, False, 0, "bf16", 0.05, False,
                 0xC0FFEE01, 1235),
        Workload("prefill_causal_bf16_n32768", 1, 32, 32768, 128, 256, 256, 7, True, 4096, "bf16", 0.05, True,
                 0xC0FFEE02, 1236),
        Workload("long_bf16_n131072", 1, 32, 131072, 64, 256, 256, 8, False, 0, "bf16", 0.05, False,
                 0xC0FFEE03, 1237),
        Workload("very_long_causal_bf16_n524288", 1, 8, 524288, 128, 512, 512, 9, True, 8192, "bf16", 0.02, True,
                 0xC0FFEE04, 1238),
    ]
}

HEADLINE = "long_bf16_n131072"


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the exactly equal fp32 values."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_head(n: int, d: int, data_seed: int, head: int, planted: float, sinks: bool):
    """Q, K, V (n, d) float32 for one (batch*head) index."""
    rng = np.random.Generator(np.random.Philox(key=[data_seed, head]))
    scale = np.float32(d ** -0.25)
    Q = rng.standard_normal((n, d), dtype=np.float32) * scale
    K = rng.standard_normal((n, d), dtype=np.float32) * scale
    V = rng.standard_normal((n, d), dtype=np.float32)
    count = int(round(planted * n))
    if count > 0:
        rows = rng.choice(n, size=count, replace=False)
        src = rng.integers(0, n, size=count)
        K[rows] = Q[src] + np.float32(0.1) * rng.standard_normal((count, d), dtype=np.float32)
    if sinks:
        K[: min(32, n)] *= np.float32(4.0)
    return Q, K, V


def make_inputs(n: int, d: int, bh: int, *, data_seed: int, planted: float = 0.05, sinks: bool = False,
                dtype: str = "bf16", heads=None):
    """Q, K, V as (len(heads), n, d) arrays: float32 for dtype "fp32", bf16 bit patterns (uint16) for "bf16".
    heads: the (batch*head) indices to generate (default: all bh)."""
    heads = list(range(bh)) if heads is None else list(heads)
    out_dt = np.float32 if dtype == "fp32" else np.uint16
    Q = np.empty((len(heads), n, d), out_dt)
    K = np.empty_like(Q)
    V = np.empty_like(Q)
    for i, h in enumerate(heads):
        q, k, v = make_head(n, d, data_seed, h, planted, sinks)
        if dtype == "fp32":
            Q[i], K[i], V[i] = q, k, v
        else:
            Q[i], K[i], V[i] = round_to_bf16_bits(q), round_to_bf16_bits(k), round_to_bf16_bits(v)
    return Q, K, V


def as_f32(x: np.ndarray) -> np.ndarray:
    """The exact float32 values of an input array (identity for float32, bit widening for bf16)."""
    return x if x.dtype == np.float32 else bf16_bits_to_f32(x)


def workload_inputs(w: Workload, heads=None):
    return make_inputs(w.n, w.d, w.bh, data_seed=w.data_seed, planted=w.planted, sinks=w.sinks,
                       dtype=w.dtype, heads=heads)
