"""Exact softmax attention on the tensor-core kernel (hyper_attn_exact) against the oracle's exact attention.

The exact output is the reference the method's speed-ups are quoted against ("HyperAttention: Long-context
Attention in Near-Linear Time", research-map summary, "Key results"). Bar: relative L2 error per head of
2e-3 (bf16 inputs, fp32 accumulation; P is rounded to bf16 before the P.V product).
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TOL = 2e-3


def dev_tensor(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.fixture(scope="module")
def ha():
    h = binding.HyperAttention(0)
    yield h
    h.close()


def run_exact(ha, Qh, Kh, Vh, *, n, d, bh, causal):
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    ha.set_options(dtype="bf16", out_dtype="fp32", stream=torch.cuda.current_stream().cuda_stream)
    ha.exact(Q, K, V, O, n=n, d=d, heads=bh, causal=causal)
    torch.cuda.synchronize()
    assert ha.status() == 0, ha.last_error()
    return O.cpu().numpy().astype(np.float64)


CASES = [
    # name, n, d, bh, causal
    ("dense_d64", 1024, 64, 2, False),
    ("dense_d128", 2048, 128, 2, False),
    ("dense_odd_tiles", 384, 64, 1, False),
    ("causal_d64", 1024, 64, 2, True),
    ("causal_odd_tiles_d128", 640, 128, 2, True),
    ("single_tile", 128, 64, 3, True),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_exact_matches_oracle(ha, case):
    _, n, d, bh, causal = case
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xE1 + n + d, dtype="bf16", sinks=causal)
    out = run_exact(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, causal=causal)
    for h in range(bh):
        ref = oracle.exact_attention(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), causal=causal)
        err = np.linalg.norm(out[h] - ref) / np.linalg.norm(ref)
        assert err < TOL, f"head {h}: relative L2 error {err:.3g}"


def test_exact_equals_method_with_one_block(ha):
    """The method with one block (b' = n) is exact attention, whatever its samples: the two entry points agree
    within the bf16 bar."""
    n, d, bh = 512, 64, 2
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xE7, dtype="bf16")
    ex = run_exact(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, causal=False)
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    ha.set_options(dtype="bf16", out_dtype="fp32", stream=torch.cuda.current_stream().cuda_stream)
    ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=n, m=64, r=6, causal=False, seed=3)
    torch.cuda.synchronize()
    meth = O.cpu().numpy().astype(np.float64)
    for h in range(bh):
        assert np.linalg.norm(meth[h] - ex[h]) / np.linalg.norm(ex[h]) < TOL


def test_exact_full_size_sampled_rows(ha):
    """n = 131072, d = 64 (the long workload's shape, 2 heads): sampled rows against the oracle."""
    n, d, bh = 131072, 64, 2
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xE9, dtype="bf16")
    out = run_exact(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, causal=False)
    rows = np.sort(np.random.default_rng(5).choice(n, 48, replace=False))
    for h in range(bh):
        ref = oracle.exact_attention(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), causal=False, rows=rows)
        err = np.linalg.norm(out[h][rows] - ref) / np.linalg.norm(ref)
        assert err < TOL, f"head {h}: relative L2 error {err:.3g}"


def test_exact_rejects_unsupported_shapes(ha):
    x = torch.zeros((1, 200, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(x)
    ha.set_options(dtype="bf16", stream=torch.cuda.current_stream().cuda_stream)
    with pytest.raises(binding.HAError) as e:
        ha.exact(x, x, x, o, n=200, d=64, heads=1, causal=False)     # n not a multiple of 128
    assert e.value.code == -2
    y = torch.zeros((1, 256, 64), dtype=torch.float32, device="cuda")
    ha.set_options(dtype="fp32", stream=torch.cuda.current_stream().cuda_stream)
    with pytest.raises(binding.HAError) as e:
        ha.exact(y, y, y, torch.zeros_like(y), n=256, d=64, heads=1, causal=False)   # fp32 inputs
    assert e.value.code == -2
