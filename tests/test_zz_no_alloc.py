"""The allocation-free entry point against the oracle and against the regular entry point.

hyper_attn_forward_noalloc is for callers that cannot call cudaMalloc (plugins inside engines that
reserve all device memory and forbid allocation while enqueueing, latency-critical loops). Its scratch
is a file-scope device array shared by every call, so two calls in a row must each give the oracle's
output on their own inputs (and the regular entry point's), with nothing left over from the previous call.
This file is collected last so that a stop-at-first-failure run has already run every other test.
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TOL = {"fp32": 1e-4, "bf16": 2e-3}


def to_dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def rel_err(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def call(lib, Q, K, V, O, n, d, heads, block, m, r, seed, dtype, stream):
    return lib.hyper_attn_forward_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), n, d, heads,
                                          block, m, r, seed, binding.DTYPES[dtype], stream)


@pytest.mark.parametrize("dtype,n,d,heads,block,m,r", [
    ("bf16", 8192, 64, 4, 256, 256, 8),
    ("fp32", 2048, 128, 3, 128, 100, 6),
])
def test_noalloc_matches_oracle_and_forward_twice(dtype, n, d, heads, block, m, r):
    lib = binding.lib()
    ha = binding.HyperAttention(0)
    stream = torch.cuda.current_stream().cuda_stream
    ha.set_options(dtype=dtype, kernel="simt", stream=stream)
    for c, seed in enumerate([101, 202]):           # two calls in a row, different inputs and seeds
        Qh, Kh, Vh = wl.make_inputs(n, d, heads, data_seed=seed + 7, dtype=dtype)
        Q, K, V = to_dev(Qh), to_dev(Kh), to_dev(Vh)
        O_ref = torch.empty_like(Q)
        O_new = torch.full_like(Q, float("nan"))
        ha.forward(Q, K, V, O_ref, n=n, d=d, heads=heads, block=block, m=m, r=r, causal=False, seed=seed)
        rc = call(lib, Q, K, V, O_new, n, d, heads, block, m, r, seed, dtype, stream)
        assert rc == 0, f"call {c}: status {rc}"
        torch.cuda.synchronize()
        a = O_new.float().cpu().numpy().astype(np.float64)
        b = O_ref.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        for h in range(heads):
            ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), block=block, m=m, r=r,
                                 causal=False, seed=seed, bh=h)["O"]
            # the output has the input's type: a bf16 output adds its own rounding (2^-9 relative)
            tol = TOL[dtype] + (2.0 ** -9 if dtype == "bf16" else 0.0)
            assert rel_err(a[h], ref) < tol, f"call {c}, head {h}: against the oracle"
            assert rel_err(a[h], b[h]) < TOL[dtype], f"call {c}, head {h}: against hyper_attn_forward"
    ha.close()


def test_noalloc_rejects_sizes_beyond_limit():
    """Every limit is checked on the host before anything is enqueued."""
    lib = binding.lib()
    stream = torch.cuda.current_stream().cuda_stream
    x = torch.zeros((2, 65536, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(x)
    small = torch.zeros((1, 1024, 64), dtype=torch.bfloat16, device="cuda")
    so = torch.zeros_like(small)
    bad = {
        "rows": (x, o, 65536, 64, 2, 256, 64, 8),
        "m": (small, so, 1024, 64, 1, 256, 1000, 8),
        "r": (small, so, 1024, 64, 1, 256, 64, 11),
        "n % block": (small, so, 1000, 64, 1, 256, 64, 8),
    }
    for what, (t, out, n, d, heads, block, m, r) in bad.items():
        assert call(lib, t, t, t, out, n, d, heads, block, m, r, 1, "bf16", stream) == binding.HA_ERR_INVALID_ARG, what
    many = torch.zeros((65, 512, 64), dtype=torch.bfloat16, device="cuda")
    assert call(lib, many, many, many, torch.zeros_like(many), 512, 64, 65, 256, 64, 8, 1, "bf16",
                stream) == binding.HA_ERR_INVALID_ARG, "heads"
    # a pointer 2 bytes past a 16-byte boundary
    flat = torch.zeros(1024 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    off = flat[1:1 + 1024 * 64]
    assert call(lib, off, small, small, so, 1024, 64, 1, 256, 64, 8, 1, "bf16", stream) == binding.HA_ERR_INVALID_ARG
    assert call(lib, small, small, small, off, 1024, 64, 1, 256, 64, 8, 1, "bf16",
                stream) == binding.HA_ERR_INVALID_ARG
    assert call(lib, small, small, small, so, 1024, 96, 1, 256, 64, 8, 1, "bf16", stream) == binding.HA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert so.abs().sum().item() == 0, "a rejected call wrote its output"


def test_noalloc_refuses_stream_capture():
    """Its draws come from pageable host arrays that the next call overwrites: a call on a capturing stream
    is refused and enqueues nothing."""
    lib = binding.lib()
    q = torch.zeros((1, 1024, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            rc = call(lib, q, q, q, o, 1024, 64, 1, 256, 64, 8, 1, "bf16", side.cuda_stream)
            o.add_(0)
    assert rc == binding.HA_ERR_UNSUPPORTED
    del g
    torch.cuda.synchronize()
