"""The allocation-free entry point against the regular one.

hyper_attn_forward_noalloc is for callers that cannot call cudaMalloc (plugins inside engines that
reserve all device memory and forbid allocation while enqueueing, latency-critical loops). Its scratch
is a file-scope device array shared by every call, so two calls in a row must each produce the same
output as hyper_attn_forward on their own inputs, with nothing left over from the previous call.
This file is collected last so that a stop-at-first-failure run has already run every other test.
"""
import numpy as np
import pytest

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


@pytest.mark.parametrize("dtype,n,d,heads,block,m,r", [
    ("bf16", 8192, 64, 4, 256, 256, 8),
    ("fp32", 2048, 128, 3, 128, 100, 6),
])
def test_noalloc_matches_forward_twice(dtype, n, d, heads, block, m, r):
    lib = binding.lib()
    ha = binding.HyperAttention(0)
    stream = torch.cuda.current_stream().cuda_stream
    ha.set_options(dtype=dtype, kernel="simt", stream=stream)
    code = binding.DTYPES[dtype]
    for call, seed in enumerate([101, 202]):           # two calls in a row, different inputs and seeds
        Qh, Kh, Vh = wl.make_inputs(n, d, heads, data_seed=seed + 7, dtype=dtype)
        Q, K, V = to_dev(Qh), to_dev(Kh), to_dev(Vh)
        O_ref = torch.empty_like(Q)
        O_new = torch.full_like(Q, float("nan"))
        ha.forward(Q, K, V, O_ref, n=n, d=d, heads=heads, block=block, m=m, r=r, causal=False, seed=seed)
        rc = lib.hyper_attn_forward_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O_new.data_ptr(), n, d, heads,
                                            block, m, r, seed, code, stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        a = O_new.float().cpu().numpy().astype(np.float64)
        b = O_ref.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        for h in range(heads):
            assert rel_err(a[h], b[h]) < TOL[dtype], f"call {call}, head {h}"
    ha.close()


def test_noalloc_rejects_sizes_beyond_limit():
    lib = binding.lib()
    x = torch.zeros((2, 65536, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(x)
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.hyper_attn_forward_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(), o.data_ptr(), 65536, 64, 2, 256,
                                        64, 8, 1, binding.DTYPES["bf16"], stream)
    assert rc == binding.HA_ERR_INVALID_ARG
    rc = lib.hyper_attn_forward_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(), o.data_ptr(), 1024, 64, 1, 256,
                                        1000, 8, 1, binding.DTYPES["bf16"], stream)
    assert rc == binding.HA_ERR_INVALID_ARG
