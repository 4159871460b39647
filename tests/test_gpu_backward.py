"""Backward pass on the GPU (hyper_attn_backward) against the oracle's gradients.

The gradients of sum(dO * O) with the sort and the draws held fixed ("HyperAttention: Long-context Attention in
Near-Linear Time", research-map summary, "Key results": the speed-ups are for the forward and backward
passes). The oracle differentiates its dense per-problem weights in double precision. Bars, as relative L2
errors per head and per gradient: 1e-4 when the forward runs on the SIMT fp32 kernels; 5e-3 when it runs on
the tensor cores, whose P is rounded to bf16 (the forward's own bar is 2e-3) and whose O and log normaliser
enter every gradient through dO . O and e^{s - L}.
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def dev_tensor(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


@pytest.fixture(scope="module")
def ha():
    h = binding.HyperAttention(0)
    yield h
    h.close()


CASES = [
    # name, n, d, bh, block, m, r, causal, base, dtype, kernel, sampling
    ("fp32_d64", 512, 64, 2, 64, 32, 5, False, 0, "fp32", "auto", "uniform"),
    ("fp32_d128_ragged", 1000, 128, 1, 100, 37, 5, False, 0, "fp32", "auto", "uniform"),
    ("bf16_d64_simt", 1024, 64, 2, 128, 64, 6, False, 0, "bf16", "simt", "uniform"),
    ("bf16_d64_tc", 1024, 64, 2, 128, 64, 6, False, 0, "bf16", "auto", "uniform"),
    ("fp32_causal", 1024, 64, 1, 64, 32, 5, True, 256, "fp32", "auto", "uniform"),
    ("bf16_causal_d128_tc", 1024, 128, 2, 128, 64, 6, True, 256, "bf16", "auto", "uniform"),
    ("fp32_rownorm", 512, 64, 2, 64, 32, 5, False, 0, "fp32", "auto", "rownorm"),
    ("bf16_causal_rownorm_tc", 1024, 64, 1, 128, 64, 6, True, 256, "bf16", "auto", "rownorm"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(ha, case):
    _, n, d, bh, block, m, r, causal, base, dtype, kernel, sampling = case
    seed = 0xBAC + n
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xB0 + n + d, dtype=dtype, sinks=causal)
    dOf = np.random.default_rng(n + d).standard_normal((bh, n, d)).astype(np.float32)
    dOh = wl.round_to_bf16_bits(dOf) if dtype == "bf16" else dOf
    grads = [torch.empty((bh, n, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    ha.set_options(dtype=dtype, causal_base=base or 4096, kernel=kernel, sampling=sampling,
                   stream=torch.cuda.current_stream().cuda_stream)
    ha.backward(dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh), dev_tensor(dOh), *grads, n=n, d=d, heads=bh,
                block=block, m=m, r=r, causal=causal, seed=seed)
    torch.cuda.synchronize()
    assert ha.status() == 0, ha.last_error()
    tc = dtype == "bf16" and kernel != "simt"
    tol = 5e-3 if tc else 1e-4
    got = [t.cpu().numpy().astype(np.float64) for t in grads]
    for h in range(bh):
        ref = oracle.backward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), wl.as_f32(dOh[h]), block=block,
                              m=m, r=r, causal=causal, base=base, seed=seed, bh=h, sampling=sampling)
        for name, g in zip(("dQ", "dK", "dV"), got):
            err = np.linalg.norm(g[h] - ref[name]) / np.linalg.norm(ref[name])
            assert err < tol, f"head {h} {name}: relative L2 error {err:.3g}"


def test_backward_rejects_aliasing_and_bad_shapes(ha):
    n, d = 256, 64
    x = torch.zeros((1, n, d), dtype=torch.float32, device="cuda")
    gq, gk, gv = (torch.zeros_like(x) for _ in range(3))
    ha.set_options(dtype="fp32", stream=torch.cuda.current_stream().cuda_stream)
    with pytest.raises(binding.HAError) as e:
        ha.backward(x, x, x, x, gq, gq, gv, n=n, d=d, heads=1, block=64, m=16, r=4, causal=False, seed=1)
    assert e.value.code == -1
    with pytest.raises(binding.HAError) as e:
        ha.backward(x, x, x, x, gq, gk, gv, n=n, d=d, heads=1, block=48, m=16, r=4, causal=False, seed=1)
    assert e.value.code == -1
