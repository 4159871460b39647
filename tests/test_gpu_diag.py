"""Hardness diagnostics (alpha, kappa) on the GPU against the oracle.

alpha = n * max_{j >= first_col} ||(D^-1 A) e_j||^2, kappa = max/min over rows of the row sums of A outside the
row's sortLSH block ("HyperAttention: Long-context Attention in Near-Linear Time", research-map summary,
"Approach", "Key results"). The kernels sum in fp32 and the oracle in double: relative tolerance 1e-4.
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
    # name, n, d, bh, block, r, dtype, sinks
    ("bf16_d64", 512, 64, 2, 64, 6, "bf16", False),
    ("bf16_d128_sinks", 1024, 128, 2, 128, 7, "bf16", True),
    ("fp32_d64_ragged", 1000, 64, 1, 100, 5, "fp32", False),
]


@pytest.mark.parametrize("first_col", [0, 32])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_diagnostics_match_oracle(ha, case, first_col):
    _, n, d, bh, block, r, dtype, sinks = case
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xD1A + n, dtype=dtype, sinks=sinks)
    ha.set_options(dtype=dtype, stream=torch.cuda.current_stream().cuda_stream)
    alpha, kappa = ha.diagnostics(dev_tensor(Qh), dev_tensor(Kh), n=n, d=d, heads=bh, block=block, r=r, seed=21,
                                  first_col=first_col)
    for h in range(bh):
        a_ref, k_ref = oracle.diagnostics(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), block=block, r=r, seed=21,
                                          first_col=first_col)
        assert alpha[h] == pytest.approx(a_ref, rel=1e-4)
        assert kappa[h] == pytest.approx(k_ref, rel=1e-4)
    assert ha.status() == 0, ha.last_error()


def test_diagnostics_one_block_and_limits(ha):
    n, d = 256, 64
    Qh, Kh, _ = wl.make_inputs(n, d, 1, data_seed=0xD2B, dtype="bf16")
    ha.set_options(dtype="bf16", stream=torch.cuda.current_stream().cuda_stream)
    Q, K = dev_tensor(Qh), dev_tensor(Kh)
    alpha, kappa = ha.diagnostics(Q, K, n=n, d=d, heads=1, block=n, r=6, seed=2)
    a_ref, _ = oracle.diagnostics(wl.as_f32(Qh[0]), wl.as_f32(Kh[0]), block=n, r=6, seed=2)
    assert alpha[0] == pytest.approx(a_ref, rel=1e-4) and np.isnan(kappa[0])
    with pytest.raises(binding.HAError):
        ha.diagnostics(Q, K, n=n, d=d, heads=1, block=64, r=6, seed=2, first_col=n)
    big = torch.zeros((1, 32768, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.HAError):
        ha.diagnostics(big, big, n=32768, d=64, heads=1, block=256, r=6, seed=2)
