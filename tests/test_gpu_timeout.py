"""Failure path of the tensor-core kernels: a device-side wait that runs out.

Every wait in the kernels is bounded; when one gives up, the kernel sets an abort flag that every role
polls, the roles stop (loaders finish their own copies, the MMA issuer drains the tensor core, TMEM is
freed), and the status word reports a timeout. The option test_stall_ms makes the first softmax wait target
a barrier that nothing ever completes, so the bound runs out without any fault. The test checks the
reported status and that the same handle then computes correct results.
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

HA_ERR_TIMEOUT = -5


def dev_tensor(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("n,d,bh,block,m,r,causal,base", [
    (2048, 64, 2, 256, 64, 6, False, 0),
    (2048, 128, 1, 256, 64, 6, True, 512),
])
def test_wait_timeout_is_reported_and_the_handle_recovers(n, d, bh, block, m, r, causal, base):
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0x7117, dtype="bf16")
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    kw = dict(n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=11)
    ha = binding.HyperAttention(0)
    try:
        stream = torch.cuda.current_stream().cuda_stream
        ha.set_options(dtype="bf16", out_dtype="fp32", causal_base=base or 4096, kernel="tc", stream=stream,
                       test_stall_ms=20)
        ha.forward(Q, K, V, O, **kw)
        torch.cuda.synchronize()
        assert ha.status() == HA_ERR_TIMEOUT
        assert "gave up" in ha.last_error()
        # the status word is cleared by reading it; the next call on the same handle is correct
        ha.set_options(dtype="bf16", out_dtype="fp32", causal_base=base or 4096, kernel="tc", stream=stream)
        ha.forward(Q, K, V, O, **kw)
        torch.cuda.synchronize()
        assert ha.status() == 0, ha.last_error()
        out = O.cpu().numpy().astype(np.float64)
        for h in range(bh):
            ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), block=block, m=m, r=r,
                                 causal=causal, base=base, seed=11, bh=h)["O"]
            assert np.linalg.norm(out[h] - ref) / np.linalg.norm(ref) < 2e-3
    finally:
        ha.close()


def test_stall_option_range():
    ha = binding.HyperAttention(0)
    try:
        with pytest.raises(binding.HAError):
            ha.set_options(test_stall_ms=1001)
        with pytest.raises(binding.HAError):
            ha.set_options(test_stall_ms=-1)
    finally:
        ha.close()
