"""The allocation-failure path, injected on the host (no GPU fault).

hyper_attn_test_fail_alloc makes the handle's next allocations fail as if memory had run out. The call that meets
one must return HA_ERR_OOM before it enqueues anything: the caller's output keeps its contents, the device
status stays clean, and the same handle then runs the same call to the oracle's result.
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

N, D, BH, BLOCK, M, R, SEED = 2048, 64, 2, 256, 128, 6, 31
TOL = 2e-3 + 2.0 ** -9   # bf16 inputs and a bf16 output


def inputs():
    Qh, Kh, Vh = wl.make_inputs(N, D, BH, data_seed=5, dtype="bf16")
    return Qh, Kh, Vh


def check_against_oracle(out, Qh, Kh, Vh):
    for h in range(BH):
        ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), block=BLOCK, m=M, r=R,
                             causal=False, seed=SEED, bh=h)["O"]
        e = float(np.linalg.norm(out[h] - ref) / np.linalg.norm(ref))
        assert e < TOL, f"head {h}: {e:.3e}"


def to_dev(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def test_device_forward_workspace_failure():
    Qh, Kh, Vh = inputs()
    Q, K, V = to_dev(Qh), to_dev(Kh), to_dev(Vh)
    O = torch.full_like(Q, 7.0)
    ha = binding.HyperAttention(0)
    ha.set_options(dtype="bf16", stream=torch.cuda.current_stream().cuda_stream)
    ha.test_fail_alloc(1)                        # a fresh handle: the first allocation is its workspace
    with pytest.raises(binding.HAError) as e:
        ha.forward(Q, K, V, O, n=N, d=D, heads=BH, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    assert e.value.code == binding.HA_ERR_OOM and "allocation" in ha.last_error()
    torch.cuda.synchronize()
    assert bool((O == 7.0).all()), "the failed call wrote the output"
    assert ha.status() == 0
    ha.forward(Q, K, V, O, n=N, d=D, heads=BH, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    torch.cuda.synchronize()
    assert ha.status() == 0
    check_against_oracle(O.float().cpu().numpy().astype(np.float64), Qh, Kh, Vh)
    ha.close()


def test_workspace_growth_failure_keeps_handle():
    """A handle that already ran a small problem fails to grow for a larger one, then grows on the next call."""
    Qh, Kh, Vh = inputs()
    Q, K, V = to_dev(Qh), to_dev(Kh), to_dev(Vh)
    O = torch.empty_like(Q)
    ha = binding.HyperAttention(0)
    ha.set_options(dtype="bf16", stream=torch.cuda.current_stream().cuda_stream)
    ha.forward(Q[:1], K[:1], V[:1], O[:1], n=N, d=D, heads=1, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    big = 64   # heads: a workspace about 64 times larger than the first call's
    Qb = Q[:1].expand(big, N, D).contiguous()
    Ob = torch.full_like(Qb, -3.0)
    ha.test_fail_alloc(1)
    with pytest.raises(binding.HAError) as e:
        ha.forward(Qb, Qb, Qb, Ob, n=N, d=D, heads=big, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    assert e.value.code == binding.HA_ERR_OOM
    torch.cuda.synchronize()
    assert bool((Ob == -3.0).all())
    ha.forward(Q, K, V, O, n=N, d=D, heads=BH, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    torch.cuda.synchronize()
    assert ha.status() == 0
    check_against_oracle(O.float().cpu().numpy().astype(np.float64), Qh, Kh, Vh)
    ha.close()


def test_host_forward_buffer_failure():
    Qh, Kh, Vh = inputs()
    O = np.full(Qh.shape, 0x3F80, np.uint16)     # bf16 1.0 everywhere
    ha = binding.HyperAttention(0)
    ha.set_options(dtype="bf16")
    ha.test_fail_alloc(1)                        # the first allocation of forward_host: its device copies
    with pytest.raises(binding.HAError) as e:
        ha.forward_host(Qh, Kh, Vh, O, n=N, d=D, heads=BH, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    assert e.value.code == binding.HA_ERR_OOM
    assert (O == 0x3F80).all()
    ha.forward_host(Qh, Kh, Vh, O, n=N, d=D, heads=BH, block=BLOCK, m=M, r=R, causal=False, seed=SEED)
    check_against_oracle(wl.as_f32(O).astype(np.float64), Qh, Kh, Vh)
    ha.close()


def test_fail_alloc_rejects_negative():
    ha = binding.HyperAttention(0)
    with pytest.raises(binding.HAError) as e:
        ha.test_fail_alloc(-1)
    assert e.value.code == binding.HA_ERR_INVALID_ARG
    ha.test_fail_alloc(0)
    ha.close()
