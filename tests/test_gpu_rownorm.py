"""Row-norm sampling of the product with V on the GPU against the oracle.

"HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach"): the sampled
part of the product with V takes m draws with replacement, row j of V with probability proportional to its
squared norm and weight 1/(m p_j); the normaliser keeps the uniform samples. The draws are integer decisions
taken from the same fp32 norms and double cumulative sums on both sides, so they are compared one by one: a
draw may differ only where u * total lies within rounding distance of a cumulative sum (the device adds the
sums in a tree order, the oracle left to right), and the test checks that for any draw that differs. The
outputs are compared at the floating-point bars of the uniform path: relative L2 error per head 1e-4 (fp32
inputs) and 2e-3 (bf16 inputs). bf16 inputs with m <= 256 run on the tensor-core kernel (its row-norm
instance), the rest and the forced-SIMT cases on the SIMT kernel.
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TOL = {"fp32": 1e-4, "bf16": 2e-3}


def dev_tensor(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


@pytest.fixture(scope="module")
def ha():
    h = binding.HyperAttention(0)
    yield h
    h.close()


def sets_of(n, causal, base):
    """(heap node, first key row, key rows) of every sample set of one problem, in heap order."""
    if not causal:
        return [(1, 0, n)]
    out = []
    L, x = 0, n
    while x > base:
        x //= 2
        L += 1
    for depth in range(L):
        node_len = n >> depth
        for idx in range(1 << depth):
            out.append(((1 << depth) + idx, idx * node_len, node_len // 2))
    return out


def _u(seed, bh, node, m):
    start = [2**64 - 1, node - 1, bh, 0]
    g = np.random.Philox(key=np.array([seed, 3], np.uint64), counter=np.array(start, np.uint64))
    w = g.random_raw(4 * ((m + 3) // 4)).astype(np.uint64)[:m]
    return (w >> np.uint64(11)).astype(np.float64) * 2.0**-53


def check_draws(got_S, got_lw, Vset, seed, bh, node, m):
    ref_S, ref_lw = oracle.draw_rownorm(seed, bh, node, Vset, m)
    diff = np.nonzero(got_S != ref_S)[0]
    if len(diff):
        # a differing draw must sit on a boundary of the cumulative distribution, up to rounding
        nrm = (Vset.astype(np.float64) ** 2).sum(axis=1)
        F = np.cumsum(nrm)
        u = _u(seed, bh, node, m)
        for t in diff:
            lo = min(got_S[t], ref_S[t])
            assert abs(F[lo] - u[t] * F[-1]) <= 1e-9 * F[-1], f"draw {t}: {got_S[t]} vs {ref_S[t]}"
        assert len(diff) <= 2
    same = got_S == ref_S
    np.testing.assert_allclose(got_lw[same], ref_lw[same], rtol=2e-7, atol=0)


def run(ha, Qh, Kh, Vh, *, dtype, n, d, bh, block, m, r, causal, base, seed, out_dtype="fp32", kernel="auto"):
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    ha.set_options(dtype=dtype, out_dtype=out_dtype, causal_base=base or 4096, kernel=kernel,
                   stream=torch.cuda.current_stream().cuda_stream, sampling="rownorm")
    ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=seed)
    torch.cuda.synchronize()
    assert ha.status() == 0, ha.last_error()
    want = "simt" if (kernel == "simt" or dtype == "fp32" or m > 256 or block % 128) else "tc"
    assert ha.last_kernel() == want
    return O.cpu().numpy().astype(np.float64)


CASES = [
    # name, n, d, bh, block, m, r, causal, base, dtype
    ("fp32_d64", 1024, 64, 2, 128, 64, 6, False, 0, "fp32"),
    ("fp32_d128_ragged", 1000, 128, 1, 100, 37, 5, False, 0, "fp32"),
    ("bf16_d64_chunks", 8192, 64, 2, 256, 128, 7, False, 0, "bf16"),
    ("bf16_d128", 2048, 128, 2, 128, 64, 6, False, 0, "bf16"),
    ("fp32_causal_small_sets", 2048, 64, 2, 64, 32, 5, True, 256, "fp32"),
    ("bf16_causal_chunks", 16384, 64, 1, 256, 96, 6, True, 2048, "bf16"),
    ("bf16_causal_d128", 4096, 128, 1, 128, 64, 6, True, 512, "bf16"),
]


RUNS = [(c, "auto") for c in CASES] + [(c, "simt") for c in CASES if c[0] in ("bf16_d64_chunks", "bf16_causal_d128")]


@pytest.mark.parametrize("case,kernel", RUNS, ids=[f"{c[0]}-{k}" for c, k in RUNS])
def test_rownorm_matches_oracle(ha, case, kernel):
    _, n, d, bh, block, m, r, causal, base, dtype = case
    seed = 0x5EED + n
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xA0 + n + d, dtype=dtype, sinks=causal)
    # rows of very different norms, and a run of zero rows that must never be drawn
    Vf = wl.as_f32(Vh)
    scale = np.exp(np.random.default_rng(n).uniform(-2.0, 2.0, (bh, n, 1))).astype(np.float32)
    Vf = Vf * scale
    Vf[:, 5:40] = 0.0
    Vh = wl.round_to_bf16_bits(Vf) if dtype == "bf16" else Vf.astype(np.float32)
    out = run(ha, Qh, Kh, Vh, dtype=dtype, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=causal, base=base,
              seed=seed, kernel=kernel)
    sets = sets_of(n, causal, base)
    got_S = ha.debug_copy("rn_s", 0, np.int32, bh * len(sets) * m).reshape(bh, len(sets), m)
    got_lw = ha.debug_copy("rn_logw", 0, np.float32, bh * len(sets) * m).reshape(bh, len(sets), m)
    for h in range(bh):
        Vf32 = wl.as_f32(Vh[h])
        for k, (node, start, length) in enumerate(sets):
            check_draws(got_S[h, k], got_lw[h, k], Vf32[start:start + length], seed, h, node, m)
            assert not np.isin(got_S[h, k] + start, np.arange(5, 40)).any()
        ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), Vf32, block=block, m=m, r=r,
                             causal=causal, base=base, seed=seed, bh=h, sampling="rownorm")["O"]
        err = np.linalg.norm(out[h] - ref) / np.linalg.norm(ref)
        assert err < TOL[dtype], f"head {h}: relative L2 error {err:.3g}"


def test_rownorm_all_zero_values(ha):
    n, d, bh, m = 512, 64, 2, 16
    Qh, Kh, _ = wl.make_inputs(n, d, bh, data_seed=0xA7, dtype="fp32")
    out = run(ha, Qh, Kh, np.zeros((bh, n, d), np.float32), dtype="fp32", n=n, d=d, bh=bh, block=64, m=m, r=5,
              causal=False, base=0, seed=3)
    assert np.all(out == 0.0)
    S = ha.debug_copy("rn_s", 0, np.int32, bh * m)
    assert np.all(S == -1)


def test_rownorm_differs_from_uniform_and_tc_limits(ha):
    n, d, bh = 1024, 64, 1
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xA8, dtype="bf16")
    kw = dict(dtype="bf16", n=n, d=d, bh=bh, block=128, m=64, r=6, causal=False, base=0, seed=4)
    rn = run(ha, Qh, Kh, Vh, **kw)
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    ha.set_options(dtype="bf16", out_dtype="fp32", stream=torch.cuda.current_stream().cuda_stream)
    ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=128, m=64, r=6, causal=False, seed=4)
    torch.cuda.synchronize()
    assert not np.array_equal(O.cpu().numpy().astype(np.float64), rn)
    # the tensor-core kernel takes m <= 256 with row-norm sampling; auto falls back to SIMT beyond it
    ha.set_options(dtype="bf16", out_dtype="fp32", kernel="tc", stream=torch.cuda.current_stream().cuda_stream,
                   sampling="rownorm")
    with pytest.raises(binding.HAError) as e:
        ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=128, m=300, r=6, causal=False, seed=4)
    assert e.value.code == -2
    big = run(ha, Qh, Kh, Vh, **dict(kw, m=300))
    ref = oracle.forward(wl.as_f32(Qh[0]), wl.as_f32(Kh[0]), wl.as_f32(Vh[0]), block=128, m=300, r=6, causal=False,
                         seed=4, bh=0, sampling="rownorm")["O"]
    assert np.linalg.norm(big[0] - ref) / np.linalg.norm(ref) < TOL["bf16"]


def test_rownorm_host_pipeline_equals_device_call(ha):
    """forward_host splits the problems into groups keyed by their global index: the same draws, the same
    output bits as one device call."""
    n, d, bh, m = 4096, 64, 4, 64
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xA9, dtype="bf16")
    dev = run(ha, Qh, Kh, Vh, dtype="bf16", n=n, d=d, bh=bh, block=256, m=m, r=6, causal=False, base=0, seed=8)
    ha.set_options(dtype="bf16", out_dtype="fp32", stream=torch.cuda.current_stream().cuda_stream,
                   sampling="rownorm")
    O = np.zeros((bh, n, d), np.float32)
    ha.forward_host(Qh, Kh, Vh, O, n=n, d=d, heads=bh, block=256, m=m, r=6, causal=False, seed=8)
    assert np.array_equal(O.astype(np.float64), dev)


def test_rownorm_full_size_sampled_rows(ha):
    """n = 131072, d = 64, 2 heads (the long workload's shape): every draw and sampled output rows."""
    n, d, bh, block, m, r = 131072, 64, 2, 256, 256, 8
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=0xAA, dtype="bf16")
    out = run(ha, Qh, Kh, Vh, dtype="bf16", n=n, d=d, bh=bh, block=block, m=m, r=r, causal=False, base=0, seed=12)
    got_S = ha.debug_copy("rn_s", 0, np.int32, bh * m).reshape(bh, m)
    got_lw = ha.debug_copy("rn_logw", 0, np.float32, bh * m).reshape(bh, m)
    rows = np.sort(np.random.default_rng(6).choice(n, 32, replace=False))
    for h in range(bh):
        Vf = wl.as_f32(Vh[h])
        check_draws(got_S[h], got_lw[h], Vf, 12, h, 1, m)
        ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), Vf, block=block, m=m, r=r, causal=False, seed=12,
                             bh=h, rows=rows, sampling="rownorm")["O"]
        err = np.linalg.norm(out[h][rows] - ref) / np.linalg.norm(ref)
        assert err < TOL["bf16"], f"head {h}: relative L2 error {err:.3g}"
