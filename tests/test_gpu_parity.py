"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Bars: sortLSH ranks, near-zero flags, sorted permutations and their inverses bit-exact; outputs within a
relative L2 error per head of 1e-4 (fp32 inputs) and 2e-3 (bf16 inputs, compared on fp32 outputs; the
bf16-rounded output is checked against the same bar plus the bf16 rounding of the output itself).
"""
import numpy as np
import pytest

import oracle
from approximate_long_context_b200 import binding
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TOL = {"fp32": 1e-4, "bf16": 2e-3}
# log of the estimated normaliser: fp32 paths sum fp32 terms; the tensor-core path sums the bf16-rounded
# probabilities it feeds to the P.V product, so |dL| <= 2^-8 (bf16 unit roundoff) plus fp32 rounding
LSE_TOL = {"fp32": 1e-4, "bf16": 2.0 ** -8 + 2.0 ** -12}


def dev_tensor(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


@pytest.fixture(scope="module")
def ha():
    assert torch.cuda.is_available()
    h = binding.HyperAttention(0)
    yield h
    h.close()


def run_gpu(ha, Qh, Kh, Vh, *, n, d, bh, block, m, r, causal, seed, base=4096, dtype="bf16", out_dtype="fp32",
            kernel="auto", debug=True):
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32 if out_dtype == "fp32" else torch.bfloat16, device="cuda")
    ha.set_options(dtype=dtype, out_dtype=out_dtype, batch=1, causal_base=base or 4096, kernel=kernel,
                   stream=torch.cuda.current_stream().cuda_stream, debug_captures=debug)
    ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=seed)
    torch.cuda.synchronize()
    assert ha.status() == 0, ha.last_error()
    return O.float().cpu().numpy().astype(np.float64)


def tc_shape(n, block, causal, base):
    """Shapes the tensor-core kernels take: every level's b' = min(b, N) and the causal leaf are multiples
    of 128."""
    if not causal:
        return min(block, n) % 128 == 0
    levels = binding.levels(n, True, base)[0]
    return min(base, n) % 128 == 0 and all(min(block, n >> l) % 128 == 0 for l in range(1, levels + 1))


def rel_err(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def check_ranks_and_perms(ha, Qf, Kf, *, n, bh, r, causal, base, seed, heads=None):
    levels = binding.levels(n, causal, base)[0] if causal else 0
    rank = ha.debug_copy("rank", 0, np.uint16, bh * 2 * n).reshape(bh, 2, n)
    near = ha.debug_copy("near", 0, np.uint8, bh * 2 * n).reshape(bh, 2, n)
    P = oracle.draw_projection(seed, Qf.shape[-1], r)
    for h in (range(bh) if heads is None else heads):
        rq, nq = oracle.hash_rows(Qf[h], P)
        rk, nk = oracle.hash_rows(Kf[h], P)
        assert np.array_equal(rank[h, 0], rq) and np.array_equal(rank[h, 1], rk), f"ranks differ (head {h})"
        assert np.array_equal(near[h, 0], nq) and np.array_equal(near[h, 1], nk), f"near flags differ (head {h})"
    lvls = [0] if not causal else list(range(1, levels + 1))
    for lvl in lvls:
        N = n if lvl == 0 else n >> lvl
        nodes = 1 if lvl == 0 else 1 << (lvl - 1)
        perm = ha.debug_copy("perm", lvl, np.int32, bh * nodes * 2 * N).reshape(bh, nodes, 2, N)
        inv = ha.debug_copy("inv", lvl, np.int32, bh * nodes * 2 * N).reshape(bh, nodes, 2, N)
        for h in (range(bh) if heads is None else heads):
            ranks = np.concatenate([rank[h, 0], rank[h, 1]])
            pq, pk = oracle.level_perms(ranks, n, lvl)
            assert np.array_equal(perm[h, :, 0].reshape(-1), pq), f"Q permutation differs (level {lvl}, head {h})"
            assert np.array_equal(perm[h, :, 1].reshape(-1), pk), f"K permutation differs (level {lvl}, head {h})"
            for j in range(nodes):
                for w in range(2):
                    assert np.array_equal(inv[h, j, w][perm[h, j, w]], np.arange(N)), "inverse permutation"


CASES = [
    # name, n, d, bh, block, m, r, causal, base, dtype
    ("tiny_fp32", 1024, 64, 1, 64, 64, 6, False, 0, "fp32"),
    ("fp32_d128", 2048, 128, 2, 128, 100, 5, False, 0, "fp32"),
    ("bf16_d64", 4096, 64, 3, 256, 256, 8, False, 0, "bf16"),
    ("bf16_d128", 4096, 128, 2, 256, 256, 7, False, 0, "bf16"),
    ("ragged_rows", 1000, 64, 3, 8, 40, 5, False, 0, "bf16"),
    ("single_block", 512, 64, 2, 512, 64, 6, False, 0, "bf16"),
    ("block_gt_n", 384, 128, 1, 1024, 32, 4, False, 0, "bf16"),
    ("no_samples", 2048, 64, 2, 128, 0, 7, False, 0, "bf16"),
    ("one_bucket", 2048, 64, 2, 128, 64, 0, False, 0, "bf16"),
    ("all_sampled", 1024, 64, 1, 64, 1024, 6, False, 0, "bf16"),
    ("r16_two_pass", 4096, 64, 2, 256, 128, 16, False, 0, "bf16"),
    ("r12_two_pass", 2048, 128, 1, 128, 64, 12, False, 0, "fp32"),
    ("r10_one_pass", 4096, 64, 2, 256, 64, 10, False, 0, "bf16"),    # 1024-way digit: large scatter stage
    ("r9_one_pass", 2048, 128, 2, 128, 64, 9, False, 0, "bf16"),
    ("causal_small", 4096, 64, 2, 128, 64, 6, True, 512, "bf16"),
    ("causal_d128", 8192, 128, 2, 256, 128, 7, True, 1024, "bf16"),
    ("causal_exact_only", 1024, 64, 2, 64, 32, 6, True, 4096, "bf16"),
    ("causal_fp32", 2048, 64, 1, 64, 64, 6, True, 256, "fp32"),
    # shapes aimed at the tensor-core kernels: ragged sample chunks, 1- and 3-tile blocks, odd leaves
    ("tc_m100", 2048, 64, 2, 256, 100, 6, False, 0, "bf16"),
    ("tc_m200_d128", 2048, 128, 2, 128, 200, 7, False, 0, "bf16"),
    ("tc_block384", 1536, 64, 2, 384, 64, 5, False, 0, "bf16"),
    ("tc_m0_d128", 1024, 128, 1, 256, 0, 6, False, 0, "bf16"),
    ("tc_many_heads", 1024, 64, 16, 256, 128, 6, False, 0, "bf16"),
    ("tc_causal_leaf384", 1536, 128, 2, 128, 64, 6, True, 384, "bf16"),
    ("tc_causal_d64", 4096, 64, 2, 256, 256, 8, True, 1024, "bf16"),
]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_hash_planted_near_zero(ha, dtype):
    """Rows planted on the near-zero boundary of the sortLSH signs ("HyperAttention: Long-context Attention in
    Near-Linear Time", summary page, "Approach": bit j is the sign of x.P_j). fp32: every 4th query and key row
    has its component along P_(row mod r) removed in float64, so that |x.P_j| lands far below 1e-4 * ||x||;
    bf16 (whose rounding cannot get that close): every 16th row is exactly zero, the sign tie (bit 0, not
    flagged). Ranks, flags, permutations and the output must match the oracle exactly like everywhere else."""
    n, d, bh, block, m, r, seed = 4096, 64, 2, 256, 128, 8, 4242
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=77, planted=0.05, dtype=dtype)
    P = oracle.draw_projection(seed, d, r).astype(np.float64)
    if dtype == "fp32":
        for X in (Qh, Kh):
            rows = np.arange(0, n, 4)
            for h in range(bh):
                x = X[h, rows].astype(np.float64)
                pj = P[:, rows % r].T                                   # (rows, d): the projection each row loses
                x -= ((x * pj).sum(axis=1) / (pj * pj).sum(axis=1))[:, None] * pj
                X[h, rows] = x.astype(np.float32)
    else:
        for X in (Qh, Kh):
            X[:, ::16] = 0
    Qf, Kf, Vf = wl.as_f32(Qh), wl.as_f32(Kh), wl.as_f32(Vh)
    got = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=False, seed=seed, dtype=dtype,
                  kernel="auto")
    check_ranks_and_perms(ha, Qf, Kf, n=n, bh=bh, r=r, causal=False, base=4096, seed=seed)
    near = ha.debug_copy("near", 0, np.uint8, bh * 2 * n).reshape(bh, 2, n)
    if dtype == "fp32":
        assert near[:, :, ::4].mean() > 0.99, "planted rows are flagged near zero"
    else:
        assert not near[:, :, ::16].any(), "zero rows: every projection is exactly 0, which is not below 0"
    for h in range(bh):
        ref = oracle.forward(Qf[h], Kf[h], Vf[h], block=block, m=m, r=r, causal=False, seed=seed, bh=h)
        assert rel_err(got[h], ref["O"]) < TOL[dtype]


@pytest.mark.parametrize("kernel", ["simt", "auto", "tc"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_parity_small(ha, case, kernel):
    name, n, d, bh, block, m, r, causal, base, dtype = case
    if kernel != "simt" and dtype == "fp32":
        pytest.skip("the tensor-core kernels take bf16 inputs")
    if kernel == "tc" and not tc_shape(n, block, causal, base):
        pytest.skip("shape outside the tensor-core kernels (b' or the causal leaf not a multiple of 128)")
    seed = 1000 + sum(map(ord, name))
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=seed, planted=0.05, sinks=causal, dtype=dtype)
    Qf, Kf, Vf = wl.as_f32(Qh), wl.as_f32(Kh), wl.as_f32(Vh)
    got = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=causal, seed=seed, base=base,
                  dtype=dtype, kernel=kernel)
    check_ranks_and_perms(ha, Qf, Kf, n=n, bh=bh, r=r, causal=causal, base=base, seed=seed)
    for h in range(bh):
        ref = oracle.forward(Qf[h], Kf[h], Vf[h], block=block, m=m, r=r, causal=causal, base=base, seed=seed, bh=h)
        e = rel_err(got[h], ref["O"])
        assert e < TOL[dtype], f"head {h}: relative L2 error {e:.3e}"
        if not causal:
            lse = ha.debug_copy("lse", 0, np.float32, bh * n).reshape(bh, n)[h]
            assert np.max(np.abs(lse - ref["L"])) < LSE_TOL[dtype]


def test_bf16_output(ha):
    n, d, bh, block, m, r, seed = 4096, 128, 2, 256, 256, 7, 55
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=seed, dtype="bf16")
    got = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=False, seed=seed, out_dtype="bf16")
    for h in range(bh):
        ref = oracle.forward(wl.as_f32(Qh[h]), wl.as_f32(Kh[h]), wl.as_f32(Vh[h]), block=block, m=m, r=r,
                             causal=False, seed=seed, bh=h)["O"]
        # the bf16 rounding of the output alone contributes up to ~2^-9 relative per element
        assert rel_err(got[h], ref) < 2e-3 + 2.0 ** -9


@pytest.mark.parametrize("n,d,bh,block,m,r,causal,base", [
    (2048, 64, 2, 128, 64, 6, False, 0),
    (1024, 128, 11, 256, 128, 7, False, 0),     # 11 problems in 8 uneven groups
    (2048, 64, 5, 128, 64, 6, True, 512),
])
def test_forward_host_matches_device(ha, n, d, bh, block, m, r, causal, base):
    """The host-buffer entry point (problem groups pipelined over copy streams) equals the device one."""
    seed = 77
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=seed, dtype="bf16")
    dev = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=causal, seed=seed, base=base,
                  out_dtype="bf16", debug=False)
    Oh = np.zeros((bh, n, d), np.uint16)
    Qp, Kp, Vp, Op = (torch.from_numpy(x.view(np.int16)).pin_memory() for x in (Qh, Kh, Vh, Oh))
    ha.forward_host(Qp, Kp, Vp, Op, n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=seed)
    assert np.array_equal(wl.as_f32(Op.numpy().view(np.uint16)).astype(np.float64), dev)
    # pageable buffers take the same path
    ha.forward_host(Qh, Kh, Vh, Oh, n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=seed)
    assert np.array_equal(wl.as_f32(Oh).astype(np.float64), dev)


def test_deterministic(ha):
    n, d, bh, block, m, r, seed = 4096, 64, 2, 256, 256, 8, 5
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=seed, dtype="bf16")
    a = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=False, seed=seed)
    b = run_gpu(ha, Qh, Kh, Vh, n=n, d=d, bh=bh, block=block, m=m, r=r, causal=False, seed=seed)
    assert np.array_equal(a, b)


def test_invalid_arguments_enqueue_nothing(ha):
    x = torch.zeros((1, 1024, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(x)
    ha.set_options(stream=torch.cuda.current_stream().cuda_stream)
    bad = [dict(n=1024, d=96, heads=1, block=64, m=8, r=4, causal=False),    # d
           dict(n=1000, d=64, heads=1, block=64, m=8, r=4, causal=False),    # n % block
           dict(n=1024, d=64, heads=1, block=64, m=2000, r=4, causal=False),  # m > n
           dict(n=1024, d=64, heads=1, block=64, m=8, r=17, causal=False),   # r
           dict(n=1024, d=64, heads=1, block=64, m=8, r=4, causal=True)]     # n = 1024 <= base is fine -> valid
    for i, kw in enumerate(bad[:-1]):
        with pytest.raises(binding.HAError):
            ha.forward(x, x, x, o, seed=1, **kw)
    with pytest.raises(binding.HAError):
        ha.forward(x, x, x, x, n=1024, d=64, heads=1, block=64, m=8, r=4, causal=False, seed=1)   # aliasing
    ha.set_options(causal_base=96, stream=torch.cuda.current_stream().cuda_stream)
    x2 = torch.zeros((1, 384, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.HAError):
        ha.forward(x2, x2, x2, torch.zeros_like(x2), n=384, d=64, heads=1, block=64, m=8, r=4, causal=True, seed=1)
    assert ha.status() == 0


# ------------------------------------------------------------------ full-size workloads, sampled rows

FULL = ["mid_bf16_n32768", "long_bf16_n131072", "prefill_causal_bf16_n32768", "very_long_causal_bf16_n524288"]


@pytest.mark.parametrize("name", FULL)
def test_parity_full_size_sampled(ha, name):
    w = wl.WORKLOADS[name]
    heads = [0, w.bh - 1]
    Qh, Kh, Vh = wl.workload_inputs(w)
    got = run_gpu(ha, Qh, Kh, Vh, n=w.n, d=w.d, bh=w.bh, block=w.block, m=w.m, r=w.r, causal=w.causal,
                  seed=w.algo_seed, base=w.base or 4096, dtype=w.dtype, debug=not w.causal)
    Qf, Kf, Vf = wl.as_f32(Qh), wl.as_f32(Kh), wl.as_f32(Vh)
    check_ranks_and_perms(ha, Qf, Kf, n=w.n, bh=w.bh, r=w.r, causal=w.causal, base=w.base or 4096,
                          seed=w.algo_seed, heads=heads)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(w.n, 192, replace=False), [0, 1, w.n // 2, w.n - 1]]))
    for h in heads:
        ref = oracle.forward(Qf[h], Kf[h], Vf[h], block=w.block, m=w.m, r=w.r, causal=w.causal, base=w.base,
                             seed=w.algo_seed, bh=h, rows=rows)["O"]
        e = rel_err(got[h][rows], ref)
        assert e < TOL[w.dtype], f"head {h}: relative L2 error {e:.3e} on {len(rows)} sampled rows"
