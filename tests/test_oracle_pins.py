"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against one of: an independent implementation of a published algorithm
(numpy's Philox), a distribution the draws must follow, a closed form the method reduces to
("HyperAttention: Long-context Attention in Near-Linear Time", summary page, "Approach": with one block
covering all keys, or with every column sampled, the estimate is exact softmax attention), an invariant
(the estimated normaliser is at least the exact block sum; every output row is a convex combination of
value rows), unbiasedness of the sampled normaliser, or a brute-force dense restatement of the whole
method on tiny inputs.
"""
import numpy as np
import pytest
from scipy import stats

from approximate_long_context_b200 import workload as wl


# ---------------------------------------------------------------- independent helpers (numpy only)

def exact_attention_np(Q, K, V, causal=False):
    S = Q.astype(np.float64) @ K.astype(np.float64).T
    if causal:
        S = np.where(np.tril(np.ones(S.shape, bool)), S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    A = np.exp(S)
    return (A @ V.astype(np.float64)) / A.sum(axis=1, keepdims=True)


def gray_code(k):
    return k ^ (k >> 1)


def ranks_np(X, P):
    """sortLSH ranks from float64 projections: bits by sign, rank = position of the code in the
    reflected Gray sequence (found by table lookup of the forward Gray code)."""
    r = P.shape[1]
    proj = X.astype(np.float64) @ P.astype(np.float64)
    bits = (proj > 0).astype(np.int64)
    code = (bits << np.arange(r)).sum(axis=1) if r > 0 else np.zeros(len(X), np.int64)
    inv = np.zeros(1 << r, np.int64)
    inv[gray_code(np.arange(1 << r))] = np.arange(1 << r)
    return inv[code], np.abs(proj)


def weights_noncausal(rq, rk, N, block, S):
    """Dense weight matrix W (N x N): 1 on same-block pairs of the sorted orders, N/m on sampled columns
    outside the query's block, 0 elsewhere."""
    bp = min(block, N)
    pq = np.argsort(rq, kind="stable")
    pk = np.argsort(rk, kind="stable")
    blk_q = np.empty(N, np.int64); blk_q[pq] = np.arange(N) // bp
    blk_k = np.empty(N, np.int64); blk_k[pk] = np.arange(N) // bp
    W = (blk_q[:, None] == blk_k[None, :]).astype(np.float64)
    m = len(S)
    if m:
        cols = np.zeros(N, bool); cols[S] = True
        W += np.where((blk_q[:, None] != blk_k[None, :]) & cols[None, :], N / m, 0.0)
    return W


def weighted_softmax_np(Q, K, V, W):
    S = Q.astype(np.float64) @ K.astype(np.float64).T
    S = np.where(W > 0, S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    A = W * np.exp(S)
    return (A @ V.astype(np.float64)) / A.sum(axis=1, keepdims=True), A.sum(axis=1)


def rand_qkv(n, d, seed, planted=0.1):
    Q, K, V = wl.make_head(n, d, seed, 0, planted, False)
    return Q, K, V


# ---------------------------------------------------------------- random draws

@pytest.mark.parametrize("key", [(0, 0), (1234, 1), (0xDEADBEEFCAFEBABE, 2), (2**64 - 1, 2**63 + 5)])
@pytest.mark.parametrize("ctr", [(1, 0, 0, 0), (7, 3, 2, 0), (2**40 + 3, 1, 0, 9), (5, 2**64 - 1, 2**63, 1)])
def test_philox_matches_numpy(ora, key, ctr):
    # numpy increments its counter before each block, so its state must hold ctr - 1 (no borrow here)
    g = np.random.Philox(key=np.array(key, np.uint64), counter=np.array((ctr[0] - 1,) + ctr[1:], np.uint64))
    expect = g.random_raw(4).astype(np.uint64)
    got = ora.philox4x64_10(np.array(ctr, np.uint64), np.array(key, np.uint64))
    assert np.array_equal(got, expect)


def test_projection_is_standard_normal(ora):
    vals = np.concatenate([ora.draw_projection(seed, 128, 16).ravel() for seed in range(40)])
    assert vals.dtype == np.float32 and vals.size == 40 * 128 * 16
    assert abs(vals.mean()) < 5 / np.sqrt(vals.size)
    assert abs(vals.var() - 1) < 5 * np.sqrt(2 / vals.size)
    assert stats.kstest(vals.astype(np.float64), "norm").pvalue > 1e-3
    # deterministic in the seed, different across seeds, layout (d, r) with r columns
    assert np.array_equal(ora.draw_projection(5, 64, 8), ora.draw_projection(5, 64, 8))
    assert not np.array_equal(ora.draw_projection(5, 64, 8), ora.draw_projection(6, 64, 8))


def test_projection_columns_independent(ora):
    P = np.concatenate([ora.draw_projection(s, 64, 9) for s in range(200)], axis=0)
    C = np.corrcoef(P.T.astype(np.float64))
    off = C[~np.eye(9, dtype=bool)]
    assert np.abs(off).max() < 5 / np.sqrt(P.shape[0])


def test_samples_basic(ora):
    for (N, m) in [(1, 1), (10, 0), (64, 64), (1000, 17), (131072, 256)]:
        S = ora.draw_samples(99, 3, 1, N, m)
        assert len(S) == m
        assert np.all(np.diff(S) > 0)
        if m:
            assert S.min() >= 0 and S.max() < N
    assert np.array_equal(ora.draw_samples(1, 0, 1, 50, 50), np.arange(50))
    with pytest.raises(ValueError):
        ora.draw_samples(1, 0, 1, 5, 6)
    a, b, c = ora.draw_samples(1, 0, 1, 1000, 20), ora.draw_samples(1, 1, 1, 1000, 20), ora.draw_samples(1, 0, 2, 1000, 20)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


def test_samples_uniform(ora):
    N, m, T = 64, 8, 4000
    counts = np.zeros(N)
    pair = np.zeros((N, N))
    for seed in range(T):
        S = ora.draw_samples(seed, 0, 1, N, m)
        counts[S] += 1
        pair[np.ix_(S, S)] += 1
    exp = T * m / N
    chi2 = ((counts - exp) ** 2 / exp).sum()
    assert stats.chi2.sf(chi2, N - 1) > 1e-4
    # pairwise inclusion probability m(m-1)/(N(N-1)) for every pair (without replacement)
    p2 = pair[~np.eye(N, dtype=bool)] / T
    target = m * (m - 1) / (N * (N - 1))
    assert abs(p2.mean() - target) < 1e-3


# ---------------------------------------------------------------- hash

def test_gray_rank_inverse_and_adjacency(ora):
    for k in range(1 << 16):
        assert ora.gray_rank(gray_code(k)) == k
    for k in range((1 << 16) - 1):
        assert bin(gray_code(k) ^ gray_code(k + 1)).count("1") == 1


@pytest.mark.parametrize("d,r", [(64, 6), (64, 8), (128, 7), (128, 9), (32, 16), (64, 0)])
def test_hash_matches_float64_signs(ora, d, r):
    X = np.random.default_rng(d * 100 + r).standard_normal((4000, d)).astype(np.float32) * np.float32(d ** -0.25)
    P = ora.draw_projection(77, d, r)
    rank, near = ora.hash_rows(X, P)
    ref, absproj = ranks_np(X, P)
    norms = np.linalg.norm(X.astype(np.float64), axis=1)
    # a projection far from zero decides its bit identically in fp32 and float64
    safe = (absproj >= 1e-3 * norms[:, None]).all(axis=1) if r else np.ones(len(X), bool)
    assert safe.mean() > 0.9
    assert np.array_equal(rank[safe].astype(np.int64), ref[safe])
    # the near-zero flag marks exactly the rows with a projection below 1e-4 * ||x|| (up to fp32 rounding)
    clearly_near = (absproj < 0.9e-4 * norms[:, None]).any(axis=1) if r else np.zeros(len(X), bool)
    clearly_far = (absproj > 1.1e-4 * norms[:, None]).all(axis=1) if r else np.ones(len(X), bool)
    assert near[clearly_near].all() and not near[clearly_far].any()
    if r == 0:
        assert (rank == 0).all()


def test_hash_sign_tie_is_zero_bit(ora):
    X = np.zeros((3, 16), np.float32)
    X[1, 0] = 1.0
    X[2, 0] = X[2, 1] = 1.0
    P = np.ones((16, 4), np.float32)
    P[0, 1] = -1.0
    P[1, 2] = -1.0
    rank, near = ora.hash_rows(X, P)
    # zero row: every projection is exactly 0 -> code 0; |p| < 1e-4 * 0 is false, so it is not flagged
    assert rank[0] == 0 and near[0] == 0
    # e_0: projections (1, -1, 1, 1) -> code 0b1101
    assert rank[1] == ora.gray_rank(0b1101) and near[1] == 0
    # e_0 + e_1: projections (2, 0, 0, 2) -> exact zeros give bit 0 and flag the row
    assert rank[2] == ora.gray_rank(0b1001) and near[2] == 1


def test_sort_stable(ora):
    rng = np.random.default_rng(3)
    for R in [1, 4, 256, 65536]:
        rank = rng.integers(0, R, 5000).astype(np.uint16)
        assert np.array_equal(ora.sort_segment(rank), np.argsort(rank, kind="stable"))


# ---------------------------------------------------------------- closed forms and invariants

@pytest.mark.parametrize("n,d,m,r", [(256, 32, 16, 4), (512, 64, 0, 6), (128, 16, 128, 3)])
def test_block_n_equals_exact(ora, n, d, m, r):
    Q, K, V = rand_qkv(n, d, 11)
    out = ora.forward(Q, K, V, block=n, m=m, r=r, causal=False, seed=5)
    np.testing.assert_allclose(out["O"], exact_attention_np(Q, K, V), rtol=1e-10, atol=1e-12)
    # the oracle's own exact routine agrees with the textbook formula too
    np.testing.assert_allclose(ora.exact_attention(Q, K, V, causal=False), exact_attention_np(Q, K, V), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n,block,r", [(256, 16, 5), (512, 64, 6), (128, 128, 2)])
def test_all_columns_sampled_equals_exact(ora, n, block, r):
    Q, K, V = rand_qkv(n, 32, 12)
    out = ora.forward(Q, K, V, block=block, m=n, r=r, causal=False, seed=6)
    np.testing.assert_allclose(out["O"], exact_attention_np(Q, K, V), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n,block", [(256, 16), (1024, 64), (192, 64)])
def test_no_samples_identical_codes_is_block_diagonal(ora, n, block):
    Q, K, V = rand_qkv(n, 32, 13)
    out = ora.forward(Q, K, V, block=block, m=0, r=0, causal=False, seed=7)
    ref = np.concatenate([exact_attention_np(Q[i:i + block], K[i:i + block], V[i:i + block])
                          for i in range(0, n, block)])
    np.testing.assert_allclose(out["O"], ref, rtol=1e-10, atol=1e-12)


def test_normaliser_at_least_block_sum(ora):
    Q, K, V = rand_qkv(1024, 64, 14)
    out = ora.forward(Q, K, V, block=64, m=64, r=6, causal=False, seed=8, want_parts=True)
    L, L1, L2 = out["L"], out["L1"], out["L2"]
    assert np.all(L >= L1)
    np.testing.assert_allclose(L, np.logaddexp(L1, L2), rtol=0, atol=1e-12)
    assert np.isfinite(L2).mean() > 0.99


def test_normaliser_unbiased(ora):
    n, d, block, m, r, T = 64, 16, 8, 8, 3, 10000
    Q, K, V = rand_qkv(n, d, 15, planted=0.2)
    D = np.exp(Q.astype(np.float64) @ K.astype(np.float64).T).sum(axis=1)
    est = np.zeros((T, n))
    for seed in range(T):
        est[seed] = np.exp(ora.forward(Q, K, V, block=block, m=m, r=r, causal=False, seed=seed)["L"])
    mean = est.mean(axis=0)
    se = est.std(axis=0, ddof=1) / np.sqrt(T)
    z = (mean - D) / se
    assert np.abs(z).max() < 5.0, np.abs(z).max()


def test_rows_are_convex_combinations(ora):
    Q, K, V = rand_qkv(2048, 64, 16)
    lo, hi = V.min(axis=0).astype(np.float64), V.max(axis=0).astype(np.float64)
    for causal, base in [(False, 0), (True, 256)]:
        O = ora.forward(Q, K, V, block=64, m=32, r=6, causal=causal, base=base, seed=9)["O"]
        assert np.all(O >= lo - 1e-12) and np.all(O <= hi + 1e-12)


# ---------------------------------------------------------------- causal

def test_causal_base_at_least_n_is_exact_causal(ora):
    Q, K, V = rand_qkv(300, 32, 17)
    out = ora.forward(Q, K, V, block=50, m=10, r=5, causal=True, base=300, seed=10)
    np.testing.assert_allclose(out["O"], exact_attention_np(Q, K, V, causal=True), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n,base,m", [(256, 32, 0), (256, 32, 32), (512, 64, 17)])
def test_causal_full_blocks_are_exact_causal(ora, n, base, m):
    Q, K, V = rand_qkv(n, 32, 18)
    out = ora.forward(Q, K, V, block=n, m=m, r=6, causal=True, base=base, seed=11)
    np.testing.assert_allclose(out["O"], exact_attention_np(Q, K, V, causal=True), rtol=1e-10, atol=1e-12)


def test_causal_rejects_bad_shapes(ora):
    Q, K, V = rand_qkv(96, 16, 19)
    with pytest.raises(ValueError):
        ora.forward(Q, K, V, block=16, m=4, r=3, causal=True, base=64, seed=1)   # 96 != 64 * 2^L
    Q, K, V = rand_qkv(128, 16, 19)
    with pytest.raises(ValueError):
        ora.forward(Q, K, V, block=16, m=40, r=3, causal=True, base=32, seed=1)  # m > smallest N = 32


# ---------------------------------------------------------------- dense brute force of the whole method

def _dense_causal_weights(Q, K, P, block, base, m, seed, bh, ora):
    n = len(Q)
    rq_all, aq = ranks_np(Q, P)
    rk_all, ak = ranks_np(K, P)
    W = np.zeros((n, n))
    leaf = min(base, n)
    for q in range(n):
        lo = q - q % leaf
        W[q, lo:q + 1] = 1.0

    def rec(node, s, length):
        if length <= leaf:
            return
        h = length // 2
        rec(2 * node, s, h)
        rec(2 * node + 1, s + h, h)
        S = ora.draw_samples(seed, bh, node, h, m)
        W[s + h:s + length, s:s + h] = weights_noncausal(rq_all[s + h:s + length], rk_all[s:s + h], h, block, S)

    rec(1, 0, n)
    return W, np.concatenate([aq, ak])


@pytest.mark.parametrize("seed", [21, 22, 23])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_bruteforce(ora, seed, causal):
    n, d, block, m, r, base, bh = 256, 16, 16, 12, 4, 32, 3
    Q, K, V = rand_qkv(n, d, seed)
    P = ora.draw_projection(seed, d, r)
    if causal:
        W, absproj = _dense_causal_weights(Q, K, P, block, base, m, seed, bh, ora)
    else:
        rq, aq = ranks_np(Q, P)
        rk, ak = ranks_np(K, P)
        W = weights_noncausal(rq, rk, n, block, ora.draw_samples(seed, bh, 1, n, m))
        absproj = np.concatenate([aq, ak])
    X = np.concatenate([Q, K]).astype(np.float64)
    # fp32 and float64 take the same sign decisions when no projection is within 1e-5 * ||x|| of zero
    assert (absproj >= 1e-5 * np.linalg.norm(X, axis=1)[:, None]).all(), "pick a seed without near-zero projections"
    ref, den = weighted_softmax_np(Q, K, V, W)
    out = ora.forward(Q, K, V, block=block, m=m, r=r, causal=causal, base=base, seed=seed, bh=bh)
    np.testing.assert_allclose(out["O"], ref, rtol=1e-10, atol=1e-12)
    S = Q.astype(np.float64) @ K.astype(np.float64).T
    mx = np.where(W > 0, S, -np.inf).max(axis=1)
    np.testing.assert_allclose(out["L"], mx + np.log(den), rtol=0, atol=1e-10)


def test_rows_subset_matches_full(ora):
    Q, K, V = rand_qkv(1024, 32, 24)
    rows = np.array([0, 5, 511, 512, 777, 1023])
    for causal in (False, True):
        full = ora.forward(Q, K, V, block=32, m=16, r=5, causal=causal, base=128, seed=3)
        part = ora.forward(Q, K, V, block=32, m=16, r=5, causal=causal, base=128, seed=3, rows=rows)
        np.testing.assert_array_equal(part["O"], full["O"][rows])


def test_level_perms(ora):
    rng = np.random.default_rng(5)
    n = 512
    rank = rng.integers(0, 16, 2 * n).astype(np.uint16)
    pq, pk = ora.level_perms(rank, n, 0)
    assert np.array_equal(pq, np.argsort(rank[:n], kind="stable"))
    assert np.array_equal(pk, np.argsort(rank[n:], kind="stable"))
    pq, pk = ora.level_perms(rank, n, 2)            # nodes of length 256: Q lower / K upper halves of 128
    for j in range(2):
        s = j * 256
        assert np.array_equal(pq[j * 128:(j + 1) * 128], np.argsort(rank[s + 128:s + 256], kind="stable"))
        assert np.array_equal(pk[j * 128:(j + 1) * 128], np.argsort(rank[n + s:n + s + 128], kind="stable"))


# ---------------------------------------------------------------------------------------- hardness diagnostics
# alpha = n * max_j ||(D^-1 A) e_j||^2 and kappa = max/min row sum of A outside the row's sortLSH block
# ("HyperAttention: Long-context Attention in Near-Linear Time", research-map summary, "Approach", "Key results").

def test_diagnostics_uniform_attention(ora):
    """Q = 0: every softmax row is uniform, so each column has squared norm n * (1/n)^2 and alpha = 1; every row
    has the same n - b' unit entries outside its block, so kappa = 1. With one block, nothing is outside: NaN."""
    rng = np.random.default_rng(41)
    n, d = 96, 16
    Q = np.zeros((n, d), np.float32)
    K = rng.standard_normal((n, d)).astype(np.float32)
    alpha, kappa = ora.diagnostics(Q, K, block=32, r=5, seed=3)
    assert alpha == pytest.approx(1.0, rel=1e-12)
    assert kappa == pytest.approx(1.0, rel=1e-12)
    alpha1, kappa1 = ora.diagnostics(Q, K, block=n, r=5, seed=3)
    assert alpha1 == pytest.approx(1.0, rel=1e-12) and np.isnan(kappa1)


def test_diagnostics_dominant_column(ora):
    """One key aligned with every query and far larger than the rest takes almost all of every row's weight:
    alpha -> n^2. Dropping that column (first_col past it) leaves alpha far below."""
    rng = np.random.default_rng(43)
    n, d = 64, 16
    u = rng.standard_normal(d).astype(np.float32)
    u /= np.linalg.norm(u)
    Q = (np.tile(u, (n, 1)) * 4.0 + 0.01 * rng.standard_normal((n, d))).astype(np.float32)
    K = (0.1 * rng.standard_normal((n, d))).astype(np.float32)
    K[0] = 8.0 * u
    alpha, _ = ora.diagnostics(Q, K, block=16, r=4, seed=5)
    assert alpha == pytest.approx(n * n, rel=1e-6)
    alpha_rest, _ = ora.diagnostics(Q, K, block=16, r=4, seed=5, first_col=1)
    assert alpha_rest < 1e-6


def test_diagnostics_kappa_planted_ratio(ora):
    """All keys equal (k = u): a query row's entries are all exp(q . u). Half the queries are 0 (entries 1), half
    are t*u (entries exp(t |u|^2)); every row has n - b' entries outside its block whatever the sort does, so
    kappa = exp(t |u|^2) exactly."""
    n, d, t = 128, 8, 0.75
    u = np.linspace(-1.0, 1.0, d).astype(np.float32)
    K = np.tile(u, (n, 1)).astype(np.float32)
    Q = np.zeros((n, d), np.float32)
    Q[n // 2:] = (t * u).astype(np.float32)
    _, kappa = ora.diagnostics(Q, K, block=32, r=6, seed=9)
    s = float(np.dot((t * u).astype(np.float32).astype(np.float64), u.astype(np.float64)))
    assert kappa == pytest.approx(np.exp(s), rel=1e-12)


def test_diagnostics_alpha_ignores_row_order(ora):
    """alpha depends on column norms of D^-1 A only: permuting the queries (rows) leaves it unchanged."""
    rng = np.random.default_rng(47)
    n, d = 80, 16
    Q = (0.5 * rng.standard_normal((n, d))).astype(np.float32)
    K = (0.5 * rng.standard_normal((n, d))).astype(np.float32)
    a0, _ = ora.diagnostics(Q, K, block=16, r=5, seed=2)
    a1, _ = ora.diagnostics(Q[rng.permutation(n)], K, block=16, r=5, seed=2)
    assert a1 == pytest.approx(a0, rel=1e-12)


# ---------------------------------------------------------------- row-norm sampling of the product with V
# "HyperAttention: Long-context Attention in Near-Linear Time" (summary page, "Approach"): the product of the
# normalised attention with V may be approximated by sampling rows of V in proportion to their squared norms.

def _philox_words(seed, bh, node, nblocks):
    """Words of Philox4x64-10 under key (seed, 3) at counters (c, node, bh, 0), c = 0..nblocks-1 (numpy)."""
    # numpy increments its 256-bit counter before each block: start one below (c=0, node, bh, 0)
    start = [2**64 - 1, node - 1, bh, 0] if node > 0 else [2**64 - 1, 2**64 - 1, bh - 1, 0]
    g = np.random.Philox(key=np.array([seed, 3], np.uint64), counter=np.array(start, np.uint64))
    return g.random_raw(4 * nblocks).astype(np.uint64)


def test_rownorm_draws_tiny_bruteforce(ora):
    """Squared norms 1, 0, 3: p = (1/4, 0, 3/4); a draw is row 0 exactly when u < 1/4, else row 2, and its
    weight is 1/(m p)."""
    V = np.zeros((3, 4), np.float32)
    V[0, 0] = 1.0
    V[2, :3] = 1.0
    m, seed, bh, node = 11, 77, 2, 5
    S, lw = ora.draw_rownorm(seed, bh, node, V, m)
    w = _philox_words(seed, bh, node, (m + 3) // 4)
    u = (w[:m] >> np.uint64(11)).astype(np.float64) * 2.0**-53
    expect = np.where(u < 0.25, 0, 2)
    assert np.array_equal(S, expect)
    p = np.array([0.25, 0.0, 0.75])
    np.testing.assert_allclose(np.exp(lw), 1.0 / (m * p[expect]), rtol=1e-14)
    assert 0 < (expect == 0).sum() < m


def test_rownorm_draw_frequencies(ora):
    rng = np.random.default_rng(31)
    N, d, m = 60, 8, 200000
    V = (rng.standard_normal((N, d)) * rng.uniform(0.1, 3.0, (N, 1))).astype(np.float32)
    V[[4, 17, 59]] = 0.0
    S, _ = ora.draw_rownorm(5, 1, 1, V, m)
    cnt = np.bincount(S, minlength=N)
    assert cnt[[4, 17, 59]].sum() == 0
    p = (V.astype(np.float64) ** 2).sum(axis=1)
    p /= p.sum()
    keep = p > 0
    chi2 = (((cnt[keep] - m * p[keep]) ** 2) / (m * p[keep])).sum()
    assert stats.chi2.sf(chi2, keep.sum() - 1) > 1e-4
    a = ora.draw_rownorm(5, 1, 1, V, 64)[0]
    assert not np.array_equal(a, ora.draw_rownorm(5, 2, 1, V, 64)[0])
    assert not np.array_equal(a, ora.draw_rownorm(5, 1, 2, V, 64)[0])
    assert not np.array_equal(a, ora.draw_rownorm(6, 1, 1, V, 64)[0])


def test_rownorm_all_zero_rows_draw_nothing(ora):
    S, lw = ora.draw_rownorm(1, 0, 1, np.zeros((16, 8), np.float32), 5)
    assert np.all(S == -1) and np.all(lw == -np.inf)
    Q, K, _ = rand_qkv(128, 16, 3)
    out = ora.forward(Q, K, np.zeros((128, 16), np.float32), block=16, m=8, r=3, causal=False, seed=1,
                      sampling="rownorm")
    assert np.all(out["O"] == 0.0)


def _dense_rownorm_weights(n, rq, rk, block, S, lw):
    """Numerator weights of one problem: 1 on same-block pairs, sum of exp(lw) over draws of column j outside
    the query's block."""
    W = weights_noncausal(rq, rk, n, block, np.zeros(0, np.int64))
    bp = min(block, n)
    pq = np.argsort(rq, kind="stable")
    pk = np.argsort(rk, kind="stable")
    blk_q = np.empty(n, np.int64); blk_q[pq] = np.arange(n) // bp
    blk_k = np.empty(n, np.int64); blk_k[pk] = np.arange(n) // bp
    add = np.zeros(n)
    np.add.at(add, S[S >= 0], np.exp(lw[S >= 0]))
    return W + np.where(blk_q[:, None] != blk_k[None, :], add[None, :], 0.0)


@pytest.mark.parametrize("seed", [41, 42])
@pytest.mark.parametrize("causal", [False, True])
def test_rownorm_dense_bruteforce(ora, seed, causal):
    """The whole estimate restated densely: numerator weights from the row-norm draws, normaliser weights
    from the uniform draws (the same dense form as test_dense_bruteforce)."""
    n, d, block, m, r, base, bh = 256, 16, 16, 12, 4, 32, 1
    Q, K, V = rand_qkv(n, d, seed)
    P = ora.draw_projection(seed, d, r)
    rq_all, aq = ranks_np(Q, P)
    rk_all, ak = ranks_np(K, P)
    X = np.concatenate([Q, K]).astype(np.float64)
    assert (np.concatenate([aq, ak]) >= 1e-5 * np.linalg.norm(X, axis=1)[:, None]).all()
    if causal:
        Wd, _ = _dense_causal_weights(Q, K, P, block, base, m, seed, bh, ora)
        Wn = np.zeros((n, n))
        for q in range(n):
            lo = q - q % base
            Wn[q, lo:q + 1] = 1.0

        def rec(node, s, length):
            if length <= base:
                return
            h = length // 2
            rec(2 * node, s, h)
            rec(2 * node + 1, s + h, h)
            S, lw = ora.draw_rownorm(seed, bh, node, V[s:s + h], m)
            Wn[s + h:s + length, s:s + h] = _dense_rownorm_weights(h, rq_all[s + h:s + length], rk_all[s:s + h],
                                                                   block, S, lw)
        rec(1, 0, n)
    else:
        Wd = weights_noncausal(rq_all, rk_all, n, block, ora.draw_samples(seed, bh, 1, n, m))
        S, lw = ora.draw_rownorm(seed, bh, 1, V, m)
        Wn = _dense_rownorm_weights(n, rq_all, rk_all, block, S, lw)
    Sc = Q.astype(np.float64) @ K.astype(np.float64).T
    mx = np.where(Wd > 0, Sc, -np.inf).max(axis=1, keepdims=True)
    E = np.exp(Sc - mx)
    ref = ((Wn * E) @ V.astype(np.float64)) / (Wd * E).sum(axis=1, keepdims=True)
    out = ora.forward(Q, K, V, block=block, m=m, r=r, causal=causal, base=base, seed=seed, bh=bh, sampling="rownorm")
    np.testing.assert_allclose(out["O"], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["L"], mx[:, 0] + np.log((Wd * E).sum(axis=1)), rtol=0, atol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
def test_rownorm_single_value_row_is_exact(ora, causal):
    """With one nonzero value row every draw picks it with weight 1/m, so the estimated numerator (output times
    estimated normaliser) is exactly the numerator of exact attention."""
    n, d = 256, 16
    Q, K, V = rand_qkv(n, d, 9)
    j0 = 70
    V1 = np.zeros_like(V)
    V1[j0] = V[j0]
    Sc = Q.astype(np.float64) @ K.astype(np.float64).T
    if causal:
        Sc = np.where(np.tril(np.ones((n, n), bool)), Sc, -np.inf)
    num = np.exp(Sc[:, j0])[:, None] * V1[j0].astype(np.float64)[None, :]
    for seed in (1, 2, 3):
        out = ora.forward(Q, K, V1, block=16, m=10, r=4, causal=causal, base=32, seed=seed, sampling="rownorm")
        np.testing.assert_allclose(out["O"] * np.exp(out["L"])[:, None], num, rtol=1e-10, atol=1e-300)


def test_rownorm_numerator_unbiased(ora):
    """Over independent draws the mean estimated numerator (output times estimated normaliser) is the exact
    numerator A V: within 5 standard errors per entry."""
    n, d, block, m, r, T = 64, 8, 8, 8, 3, 4000
    Q, K, V = rand_qkv(n, d, 16, planted=0.2)
    ref = np.exp(Q.astype(np.float64) @ K.astype(np.float64).T) @ V.astype(np.float64)
    est = np.zeros((T, n, d))
    for seed in range(T):
        out = ora.forward(Q, K, V, block=block, m=m, r=r, causal=False, seed=seed, sampling="rownorm")
        est[seed] = out["O"] * np.exp(out["L"])[:, None]
    se = est.std(axis=0, ddof=1) / np.sqrt(T)
    z = (est.mean(axis=0) - ref) / se
    assert np.abs(z).max() < 5.0, np.abs(z).max()


# ---------------------------------------------------------------- backward pass
# The gradients of sum(dO * O) with the sort and the draws held fixed. Pinned by finite differences of the
# (separately pinned) forward, by exact attention's gradient where the method reduces to it, and by two
# identities of a weighted softmax that hold for any weights.

def _loss(ora, Q, K, V, dO, kw):
    return float((ora.forward(Q, K, V, **kw)["O"] * dO.astype(np.float64)).sum())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sampling", ["uniform", "rownorm"])
def test_weights_reproduce_forward(ora, causal, sampling):
    n, d = 256, 16
    Q, K, V = rand_qkv(n, d, 61)
    kw = dict(block=16, m=12, r=4, causal=causal, base=32, seed=5, bh=2, sampling=sampling)
    Wn, Wd = ora.weights(Q, K, V, **kw)
    S = Q.astype(np.float64) @ K.astype(np.float64).T
    mx = np.where((Wn > 0) | (Wd > 0), S, -np.inf).max(axis=1, keepdims=True)
    E = np.exp(S - mx)
    ref = ora.forward(Q, K, V, **kw)
    np.testing.assert_allclose((Wn * E) @ V.astype(np.float64) / (Wd * E).sum(1, keepdims=True), ref["O"],
                               rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(mx[:, 0] + np.log((Wd * E).sum(1)), ref["L"], rtol=0, atol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sampling,which", [("uniform", "Q"), ("uniform", "K"), ("uniform", "V"),
                                            ("rownorm", "Q"), ("rownorm", "K")])
def test_backward_finite_differences(ora, causal, sampling, which):
    """Central differences of the forward along a random direction. With row-norm sampling V also sets the
    draws and their weights, which the backward holds fixed, so V is checked by the identity test below."""
    n, d, eps = 128, 16, 1e-3
    Q, K, V = rand_qkv(n, d, 62)
    rng = np.random.default_rng(7)
    dO = rng.standard_normal((n, d)).astype(np.float32)
    kw = dict(block=16, m=12, r=4, causal=causal, base=32, seed=9, bh=0, sampling=sampling)
    g = ora.backward(Q, K, V, dO, **kw)["d" + which]
    X = {"Q": Q, "K": K, "V": V}[which]
    E = rng.standard_normal(X.shape)
    if which in "QK":   # leave alone the rows with a projection close enough to zero to change sign
        proj = X.astype(np.float64) @ ora.draw_projection(9, d, 4).astype(np.float64)
        E[np.abs(proj).min(axis=1) < 0.05] = 0.0
    Xp = (X + eps * E).astype(np.float32)
    Xm = (X - eps * E).astype(np.float32)
    args = lambda Y: [Y if nm == which else {"Q": Q, "K": K, "V": V}[nm] for nm in "QKV"]
    rank0 = ora.forward(Q, K, V, **kw)["rank"]
    for Y in (Xp, Xm):   # the perturbation must not move a row to another bucket
        assert np.array_equal(ora.forward(*args(Y), **kw)["rank"], rank0)
    fd = _loss(ora, *args(Xp), dO, kw) - _loss(ora, *args(Xm), dO, kw)
    an = float((g * (Xp.astype(np.float64) - Xm.astype(np.float64))).sum())
    assert abs(fd - an) <= 1e-5 * abs(an) + 1e-9, (fd, an)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_reduces_to_exact_attention(ora, causal):
    """One block covering every key (non-causal), or one exact causal leaf (c >= n): the estimate is exact
    softmax attention, and so is its gradient, written here from the definition."""
    n, d = 128, 16
    Q, K, V = rand_qkv(n, d, 63)
    dO = np.random.default_rng(8).standard_normal((n, d)).astype(np.float32)
    out = ora.backward(Q, K, V, dO, block=n, m=16, r=4, causal=causal, base=n, seed=2)
    Qd, Kd, Vd, G = (x.astype(np.float64) for x in (Q, K, V, dO))
    S = Qd @ Kd.T
    if causal:
        S = np.where(np.tril(np.ones((n, n), bool)), S, -np.inf)
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    dP = G @ Vd.T
    dS = P * (dP - (dP * P).sum(1, keepdims=True))
    np.testing.assert_allclose(out["dV"], P.T @ G, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(out["dQ"], dS @ Kd, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(out["dK"], dS.T @ Qd, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sampling", ["uniform", "rownorm"])
def test_backward_identities(ora, causal, sampling):
    """For any weighted softmax: shifting every key by the same vector leaves each row's output unchanged,
    so the key gradients sum to zero; and O is linear in V at fixed weights, so sum(dV * V) = sum(dO * O)."""
    n, d = 256, 16
    Q, K, V = rand_qkv(n, d, 64)
    dO = np.random.default_rng(9).standard_normal((n, d)).astype(np.float32)
    out = ora.backward(Q, K, V, dO, block=16, m=12, r=4, causal=causal, base=32, seed=4, bh=1, sampling=sampling)
    scale = np.abs(out["dK"]).sum(0).max()
    assert np.abs(out["dK"].sum(0)).max() <= 1e-12 * scale + 1e-13
    lhs = float((out["dV"] * V.astype(np.float64)).sum())
    rhs = float((out["O"] * dO.astype(np.float64)).sum())
    assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sampling", ["uniform", "rownorm"])
def test_backward_rows_equal_dense(ora, causal, sampling):
    """dQ of selected rows, computed per subproblem without dense weights (for large n), equals the dense
    backward's rows."""
    n, d = 512, 16
    Q, K, V = rand_qkv(n, d, 65)
    dO = np.random.default_rng(10).standard_normal((n, d)).astype(np.float32)
    rows = np.array([0, 1, 63, 64, 200, 255, 256, 300, 511])
    kw = dict(block=32, m=24, r=5, causal=causal, base=64, seed=6, bh=3, sampling=sampling)
    dense = ora.backward(Q, K, V, dO, **kw)["dQ"][rows]
    np.testing.assert_allclose(ora.backward_rows(Q, K, V, dO, rows, **kw), dense, rtol=1e-10, atol=1e-12)
