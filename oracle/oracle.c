/*
 * oracle.c -- plain, slow CPU reference of the HyperAttention forward pass and its gradients.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's CPU-baseline
 * leg load this library. It shares no code, header, table or helper with the CUDA library and it
 * never reads anything the CUDA library produced: every input it sees is the seeded synthetic data
 * and the seed itself, from which it draws its own random projections and column samples.
 *
 * What it computes follows "HyperAttention: Long-context Attention in Near-Linear Time":
 *   - research-map summary page, section "Approach": large entries are found with Hamming-sorted LSH
 *     blocks; the softmax normaliser D is estimated from exact masked row sums plus uniform column
 *     sampling; the product with V is approximated from sampled columns;
 *   - the same page's one-line summary: a recursive causal-masking extension;
 *   - the same page, "Limitations": the causal variant partitions and merges;
 *   - the OpenReview abstract: LSH finds the large entries.
 * The pages give the method in outline only. Every step they leave open is fixed below by the plainest
 * reading; each such reading is marked READING and listed in the design notes.
 *
 * Precision: attention arithmetic is double. The one floating-point decision that produces an integer
 * (the sign of a projection, which sets a hash bit) is taken in fp32 with a sequential fused
 * multiply-add over the row in index order, the precision of the GPU kernel, so both sides take the same
 * decision (see hash_row).
 *
 * Random draws: Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
 * SC'11), Box-Muller for normals, Lemire's multiply-shift with rejection for bounded integers, and
 * Floyd's algorithm for a uniform m-subset. Written here from those publications.
 *
 * Build: cc -O2 -fopenmp -ffp-contract=off -shared -fPIC oracle.c -o liboracle.so -lm
 * (-ffp-contract=off: no multiply-add is fused unless written as fma/fmaf.)
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

#define ORA_OK 0
#define ORA_EINVAL (-1)
#define ORA_ENOMEM (-4)

/* ------------------------------------------------------------------------------------------------ */
/* Philox4x64-10 (SC'11, section 3): round function on a 4-word counter under a 2-word key.           */
/* ------------------------------------------------------------------------------------------------ */

static const uint64_t PHILOX_M0 = 0xD2E7470EE14C6C93ULL;   /* multipliers for 4x64 */
static const uint64_t PHILOX_M1 = 0xCA5A826395121157ULL;
static const uint64_t PHILOX_W0 = 0x9E3779B97F4A7C15ULL;   /* Weyl key increments: golden ratio, sqrt(3)-1 */
static const uint64_t PHILOX_W1 = 0xBB67AE8584CAA73BULL;

void ora_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4])
{
    uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        unsigned __int128 p0 = (unsigned __int128)PHILOX_M0 * x0;
        unsigned __int128 p1 = (unsigned __int128)PHILOX_M1 * x2;
        uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        uint64_t y0 = hi1 ^ x1 ^ k0;
        uint64_t y1 = lo1;
        uint64_t y2 = hi0 ^ x3 ^ k1;
        uint64_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Stream tags (second key word) that separate the two kinds of draws made from one seed. */
#define TAG_PROJECTION 1ULL
#define TAG_SAMPLES 2ULL

/* ------------------------------------------------------------------------------------------------ */
/* Projection matrix P (d x r, row-major P[k*r + j]) with i.i.d. N(0,1) entries.                      */
/* "Approach": sortLSH hashes with random Gaussian directions. READING: one P per call, shared by Q    */
/* and K (they must share it for matching buckets), by all heads, the batch and all causal nodes.     */
/* Entry e = k*r + j uses Philox counter (e,0,0,0) under key (seed, TAG_PROJECTION); words 0 and 1     */
/* give two uniforms and Box-Muller (cosine branch) gives the normal, computed in double and rounded  */
/* to float.                                                                                          */
/* ------------------------------------------------------------------------------------------------ */

void ora_draw_projection(uint64_t seed, int d, int r, float *P)
{
    const uint64_t key[2] = {seed, TAG_PROJECTION};
    const double two_pi = 6.283185307179586476925286766559;
    const double inv2_53 = 1.0 / 9007199254740992.0;   /* 2^-53 */
    for (int64_t e = 0; e < (int64_t)d * r; ++e) {
        uint64_t ctr[4] = {(uint64_t)e, 0, 0, 0}, w[4];
        ora_philox4x64_10(ctr, key, w);
        double u1 = (double)((w[0] >> 11) + 1) * inv2_53;   /* (0, 1] */
        double u2 = (double)(w[1] >> 11) * inv2_53;         /* [0, 1) */
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        P[e] = (float)z;
    }
}

/* ------------------------------------------------------------------------------------------------ */
/* Column samples. "Approach": uniform column sampling estimates D. READING: m distinct indices drawn */
/* uniformly from [0, N) (without replacement), shared by every query of one (batch*head, node), and  */
/* returned in ascending order. node = 1 for the non-causal problem; in the causal recursion the      */
/* nodes are numbered in heap order (root 1, children 2i and 2i+1).                                   */
/* Word t of the stream for (bh, node) is word t%4 of Philox(counter (t/4, node, bh, 0),               */
/* key (seed, TAG_SAMPLES)).                                                                          */
/* ------------------------------------------------------------------------------------------------ */

typedef struct {
    uint64_t key[2];
    uint64_t bh, node;
    uint64_t t;          /* index of the next word */
    uint64_t buf[4];
} word_stream;

static uint64_t next_word(word_stream *s)
{
    if ((s->t & 3) == 0) {
        uint64_t ctr[4] = {s->t >> 2, s->node, s->bh, 0};
        ora_philox4x64_10(ctr, s->key, s->buf);
    }
    uint64_t w = s->buf[s->t & 3];
    s->t++;
    return w;
}

/* Uniform integer in [0, range), range >= 1: Lemire, "Fast Random Integer Generation in an Interval"
 * (ACM TOMACS 2019), multiply-shift with rejection of the biased low products. */
static uint64_t bounded(word_stream *s, uint64_t range)
{
    uint64_t x = next_word(s);
    unsigned __int128 mm = (unsigned __int128)x * range;
    uint64_t low = (uint64_t)mm;
    if (low < range) {
        uint64_t threshold = (0 - range) % range;
        while (low < threshold) {
            x = next_word(s);
            mm = (unsigned __int128)x * range;
            low = (uint64_t)mm;
        }
    }
    return (uint64_t)(mm >> 64);
}

int ora_draw_samples(uint64_t seed, int64_t bh, int64_t node, int64_t N, int m, int32_t *S)
{
    if (m < 0 || N < 0 || m > N) return ORA_EINVAL;
    if (m == 0) return ORA_OK;
    unsigned char *chosen = (unsigned char *)calloc((size_t)N, 1);
    if (!chosen) return ORA_ENOMEM;
    word_stream s;
    memset(&s, 0, sizeof s);
    s.key[0] = seed; s.key[1] = TAG_SAMPLES; s.bh = (uint64_t)bh; s.node = (uint64_t)node;
    /* Floyd's algorithm (Bentley & Floyd, CACM 1987): for j = N-m .. N-1 draw t in [0, j]; take t if
     * it is new, else take j. Every m-subset comes out with equal probability. */
    for (int64_t j = N - m; j < N; ++j) {
        int64_t t = (int64_t)bounded(&s, (uint64_t)j + 1);
        if (chosen[t]) chosen[j] = 1; else chosen[t] = 1;
    }
    int64_t c = 0;
    for (int64_t i = 0; i < N; ++i)
        if (chosen[i]) S[c++] = (int32_t)i;
    free(chosen);
    return c == m ? ORA_OK : ORA_EINVAL;
}

/* ------------------------------------------------------------------------------------------------ */
/* sortLSH hash. "Approach" / "Experimental setup": Hamming-sorted LSH. For a row x: bit j = [x.P_j > 0]*/
/* (READING: an exact zero gives bit 0; projection j is bit j, least significant first). The r-bit    */
/* code h is read as a Gray codeword and its rank is the inverse Gray code, so buckets with adjacent  */
/* ranks differ in exactly one hash bit (Hamming distance 1).                                         */
/* ------------------------------------------------------------------------------------------------ */

uint32_t ora_gray_rank(uint32_t h)
{
    /* inverse of g = b ^ (b >> 1):  b = g ^ (g >> 1) ^ (g >> 2) ^ ... */
    uint32_t b = 0;
    for (uint32_t s = h; s != 0; s >>= 1) b ^= s;
    return b;
}

/* One row: the projections x.P_j and the squared norm are each a sequential fp32 fused multiply-add
 * chain over k = 0..d-1 starting from +0. A projection is "near zero" when |x.P_j| < 1e-4 * ||x||_2
 * (fp32, sqrtf correctly rounded); such rows are reported. */
static void hash_row(const float *x, int d, const float *P, int r, uint16_t *rank, uint8_t *near)
{
    float nrm2 = 0.0f;
    for (int k = 0; k < d; ++k) nrm2 = fmaf(x[k], x[k], nrm2);
    const float thr = 1e-4f * sqrtf(nrm2);
    uint32_t h = 0;
    uint8_t flag = 0;
    for (int j = 0; j < r; ++j) {
        float p = 0.0f;
        for (int k = 0; k < d; ++k) p = fmaf(x[k], P[(int64_t)k * r + j], p);
        if (p > 0.0f) h |= 1u << j;
        if (fabsf(p) < thr) flag = 1;
    }
    *rank = (uint16_t)ora_gray_rank(h);
    *near = flag;
}

int ora_hash_rows(const float *X, int64_t rows, int d, const float *P, int r, uint16_t *rank, uint8_t *near)
{
    if (r < 0 || r > 16 || d <= 0 || rows < 0) return ORA_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) hash_row(X + i * d, d, P, r, rank + i, near + i);
    return ORA_OK;
}

/* ------------------------------------------------------------------------------------------------ */
/* Sort by bucket rank. READING: stable, ties by original index ascending, so the order is unique.    */
/* perm[p] = index (0..N-1) of the row at sorted position p.                                         */
/* ------------------------------------------------------------------------------------------------ */

typedef struct { uint32_t rank; int32_t idx; } rank_idx;

static int cmp_rank_idx(const void *a, const void *b)
{
    const rank_idx *x = (const rank_idx *)a, *y = (const rank_idx *)b;
    if (x->rank != y->rank) return x->rank < y->rank ? -1 : 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

int ora_sort_segment(const uint16_t *rank, int64_t N, int32_t *perm)
{
    rank_idx *a = (rank_idx *)malloc(sizeof(rank_idx) * (size_t)(N > 0 ? N : 1));
    if (!a) return ORA_ENOMEM;
    for (int64_t i = 0; i < N; ++i) { a[i].rank = rank[i]; a[i].idx = (int32_t)i; }
    qsort(a, (size_t)N, sizeof(rank_idx), cmp_rank_idx);
    for (int64_t p = 0; p < N; ++p) perm[p] = a[p].idx;
    free(a);
    return ORA_OK;
}

/* ------------------------------------------------------------------------------------------------ */
/* Attention parts. A part of a query row is the pair (O, L): O = N/D, L = log D, with                */
/* N = sum_k w_k exp(q.k) v_k and D = sum_k w_k exp(q.k) over the part's keys and weights. Parts of   */
/* one row merge exactly: D = sum_i exp(L_i), O = sum_i exp(L_i - L) O_i.                            */
/* READING: no softmax scale inside exp (the inputs are pre-scaled by d^-1/4; the interface has no    */
/* scale argument).                                                                                   */
/* ------------------------------------------------------------------------------------------------ */

static double dot_fd(const float *a, const float *b, int d)
{
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += (double)a[k] * (double)b[k];
    return s;
}

/* merge part (Op, Lp) into the running (O, L) of one row; L = -inf means "empty". */
static void merge_part(double *O, double *L, const double *Op, double Lp, int d)
{
    if (Lp == -INFINITY) return;
    if (*L == -INFINITY) {
        for (int k = 0; k < d; ++k) O[k] = Op[k];
        *L = Lp;
        return;
    }
    double mx = *L > Lp ? *L : Lp;
    double a = exp(*L - mx), b = exp(Lp - mx);
    for (int k = 0; k < d; ++k) O[k] = (a * O[k] + b * Op[k]) / (a + b);
    *L = mx + log(a + b);
}

/*
 * Row-norm samples of one problem ("Approach": the product with values via row-norm sampling).
 * READING: m draws, independent and with replacement, of a key row j with probability p_j = ||v_j||^2 /
 * sum_j' ||v_j'||^2 over the problem's N value rows; draw t carries the weight 1/(m p_j), so that the sum of
 * weight * a_j v_j over the draws is an unbiased estimate of sum_j a_j v_j. The squared norms are sequential
 * fp32 fused multiply-adds over k = 0..d-1 from +0 (a decision taken in fp32, the same on both sides); draw t
 * uses u_t = (w >> 11) * 2^-53 with w = output word t mod 4 of Philox4x64-10 under key (seed, 3) at counter
 * (t / 4, node, bh, 0), and picks the smallest j whose cumulative sum (double, index order) exceeds u_t times
 * the total. logw[t] = log(1 / (m p_j)). If every norm is zero, S[t] = -1 (no draw).
 */
int ora_draw_rownorm(uint64_t seed, int64_t bh, int64_t node, const float *Vk, int64_t N, int d, int m,
                     int32_t *S, double *logw)
{
    if (N <= 0 || m < 0) return ORA_EINVAL;
    if (m == 0) return ORA_OK;
    double *cdf = (double *)malloc(sizeof(double) * (size_t)N);
    float *nrm = (float *)malloc(sizeof(float) * (size_t)N);
    if (!cdf || !nrm) { free(cdf); free(nrm); return ORA_ENOMEM; }
    double run = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        float a = 0.0f;
        for (int k = 0; k < d; ++k) a = fmaf(Vk[j * d + k], Vk[j * d + k], a);
        nrm[j] = a;
        run += (double)a;
        cdf[j] = run;
    }
    const double total = run;
    uint64_t key[2] = {seed, 3}, out4[4] = {0, 0, 0, 0};
    for (int t = 0; t < m; ++t) {
        if ((t & 3) == 0) {
            uint64_t ctr[4] = {(uint64_t)(t / 4), (uint64_t)node, (uint64_t)bh, 0};
            ora_philox4x64_10(ctr, key, out4);
        }
        if (total <= 0.0) { S[t] = -1; logw[t] = -INFINITY; continue; }
        const double u = (double)(out4[t & 3] >> 11) * 0x1.0p-53;
        const double target = u * total;
        int64_t lo = 0, hi = N - 1;            /* smallest j with cdf[j] > target */
        while (lo < hi) {
            int64_t mid = lo + (hi - lo) / 2;
            if (cdf[mid] > target) hi = mid; else lo = mid + 1;
        }
        S[t] = (int32_t)lo;
        logw[t] = log(total / ((double)m * (double)nrm[lo]));
    }
    free(cdf); free(nrm);
    return ORA_OK;
}

/*
 * The non-causal HyperAttention problem on N queries and N keys ("Approach"):
 *   1. sort queries and keys by hash rank (rq, rk);
 *   2. sorted query block i = positions [i*b', (i+1)*b'), b' = min(block, N) (READING: aligned diagonal
 *      blocks; query block i pairs with key block i);
 *   3. block part: exact sums over the key block -> (N1, D1) ("exact masked row sums");
 *   4. sample part: over the sampled columns s whose key lies outside the query's block, weight N/m
 *      (READING: in-block columns are already counted exactly, so they are dropped from the sample,
 *      which keeps the estimate unbiased for the out-of-block mass; the product with V reuses the same
 *      uniform samples) -> (N2, D2);
 *   5. D~ = D1 + D2, O = (N1 + N2) / D~.
 * Output for each selected query (local index qsel[t]): O (d doubles), L = log D~, and, if not NULL,
 * L1 = log D1 and L2 = log D2 (-inf when there are no sampled columns left).
 */
static int hyper_subproblem(const float *Qr, const float *Kr, const float *Vr, int64_t N, int d,
                            const uint16_t *rq, const uint16_t *rk, int64_t block, const int32_t *S, int m,
                            const int32_t *Srn, const double *lwrn,
                            const int64_t *qsel, int64_t nsel,
                            double *Oout, double *Lout, double *L1out, double *L2out)
{
    int64_t bp = block < N ? block : N;
    if (bp <= 0 || N % bp != 0) return ORA_EINVAL;
    int32_t *permQ = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t *permK = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int64_t *posQ = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int64_t *posK = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    if (!permQ || !permK || !posQ || !posK) { free(permQ); free(permK); free(posQ); free(posK); return ORA_ENOMEM; }
    int rc = ora_sort_segment(rq, N, permQ);
    if (rc == ORA_OK) rc = ora_sort_segment(rk, N, permK);
    if (rc != ORA_OK) { free(permQ); free(permK); free(posQ); free(posK); return rc; }
    for (int64_t p = 0; p < N; ++p) { posQ[permQ[p]] = p; posK[permK[p]] = p; }
    const double wsamp = m > 0 ? (double)N / (double)m : 0.0;

#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)(bp + 2 * m + 1));
        double *n1 = (double *)malloc(sizeof(double) * (size_t)d);
        double *n2 = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < nsel; ++t) {
            int64_t q = qsel[t];
            int64_t i = posQ[q] / bp;
            const float *qv = Qr + q * d;
            /* scores: block keys, then the sampled keys outside the block */
            double mx = -INFINITY;
            for (int64_t j = 0; j < bp; ++j) {
                sc[j] = dot_fd(qv, Kr + (int64_t)permK[i * bp + j] * d, d);
                if (sc[j] > mx) mx = sc[j];
            }
            for (int u = 0; u < m; ++u) {
                int64_t s = S[u];
                if (posK[s] / bp == i) { sc[bp + u] = -INFINITY; continue; }
                sc[bp + u] = dot_fd(qv, Kr + s * d, d);
                if (sc[bp + u] > mx) mx = sc[bp + u];
            }
            /* row-norm variant: the numerator's sampled part comes from the row-norm draws */
            for (int u = 0; Srn && u < m; ++u) {
                int64_t s = Srn[u];
                if (s < 0 || posK[s] / bp == i) { sc[bp + m + u] = -INFINITY; continue; }
                sc[bp + m + u] = dot_fd(qv, Kr + s * d, d);
                if (sc[bp + m + u] > mx) mx = sc[bp + m + u];
            }
            double d1 = 0.0, d2 = 0.0;
            for (int k = 0; k < d; ++k) { n1[k] = 0.0; n2[k] = 0.0; }
            for (int64_t j = 0; j < bp; ++j) {
                double e = exp(sc[j] - mx);
                const float *v = Vr + (int64_t)permK[i * bp + j] * d;
                d1 += e;
                for (int k = 0; k < d; ++k) n1[k] += e * (double)v[k];
            }
            for (int u = 0; u < m; ++u) {
                if (sc[bp + u] == -INFINITY) continue;
                double e = wsamp * exp(sc[bp + u] - mx);
                const float *v = Vr + (int64_t)S[u] * d;
                d2 += e;
                if (!Srn)
                    for (int k = 0; k < d; ++k) n2[k] += e * (double)v[k];
            }
            for (int u = 0; Srn && u < m; ++u) {
                if (sc[bp + m + u] == -INFINITY) continue;
                double e = exp(sc[bp + m + u] - mx + lwrn[u]);
                const float *v = Vr + (int64_t)Srn[u] * d;
                for (int k = 0; k < d; ++k) n2[k] += e * (double)v[k];
            }
            double dt = d1 + d2;
            for (int k = 0; k < d; ++k) Oout[t * d + k] = (n1[k] + n2[k]) / dt;
            Lout[t] = mx + log(dt);
            if (L1out) L1out[t] = mx + log(d1);
            if (L2out) L2out[t] = d2 > 0.0 ? mx + log(d2) : -INFINITY;
        }
        free(sc); free(n1); free(n2);
    }
    free(permQ); free(permK); free(posQ); free(posK);
    return ORA_OK;
}

/* Exact causal softmax attention of one query row q over keys [lo, q] (inclusive). */
static void exact_causal_row(const float *Q, const float *K, const float *V, int d, int64_t lo, int64_t q,
                             double *sc, double *O, double *L)
{
    double mx = -INFINITY;
    for (int64_t k = lo; k <= q; ++k) {
        sc[k - lo] = dot_fd(Q + q * d, K + k * d, d);
        if (sc[k - lo] > mx) mx = sc[k - lo];
    }
    double den = 0.0;
    for (int c = 0; c < d; ++c) O[c] = 0.0;
    for (int64_t k = lo; k <= q; ++k) {
        double e = exp(sc[k - lo] - mx);
        den += e;
        for (int c = 0; c < d; ++c) O[c] += e * (double)V[k * d + c];
    }
    for (int c = 0; c < d; ++c) O[c] /= den;
    *L = mx + log(den);
}

static int valid_causal_shape(int64_t n, int64_t base)
{
    if (base <= 0) return 0;
    if (n <= base) return 1;
    int64_t x = n;
    while (x > base) { if (x & 1) return 0; x >>= 1; }
    return x == base;
}

/*
 * Full forward for one (batch*head) problem bh of n rows.
 * causal = 0: the non-causal problem above on all n rows (node 1).
 * causal = 1: the recursive causal extension (summary page, one-line summary and "Limitations").
 *   READING: a node covering rows [s, s+len) with len > base splits into the causal upper-left half
 *   [s, s+len/2), the causal lower-right half [s+len/2, s+len) and the non-causal off-diagonal block
 *   (queries of the lower half against keys/values of the upper half, N = len/2, samples of that node);
 *   a node with len <= base is exact causal attention (key index <= query index). Every query row's parts
 *   are merged in log space. Requires n = base * 2^L.
 * rows/nrows: the original query rows to produce (rows == NULL: all rows, in order).
 * O: nrows x d doubles; L (may be NULL): log D~ per produced row.
 * For causal = 0 only: L1, L2 (may be NULL) per produced row, as in hyper_subproblem.
 * rank_out (may be NULL): 2n ranks (Q rows then K rows); near_out (may be NULL): 2n flags.
 */
/* sampling 0: the product with V reuses the uniform samples; 1: it uses row-norm samples (ora_draw_rownorm). */
int ora_forward_sampling(const float *Q, const float *K, const float *V, int64_t n, int d, int64_t block, int m,
                         int r, int causal, int64_t base, uint64_t seed, int64_t bh,
                         const int64_t *rows, int64_t nrows,
                         double *O, double *L, double *L1, double *L2, uint16_t *rank_out, uint8_t *near_out,
                         int sampling);

int ora_forward(const float *Q, const float *K, const float *V, int64_t n, int d, int64_t block, int m, int r,
                int causal, int64_t base, uint64_t seed, int64_t bh,
                const int64_t *rows, int64_t nrows,
                double *O, double *L, double *L1, double *L2, uint16_t *rank_out, uint8_t *near_out)
{
    return ora_forward_sampling(Q, K, V, n, d, block, m, r, causal, base, seed, bh, rows, nrows, O, L, L1, L2,
                                rank_out, near_out, 0);
}

int ora_forward_sampling(const float *Q, const float *K, const float *V, int64_t n, int d, int64_t block, int m,
                         int r, int causal, int64_t base, uint64_t seed, int64_t bh,
                         const int64_t *rows, int64_t nrows,
                         double *O, double *L, double *L1, double *L2, uint16_t *rank_out, uint8_t *near_out,
                         int sampling)
{
    if (sampling != 0 && sampling != 1) return ORA_EINVAL;
    if (n <= 0 || d <= 0 || block <= 0 || m < 0 || r < 0 || r > 16) return ORA_EINVAL;
    if (causal && !valid_causal_shape(n, base)) return ORA_EINVAL;
    int64_t nsel = rows ? nrows : n;
    int rc = ORA_OK;
    float *P = (float *)malloc(sizeof(float) * (size_t)(d * (r > 0 ? r : 1)));
    uint16_t *rank = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(2 * n));
    uint8_t *near = (uint8_t *)malloc((size_t)(2 * n));
    int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nsel > 0 ? nsel : 1));
    double *Lloc = (double *)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
    if (!P || !rank || !near || !sel || !Lloc) { rc = ORA_ENOMEM; goto out; }
    for (int64_t t = 0; t < nsel; ++t) sel[t] = rows ? rows[t] : t;
    for (int64_t t = 0; t < nsel; ++t) if (sel[t] < 0 || sel[t] >= n) { rc = ORA_EINVAL; goto out; }

    ora_draw_projection(seed, d, r, P);
    ora_hash_rows(Q, n, d, P, r, rank, near);
    ora_hash_rows(K, n, d, P, r, rank + n, near + n);
    if (rank_out) memcpy(rank_out, rank, sizeof(uint16_t) * (size_t)(2 * n));
    if (near_out) memcpy(near_out, near, (size_t)(2 * n));

    if (!causal) {
        if (m > n) { rc = ORA_EINVAL; goto out; }
        int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
        int32_t *Srn = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
        double *lw = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
        if (!S || !Srn || !lw) { free(S); free(Srn); free(lw); rc = ORA_ENOMEM; goto out; }
        rc = ora_draw_samples(seed, bh, 1, n, m, S);
        if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, 1, V, n, d, m, Srn, lw);
        if (rc == ORA_OK)
            rc = hyper_subproblem(Q, K, V, n, d, rank, rank + n, block, S, m, sampling ? Srn : NULL,
                                  sampling ? lw : NULL, sel, nsel, O, L ? L : Lloc, L1, L2);
        free(S); free(Srn); free(lw);
        goto out;
    }

    /* causal: running (O, L) per produced row, starting empty */
    for (int64_t t = 0; t < nsel; ++t) Lloc[t] = -INFINITY;
    {
        /* exact causal leaves: row q lies in leaf [q - q % base', ...), base' = min(base, n) */
        int64_t leaf = base < n ? base : n;
#pragma omp parallel
        {
            double *sc = (double *)malloc(sizeof(double) * (size_t)leaf);
            double *Op = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < nsel; ++t) {
                int64_t q = sel[t];
                double Lp;
                exact_causal_row(Q, K, V, d, q - q % leaf, q, sc, Op, &Lp);
                merge_part(O + t * d, &Lloc[t], Op, Lp, d);
            }
            free(sc); free(Op);
        }
        /* internal nodes, level by level: at level l (1-based) nodes have len = n >> (l-1), heap ids
         * 2^(l-1) + j for node j = 0 .. 2^(l-1)-1 covering rows [j*len, (j+1)*len). */
        for (int64_t len = n; len > leaf && rc == ORA_OK; len >>= 1) {
            int64_t half = len / 2, nodes = n / len;
            for (int64_t j = 0; j < nodes && rc == ORA_OK; ++j) {
                int64_t s0 = j * len, node = nodes + j;
                /* produced rows that are queries of this node's off-diagonal block */
                int64_t cnt = 0;
                for (int64_t t = 0; t < nsel; ++t) if (sel[t] >= s0 + half && sel[t] < s0 + len) ++cnt;
                if (cnt == 0) continue;
                int64_t *lq = (int64_t *)malloc(sizeof(int64_t) * (size_t)cnt);
                int64_t *ts = (int64_t *)malloc(sizeof(int64_t) * (size_t)cnt);
                double *Op = (double *)malloc(sizeof(double) * (size_t)(cnt * d));
                double *Lp = (double *)malloc(sizeof(double) * (size_t)cnt);
                int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
                int32_t *Srn = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
                double *lw = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
                if (!lq || !ts || !Op || !Lp || !S || !Srn || !lw) rc = ORA_ENOMEM;
                if (rc == ORA_OK && m > half) rc = ORA_EINVAL;
                if (rc == ORA_OK) {
                    int64_t c = 0;
                    for (int64_t t = 0; t < nsel; ++t)
                        if (sel[t] >= s0 + half && sel[t] < s0 + len) { lq[c] = sel[t] - (s0 + half); ts[c] = t; ++c; }
                    rc = ora_draw_samples(seed, bh, node, half, m, S);
                    if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, node, V + s0 * d, half, d, m, Srn, lw);
                }
                if (rc == ORA_OK)
                    rc = hyper_subproblem(Q + (s0 + half) * d, K + s0 * d, V + s0 * d, half, d,
                                          rank + s0 + half, rank + n + s0, block, S, m, sampling ? Srn : NULL,
                                          sampling ? lw : NULL, lq, cnt, Op, Lp, NULL, NULL);
                if (rc == ORA_OK)
                    for (int64_t c = 0; c < cnt; ++c) merge_part(O + ts[c] * d, &Lloc[ts[c]], Op + c * d, Lp[c], d);
                free(lq); free(ts); free(Op); free(Lp); free(S); free(Srn); free(lw);
            }
        }
    }
    if (L && rc == ORA_OK) memcpy(L, Lloc, sizeof(double) * (size_t)nsel);
out:
    free(P); free(rank); free(near); free(sel); free(Lloc);
    return rc;
}

/*
 * Sorted permutations of one level, for comparing the GPU's sort bit for bit.
 * level 0: the non-causal problem, one Q segment and one K segment of n rows.
 * level l >= 1 (causal): for each node j at that level (len = n >> (l-1)), the Q segment is the lower
 * half [j*len + len/2, (j+1)*len) and the K segment the upper half [j*len, j*len + len/2); the segments
 * are concatenated in node order, each holding indices local to its segment. rank: 2n ranks (Q then K).
 * permQ, permK: n (level 0) or n/2 (level >= 1) entries each.
 */
int ora_level_perms(const uint16_t *rank, int64_t n, int level, int32_t *permQ, int32_t *permK)
{
    if (level == 0) {
        int rc = ora_sort_segment(rank, n, permQ);
        return rc != ORA_OK ? rc : ora_sort_segment(rank + n, n, permK);
    }
    int64_t len = n >> (level - 1), half = len / 2, nodes = n / len;
    for (int64_t j = 0; j < nodes; ++j) {
        int rc = ora_sort_segment(rank + j * len + half, half, permQ + j * half);
        if (rc == ORA_OK) rc = ora_sort_segment(rank + n + j * len, half, permK + j * half);
        if (rc != ORA_OK) return rc;
    }
    return ORA_OK;
}

/* Exact softmax attention (the textbook definition), for the pins and the approximation error:
 * O_q = sum_k exp(q.k) v_k / sum_k exp(q.k) over all keys (causal = 0) or keys k <= q (causal = 1). */
int ora_exact_attention(const float *Q, const float *K, const float *V, int64_t n, int d, int causal,
                        const int64_t *rows, int64_t nrows, double *O)
{
    int64_t nsel = rows ? nrows : n;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < nsel; ++t) {
            int64_t q = rows ? rows[t] : t;
            int64_t hi = causal ? q : n - 1;
            double mx = -INFINITY, den = 0.0;
            for (int64_t k = 0; k <= hi; ++k) {
                sc[k] = dot_fd(Q + q * d, K + k * d, d);
                if (sc[k] > mx) mx = sc[k];
            }
            double *o = O + t * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t k = 0; k <= hi; ++k) {
                double e = exp(sc[k] - mx);
                den += e;
                for (int c = 0; c < d; ++c) o[c] += e * (double)V[k * d + c];
            }
            for (int c = 0; c < d; ++c) o[c] /= den;
        }
        free(sc);
    }
    return ORA_OK;
}

/* Hardness diagnostics of one (non-causal) problem ("HyperAttention: Long-context Attention in Near-Linear
 * Time", research-map summary, "Approach", "Key results", "Limitations", and the abstract page: the guarantee
 * rests on the max column norm of the normalised attention matrix D^-1 A and on the ratio of row norms of A
 * once its large entries are removed).
 * READING (alpha): alpha = n * max_{j >= first_col} sum_i W_ij^2 with W = D^-1 A, A_ij = exp(q_i . k_j); it is
 *   1 for uniform attention and n^2 when every row puts all its weight on one column. first_col > 0 drops the
 *   first columns (the pages drop 32 sink-like columns for one model).
 * READING (kappa): the large entries are the ones the method computes exactly, i.e. the aligned blocks of the
 *   sortLSH order (block b' = min(block, n), ranks from this oracle's hash, stable sort). Row norm = row sum
 *   (the quantity the normaliser estimate needs). kappa = max_i R_i / min_i R_i with R_i = sum of A_ij over
 *   the columns outside row i's block; 0/0 gives NaN and x/0 gives +inf.
 * Everything in double precision, in the order of the definitions. */
int ora_diagnostics(const float *Q, const float *K, int64_t n, int d, int64_t block, int r, uint64_t seed,
                    int64_t first_col, double *alpha_out, double *kappa_out)
{
    if (n <= 0 || d <= 0 || block <= 0 || r < 0 || r > 16 || first_col < 0 || first_col >= n) return ORA_EINVAL;
    const int64_t bp = block < n ? block : n;
    float *P = (float *)malloc(sizeof(float) * (size_t)(d * (r > 0 ? r : 1)));
    uint16_t *rq = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n), *rk = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n);
    uint8_t *fl = (uint8_t *)malloc((size_t)n);
    int32_t *pq = (int32_t *)malloc(sizeof(int32_t) * (size_t)n), *pk = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int64_t *posq = (int64_t *)malloc(sizeof(int64_t) * (size_t)n), *posk = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
    double *m = (double *)malloc(sizeof(double) * (size_t)n), *D = (double *)malloc(sizeof(double) * (size_t)n);
    double *logR = (double *)malloc(sizeof(double) * (size_t)n), *col = (double *)calloc((size_t)n, sizeof(double));
    if (!P || !rq || !rk || !fl || !pq || !pk || !posq || !posk || !m || !D || !logR || !col) return ORA_ENOMEM;
    if (r > 0) ora_draw_projection(seed, d, r, P);
    ora_hash_rows(Q, n, d, P, r, rq, fl);
    ora_hash_rows(K, n, d, P, r, rk, fl);
    ora_sort_segment(rq, n, pq);
    ora_sort_segment(rk, n, pk);
    for (int64_t p = 0; p < n; ++p) { posq[pq[p]] = p; posk[pk[p]] = p; }
    /* rows: max, normaliser, and the sum outside the row's block (all shifted by the row max) */
    for (int64_t i = 0; i < n; ++i) {
        double mx = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double s = dot_fd(Q + i * d, K + j * d, d);
            if (s > mx) mx = s;
        }
        double den = 0.0, rest = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double e = exp(dot_fd(Q + i * d, K + j * d, d) - mx);
            den += e;
            if (posk[j] / bp != posq[i] / bp) rest += e;
        }
        m[i] = mx;
        D[i] = den;
        logR[i] = rest > 0.0 ? log(rest) + mx : -INFINITY;
    }
    /* columns: squared norms of W = D^-1 A */
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double w = exp(dot_fd(Q + i * d, K + j * d, d) - m[i]) / D[i];
            col[j] += w * w;
        }
    double cmax = 0.0;
    for (int64_t j = first_col; j < n; ++j) if (col[j] > cmax) cmax = col[j];
    *alpha_out = (double)n * cmax;
    double lo = INFINITY, hi = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        if (logR[i] < lo) lo = logR[i];
        if (logR[i] > hi) hi = logR[i];
    }
    if (hi == -INFINITY) *kappa_out = NAN;              /* every row: nothing outside its block */
    else if (lo == -INFINITY) *kappa_out = INFINITY;    /* some rows have nothing outside their block */
    else *kappa_out = exp(hi - lo);
    free(P); free(rq); free(rk); free(fl); free(pq); free(pk); free(posq); free(posk);
    free(m); free(D); free(logR); free(col);
    return ORA_OK;
}

/*
 * Dense weights of one problem, for the backward pass. The forward estimate of every row q is a weighted
 * softmax over the keys: O_q = sum_k Wn[q][k] e^{s_qk} v_k / sum_k Wd[q][k] e^{s_qk}, s_qk = q . k, where
 *   - a key in q's sortLSH block (of a level's subproblem, or of q's exact causal leaf) has Wn = Wd = 1;
 *   - a uniform sample outside the block has Wd = N/m, and Wn = N/m unless the product with V is row-norm
 *     sampled;
 *   - with row-norm sampling, every draw outside the block adds 1/(m p_j) to Wn (draws may repeat).
 * The log-space merges of the causal recursion combine the parts into exactly this form, because the parts'
 * key sets are disjoint. The weights follow the same steps as ora_forward_sampling (same projection, ranks,
 * sorts and draws); the sort permutation and the draws are constants of the forward pass.
 */
static int sub_weights(int64_t n, int64_t N, int64_t q0, int64_t k0, const uint16_t *rq, const uint16_t *rk,
                       int64_t block, const int32_t *S, int m, const int32_t *Srn, const double *lwrn,
                       double *Wn, double *Wd)
{
    int64_t bp = block < N ? block : N;
    if (bp <= 0 || N % bp != 0) return ORA_EINVAL;
    int32_t *permQ = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t *permK = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int64_t *posQ = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int64_t *posK = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int rc = (!permQ || !permK || !posQ || !posK) ? ORA_ENOMEM : ORA_OK;
    if (rc == ORA_OK) rc = ora_sort_segment(rq, N, permQ);
    if (rc == ORA_OK) rc = ora_sort_segment(rk, N, permK);
    if (rc == ORA_OK) {
        for (int64_t p = 0; p < N; ++p) { posQ[permQ[p]] = p; posK[permK[p]] = p; }
        const double w = m > 0 ? (double)N / (double)m : 0.0;
        for (int64_t q = 0; q < N; ++q) {
            const int64_t i = posQ[q] / bp;
            double *wn = Wn + (q0 + q) * n + k0, *wd = Wd + (q0 + q) * n + k0;
            for (int64_t j = 0; j < bp; ++j) {
                const int64_t k = permK[i * bp + j];
                wn[k] += 1.0;
                wd[k] += 1.0;
            }
            for (int u = 0; u < m; ++u) {
                const int64_t k = S[u];
                if (posK[k] / bp == i) continue;
                wd[k] += w;
                if (!Srn) wn[k] += w;
            }
            for (int u = 0; Srn && u < m; ++u) {
                const int64_t k = Srn[u];
                if (k < 0 || posK[k] / bp == i) continue;
                wn[k] += exp(lwrn[u]);
            }
        }
    }
    free(permQ); free(permK); free(posQ); free(posK);
    return rc;
}

int ora_weights(const float *Q, const float *K, const float *V, int64_t n, int d, int64_t block, int m, int r,
                int causal, int64_t base, uint64_t seed, int64_t bh, int sampling, double *Wn, double *Wd)
{
    if (sampling != 0 && sampling != 1) return ORA_EINVAL;
    if (n <= 0 || d <= 0 || block <= 0 || m < 0 || r < 0 || r > 16) return ORA_EINVAL;
    if (causal && !valid_causal_shape(n, base)) return ORA_EINVAL;
    int rc = ORA_OK;
    float *P = (float *)malloc(sizeof(float) * (size_t)(d * (r > 0 ? r : 1)));
    uint16_t *rank = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(2 * n));
    uint8_t *near = (uint8_t *)malloc((size_t)(2 * n));
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
    int32_t *Srn = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
    double *lw = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
    if (!P || !rank || !near || !S || !Srn || !lw) { rc = ORA_ENOMEM; goto out; }
    memset(Wn, 0, sizeof(double) * (size_t)(n * n));
    memset(Wd, 0, sizeof(double) * (size_t)(n * n));
    ora_draw_projection(seed, d, r, P);
    ora_hash_rows(Q, n, d, P, r, rank, near);
    ora_hash_rows(K, n, d, P, r, rank + n, near + n);
    if (!causal) {
        if (m > n) { rc = ORA_EINVAL; goto out; }
        rc = ora_draw_samples(seed, bh, 1, n, m, S);
        if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, 1, V, n, d, m, Srn, lw);
        if (rc == ORA_OK)
            rc = sub_weights(n, n, 0, 0, rank, rank + n, block, S, m, sampling ? Srn : NULL, lw, Wn, Wd);
        goto out;
    }
    {
        const int64_t leaf = base < n ? base : n;
        for (int64_t q = 0; q < n; ++q)
            for (int64_t k = q - q % leaf; k <= q; ++k) { Wn[q * n + k] = 1.0; Wd[q * n + k] = 1.0; }
        for (int64_t len = n; len > leaf && rc == ORA_OK; len >>= 1) {
            const int64_t half = len / 2, nodes = n / len;
            if (m > half) { rc = ORA_EINVAL; break; }
            for (int64_t j = 0; j < nodes && rc == ORA_OK; ++j) {
                const int64_t s0 = j * len, node = nodes + j;
                rc = ora_draw_samples(seed, bh, node, half, m, S);
                if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, node, V + s0 * d, half, d, m, Srn, lw);
                if (rc == ORA_OK)
                    rc = sub_weights(n, half, s0 + half, s0, rank + s0 + half, rank + n + s0, block, S, m,
                                     sampling ? Srn : NULL, lw, Wn, Wd);
            }
        }
    }
out:
    free(P); free(rank); free(near); free(S); free(Srn); free(lw);
    return rc;
}

/*
 * Backward pass of one problem: the gradients of sum_q dO_q . O_q with respect to Q, K and V, with the sort
 * permutations and the draws held fixed (they are constants of the forward pass). With the dense weights
 * above, E_qk = e^{s_qk - L_q} where L_q = log sum_k Wd[q][k] e^{s_qk}, and g_q = dO_q . O_q:
 *   dV_k = sum_q Wn[q][k] E_qk dO_q,
 *   dS_qk = E_qk (Wn[q][k] (dO_q . v_k) - Wd[q][k] g_q),
 *   dQ_q = sum_k dS_qk k_k,   dK_k = sum_q dS_qk q_q.
 * (O_q = N_q / D_q with N_q = sum_k Wn e^{s} v_k and D_q = sum_k Wd e^{s}; differentiate the quotient.) Double
 * precision, dense over all (q, k): for small n. Also returns O and L.
 */
int ora_backward(const float *Q, const float *K, const float *V, const float *dO, int64_t n, int d, int64_t block,
                 int m, int r, int causal, int64_t base, uint64_t seed, int64_t bh, int sampling,
                 double *dQ, double *dK, double *dV, double *O, double *L)
{
    double *Wn = (double *)malloc(sizeof(double) * (size_t)(n * n));
    double *Wd = (double *)malloc(sizeof(double) * (size_t)(n * n));
    double *sc = (double *)malloc(sizeof(double) * (size_t)n);
    if (!Wn || !Wd || !sc) { free(Wn); free(Wd); free(sc); return ORA_ENOMEM; }
    int rc = ora_weights(Q, K, V, n, d, block, m, r, causal, base, seed, bh, sampling, Wn, Wd);
    if (rc == ORA_OK) {
        memset(dQ, 0, sizeof(double) * (size_t)(n * d));
        memset(dK, 0, sizeof(double) * (size_t)(n * d));
        memset(dV, 0, sizeof(double) * (size_t)(n * d));
        for (int64_t q = 0; q < n; ++q) {
            const double *wn = Wn + q * n, *wd = Wd + q * n;
            double mx = -INFINITY;
            for (int64_t k = 0; k < n; ++k) {
                sc[k] = (wn[k] != 0.0 || wd[k] != 0.0) ? dot_fd(Q + q * d, K + k * d, d) : -INFINITY;
                if (sc[k] > mx) mx = sc[k];
            }
            double den = 0.0;
            double *o = O + q * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t k = 0; k < n; ++k) {
                if (sc[k] == -INFINITY) continue;
                const double e = exp(sc[k] - mx);
                den += wd[k] * e;
                for (int c = 0; c < d; ++c) o[c] += wn[k] * e * (double)V[k * d + c];
            }
            for (int c = 0; c < d; ++c) o[c] /= den;
            const double Lq = mx + log(den);
            L[q] = Lq;
            double g = 0.0;
            for (int c = 0; c < d; ++c) g += (double)dO[q * d + c] * o[c];
            for (int64_t k = 0; k < n; ++k) {
                if (sc[k] == -INFINITY) continue;
                const double E = exp(sc[k] - Lq);
                double dov = 0.0;
                for (int c = 0; c < d; ++c) dov += (double)dO[q * d + c] * (double)V[k * d + c];
                const double ds = E * (wn[k] * dov - wd[k] * g);
                for (int c = 0; c < d; ++c) {
                    dV[k * d + c] += wn[k] * E * (double)dO[q * d + c];
                    dQ[q * d + c] += ds * (double)K[k * d + c];
                    dK[k * d + c] += ds * (double)Q[q * d + c];
                }
            }
        }
    }
    free(Wn); free(Wd); free(sc);
    return rc;
}

/*
 * dQ of selected rows only, for problems too large for the dense weights: the same key terms and formula as
 * ora_backward (dS_qk = e^{s_qk - L_q} (Wn (dO_q . v_k) - Wd (dO_q . O_q)), dQ_q = sum_k dS_qk k_k), visited
 * per subproblem like ora_forward_sampling. O_q and L_q come from ora_forward_sampling for the same rows.
 */
static int sub_dq(const float *Qr, const float *Kr, const float *Vr, const float *dOr, int64_t N, int d,
                  const uint16_t *rq, const uint16_t *rk, int64_t block, const int32_t *S, int m, const int32_t *Srn,
                  const double *lwrn, const int64_t *lq, const int64_t *ts, int64_t cnt, const double *L,
                  const double *g, double *dQ)
{
    int64_t bp = block < N ? block : N;
    if (bp <= 0 || N % bp != 0) return ORA_EINVAL;
    int32_t *permQ = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t *permK = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int64_t *posQ = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int64_t *posK = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    int rc = (!permQ || !permK || !posQ || !posK) ? ORA_ENOMEM : ORA_OK;
    if (rc == ORA_OK) rc = ora_sort_segment(rq, N, permQ);
    if (rc == ORA_OK) rc = ora_sort_segment(rk, N, permK);
    if (rc == ORA_OK) {
        for (int64_t p = 0; p < N; ++p) { posQ[permQ[p]] = p; posK[permK[p]] = p; }
        const double lw = m > 0 ? log((double)N / (double)m) : 0.0;
        for (int64_t c = 0; c < cnt; ++c) {
            const int64_t q = lq[c], t = ts[c], i = posQ[q] / bp;
            const float *qv = Qr + q * d, *go = dOr + q * d;
            double *dq = dQ + t * d;
            /* one term: key k with log weights (ln_wn, ln_wd); -INFINITY = weight 0 */
#define ORA_TERM(kk, ln_wn, ln_wd)                                                                            \
            do {                                                                                              \
                const int64_t k_ = (kk);                                                                      \
                const double s_ = dot_fd(qv, Kr + k_ * d, d);                                                 \
                const double en_ = (ln_wn) == -INFINITY ? 0.0 : exp(s_ + (ln_wn) - L[t]);                     \
                const double ed_ = (ln_wd) == -INFINITY ? 0.0 : exp(s_ + (ln_wd) - L[t]);                     \
                const double dov_ = dot_fd(go, Vr + k_ * d, d);                                               \
                const double ds_ = en_ * dov_ - ed_ * g[t];                                                   \
                for (int x = 0; x < d; ++x) dq[x] += ds_ * (double)Kr[k_ * d + x];                            \
            } while (0)
            for (int64_t j = 0; j < bp; ++j) ORA_TERM(permK[i * bp + j], 0.0, 0.0);
            for (int u = 0; u < m; ++u) {
                if (posK[S[u]] / bp == i) continue;
                ORA_TERM(S[u], Srn ? -INFINITY : lw, lw);
            }
            for (int u = 0; Srn && u < m; ++u) {
                if (Srn[u] < 0 || posK[Srn[u]] / bp == i) continue;
                ORA_TERM(Srn[u], lwrn[u], -INFINITY);
            }
#undef ORA_TERM
        }
    }
    free(permQ); free(permK); free(posQ); free(posK);
    return rc;
}

int ora_backward_rows(const float *Q, const float *K, const float *V, const float *dO, int64_t n, int d,
                      int64_t block, int m, int r, int causal, int64_t base, uint64_t seed, int64_t bh, int sampling,
                      const int64_t *rows, int64_t nrows, double *dQ)
{
    if (nrows <= 0) return ORA_EINVAL;
    int rc = ORA_OK;
    double *O = (double *)malloc(sizeof(double) * (size_t)(nrows * d));
    double *L = (double *)malloc(sizeof(double) * (size_t)nrows);
    double *g = (double *)malloc(sizeof(double) * (size_t)nrows);
    float *P = (float *)malloc(sizeof(float) * (size_t)(d * (r > 0 ? r : 1)));
    uint16_t *rank = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(2 * n));
    uint8_t *near = (uint8_t *)malloc((size_t)(2 * n));
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
    int32_t *Srn = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
    double *lw = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
    int64_t *lq = (int64_t *)malloc(sizeof(int64_t) * (size_t)nrows);
    int64_t *ts = (int64_t *)malloc(sizeof(int64_t) * (size_t)nrows);
    if (!O || !L || !g || !P || !rank || !near || !S || !Srn || !lw || !lq || !ts) { rc = ORA_ENOMEM; goto out; }
    rc = ora_forward_sampling(Q, K, V, n, d, block, m, r, causal, base, seed, bh, rows, nrows, O, L, NULL, NULL,
                              rank, near, sampling);
    if (rc != ORA_OK) goto out;
    for (int64_t t = 0; t < nrows; ++t) {
        g[t] = 0.0;
        for (int x = 0; x < d; ++x) g[t] += (double)dO[rows[t] * d + x] * O[t * d + x];
    }
    memset(dQ, 0, sizeof(double) * (size_t)(nrows * d));
    if (!causal) {
        rc = ora_draw_samples(seed, bh, 1, n, m, S);
        if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, 1, V, n, d, m, Srn, lw);
        for (int64_t t = 0; t < nrows; ++t) { lq[t] = rows[t]; ts[t] = t; }
        if (rc == ORA_OK)
            rc = sub_dq(Q, K, V, dO, n, d, rank, rank + n, block, S, m, sampling ? Srn : NULL, lw, lq, ts, nrows, L,
                        g, dQ);
        goto out;
    }
    {
        const int64_t leaf = base < n ? base : n;
        for (int64_t t = 0; t < nrows; ++t) {   /* exact causal leaf: keys q - q % leaf .. q, weight 1 */
            const int64_t q = rows[t];
            for (int64_t k = q - q % leaf; k <= q; ++k) {
                const double s_ = dot_fd(Q + q * d, K + k * d, d);
                const double e_ = exp(s_ - L[t]);
                const double ds_ = e_ * (dot_fd(dO + q * d, V + k * d, d) - g[t]);
                for (int x = 0; x < d; ++x) dQ[t * d + x] += ds_ * (double)K[k * d + x];
            }
        }
        for (int64_t len = n; len > leaf && rc == ORA_OK; len >>= 1) {
            const int64_t half = len / 2, nodes = n / len;
            for (int64_t j = 0; j < nodes && rc == ORA_OK; ++j) {
                const int64_t s0 = j * len, node = nodes + j;
                int64_t cnt = 0;
                for (int64_t t = 0; t < nrows; ++t)
                    if (rows[t] >= s0 + half && rows[t] < s0 + len) { lq[cnt] = rows[t] - (s0 + half); ts[cnt] = t; ++cnt; }
                if (cnt == 0) continue;
                rc = ora_draw_samples(seed, bh, node, half, m, S);
                if (rc == ORA_OK && sampling) rc = ora_draw_rownorm(seed, bh, node, V + s0 * d, half, d, m, Srn, lw);
                if (rc == ORA_OK)
                    rc = sub_dq(Q + (s0 + half) * d, K + s0 * d, V + s0 * d, dO + (s0 + half) * d, half, d,
                                rank + s0 + half, rank + n + s0, block, S, m, sampling ? Srn : NULL, lw, lq, ts, cnt,
                                L, g, dQ);
            }
        }
    }
out:
    free(O); free(L); free(g); free(P); free(rank); free(near); free(S); free(Srn); free(lw); free(lq); free(ts);
    return rc;
}

int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
