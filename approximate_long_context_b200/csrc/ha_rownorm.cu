// ha_rownorm.cu -- row-norm samples for the product with V, drawn on the device.
//
// "HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach"): the
// product of the normalised attention matrix with V can be approximated by sampling rows of V with
// probability proportional to their squared norms. Every sample set (problem b, heap node k; non-causal:
// node 1 over all n rows; causal node k: the key half of the node) takes m draws with replacement, row j
// with p_j = ||v_j||^2 / sum of ||v||^2 over the set's key rows, each draw weighted 1 / (m p_j).
//
//   rownorm_sq_kernel   ||v_j||^2 of every row: sequential fp32 fused multiply-adds over k = 0..d-1, so the
//                       value is the same on every implementation that follows this order
//   chunk_sum_kernel    double sums of 2048-row chunks of every sample set
//   cdf_scan_kernel     inclusive double prefix sums of every set (its cumulative distribution)
//   draw_kernel         one thread per draw t: Philox4x64-10 under key (seed, 3) at counter (t / 4, node,
//                       bh, 0), output word t mod 4, u = (w >> 11) 2^-53; the smallest j with
//                       cdf[j] > u * total (binary search); weight log(total / (m ||v_j||^2)).
// The prefix sums are added in a tree order inside each chunk, not left to right, so a draw can differ from a
// left-to-right sum only when u * total lies within rounding distance of a cumulative sum. A row of zero norm
// is never returned: if rounding makes the search land on one, the draw moves to the nearest row of nonzero
// norm after it (before it at the end of the set). A set whose rows are all zero returns index -1.
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;
constexpr int kChunk = kScanThreads * kScanItems;   // rows per chunk

// Geometry of one sample set: its key rows [start, start + len) of the problem and its cdf offset.
struct SetGeom {
    int64_t start, len, off, heap;
};

__device__ __forceinline__ SetGeom set_of(const RowNormGeom &g, int depth, int64_t idx) {
    SetGeom s;
    if (!g.causal) {
        s.start = 0; s.len = g.n; s.off = 0; s.heap = 1;
    } else {
        const int64_t node_len = g.n >> depth;
        s.len = node_len >> 1;
        s.start = idx * node_len;
        s.off = static_cast<int64_t>(depth) * (g.n >> 1) + idx * s.len;
        s.heap = (int64_t(1) << depth) + idx;
    }
    return s;
}

// chunk slot -> (depth, set index, chunk index)
__device__ __forceinline__ void slot_of(const RowNormGeom &g, int64_t slot, int *depth, int64_t *idx, int64_t *c,
                                        int64_t *cpd) {
    int dp = 0;
    while (dp + 1 < g.depths && slot >= g.slot0[dp + 1]) ++dp;
    const int64_t len = g.causal ? (g.n >> (dp + 1)) : g.n;
    const int64_t per = (len + kChunk - 1) / kChunk;
    const int64_t rem = slot - g.slot0[dp];
    *depth = dp;
    *idx = rem / per;
    *c = rem % per;
    *cpd = per;
}

template <int D, int DT>
__global__ void __launch_bounds__(256) rownorm_sq_kernel(const void *__restrict__ V, int64_t rows,
                                                         float *__restrict__ nrm) {
    const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    float a = 0.0f;
    if (DT == 0) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(V) + r * D);
#pragma unroll
        for (int v = 0; v < D / 8; ++v) {
            const uint4 w = __ldg(p + v);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float lo = __uint_as_float(ws[h] << 16), hi = __uint_as_float(ws[h] & 0xffff0000u);
                a = fmaf(lo, lo, a);
                a = fmaf(hi, hi, a);
            }
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(V) + r * D);
#pragma unroll
        for (int v = 0; v < D / 4; ++v) {
            const float4 w = __ldg(p + v);
            a = fmaf(w.x, w.x, a);
            a = fmaf(w.y, w.y, a);
            a = fmaf(w.z, w.z, a);
            a = fmaf(w.w, w.w, a);
        }
    }
    nrm[r] = a;
}

__device__ __forceinline__ double block_sum(double v, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kScanThreads / 32; ++w) t += red[w];
    return t;   // valid in thread 0
}

__global__ void __launch_bounds__(kScanThreads) chunk_sum_kernel(RowNormGeom g, const float *__restrict__ nrm,
                                                                 double *__restrict__ csum) {
    __shared__ double red[kScanThreads / 32];
    const int64_t b = blockIdx.y, slot = blockIdx.x;
    int depth;
    int64_t idx, c, cpd;
    slot_of(g, slot, &depth, &idx, &c, &cpd);
    const SetGeom s = set_of(g, depth, idx);
    const float *x = nrm + b * g.n + s.start;
    const int64_t j0 = c * kChunk + static_cast<int64_t>(threadIdx.x) * kScanItems;
    double acc = 0.0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k)
        if (j0 + k < s.len) acc += static_cast<double>(x[j0 + k]);
    const double t = block_sum(acc, red);
    if (threadIdx.x == 0) csum[b * g.slots + slot] = t;
}

__global__ void __launch_bounds__(kScanThreads) cdf_scan_kernel(RowNormGeom g, const float *__restrict__ nrm,
                                                                const double *__restrict__ csum,
                                                                double *__restrict__ cdf) {
    __shared__ double wtot[kScanThreads / 32];
    __shared__ double carry_s;
    const int64_t b = blockIdx.y, slot = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int depth;
    int64_t idx, c, cpd;
    slot_of(g, slot, &depth, &idx, &c, &cpd);
    const SetGeom s = set_of(g, depth, idx);
    if (threadIdx.x == 0) {
        double carry = 0.0;
        for (int64_t q = slot - c; q < slot; ++q) carry += csum[b * g.slots + q];
        carry_s = carry;
    }
    const float *x = nrm + b * g.n + s.start;
    const int64_t j0 = c * kChunk + static_cast<int64_t>(threadIdx.x) * kScanItems;
    double pre[kScanItems];
    double run = 0.0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        if (j0 + k < s.len) run += static_cast<double>(x[j0 + k]);
        pre[k] = run;
    }
    // exclusive scan of the thread totals: inside the warp, then over the warps
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    double wexcl = 0.0;
    for (int w = 0; w < warp; ++w) wexcl += wtot[w];
    const double base = carry_s + (wexcl + excl);
    double *out = cdf + b * g.per_prob + s.off;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k)
        if (j0 + k < s.len) out[j0 + k] = base + pre[k];
}

// Philox4x64-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11).
__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3, uint64_t k0,
                                              uint64_t k1, uint64_t out[4]) {
    const uint64_t kMulA = 0xD2E7470EE14C6C93ULL, kMulB = 0xCA5A826395121157ULL;
    const uint64_t kBumpA = 0x9E3779B97F4A7C15ULL, kBumpB = 0xBB67AE8584CAA73BULL;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        if (i) { k0 += kBumpA; k1 += kBumpB; }
        const uint64_t hA = __umul64hi(kMulA, c0), lA = kMulA * c0;
        const uint64_t hB = __umul64hi(kMulB, c2), lB = kMulB * c2;
        const uint64_t n0 = hB ^ c1 ^ k0, n2 = hA ^ c3 ^ k1;
        c0 = n0; c1 = lB; c2 = n2; c3 = lA;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

__global__ void __launch_bounds__(256) draw_kernel(RowNormGeom g, const float *__restrict__ nrm,
                                                   const double *__restrict__ cdf, uint64_t seed, int64_t bh,
                                                   int64_t bh_offset, int32_t *__restrict__ S,
                                                   float *__restrict__ logw) {
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= bh * g.nodes_total * g.m) return;
    const int64_t t = gid % g.m;
    const int64_t set = (gid / g.m) % g.nodes_total;      // heap node - 1
    const int64_t b = gid / (g.m * g.nodes_total);
    int depth = 0;
    while ((int64_t(2) << depth) <= set + 1) ++depth;     // floor(log2(heap node))
    const SetGeom s = set_of(g, depth, set + 1 - (int64_t(1) << depth));
    const double *F = cdf + b * g.per_prob + s.off;
    const float *x = nrm + b * g.n + s.start;
    const double total = F[s.len - 1];
    uint64_t w[4];
    philox4x64_10(static_cast<uint64_t>(t >> 2), static_cast<uint64_t>(s.heap), static_cast<uint64_t>(bh_offset + b),
                  0, seed, 3, w);
    const int64_t o = gid;   // [b][set][t]
    if (!(total > 0.0)) {
        S[o] = -1;
        logw[o] = -INFINITY;
        return;
    }
    const double u = static_cast<double>(w[t & 3] >> 11) * 0x1.0p-53;
    const double target = u * total;
    int64_t lo = 0, hi = s.len - 1;                       // smallest j with F[j] > target
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (F[mid] > target) hi = mid;
        else lo = mid + 1;
    }
    int64_t j = lo;
    while (x[j] == 0.0f && j + 1 < s.len) ++j;
    while (x[j] == 0.0f && j > 0) --j;
    S[o] = static_cast<int32_t>(j);
    logw[o] = static_cast<float>(log(total / (static_cast<double>(g.m) * static_cast<double>(x[j]))));
}

}  // namespace

RowNormGeom rownorm_geometry(int64_t n, int causal, int levels, int m, int64_t nodes_total) {
    RowNormGeom g{};
    g.n = n;
    g.causal = causal;
    g.m = m;
    g.nodes_total = nodes_total;
    g.depths = causal ? levels : 1;
    int64_t slot = 0;
    for (int dp = 0; dp < g.depths; ++dp) {
        g.slot0[dp] = slot;
        const int64_t len = causal ? (n >> (dp + 1)) : n;
        const int64_t sets = causal ? (int64_t(1) << dp) : 1;
        slot += sets * ((len + kChunk - 1) / kChunk);
    }
    g.slot0[g.depths] = slot;
    g.slots = slot;
    g.per_prob = causal ? static_cast<int64_t>(levels) * (n / 2) : n;
    return g;
}

int launch_rownorm_draws(const RowNormGeom &g, const void *V, int dtype, int d, int64_t bh, uint64_t seed,
                         int64_t bh_offset, float *nrm, double *csum, double *cdf, int32_t *S, float *logw,
                         cudaStream_t st) {
    if (g.m <= 0 || g.slots <= 0) return 0;
    if (bh > 65535 || g.slots > 0x7fffffff) return -2;
    const int64_t rows = bh * g.n;
    const unsigned gr = static_cast<unsigned>((rows + 255) / 256);
    if (d == 64 && dtype == 0) rownorm_sq_kernel<64, 0><<<gr, 256, 0, st>>>(V, rows, nrm);
    else if (d == 128 && dtype == 0) rownorm_sq_kernel<128, 0><<<gr, 256, 0, st>>>(V, rows, nrm);
    else if (d == 64) rownorm_sq_kernel<64, 1><<<gr, 256, 0, st>>>(V, rows, nrm);
    else if (d == 128) rownorm_sq_kernel<128, 1><<<gr, 256, 0, st>>>(V, rows, nrm);
    else return -1;
    const dim3 grid(static_cast<unsigned>(g.slots), static_cast<unsigned>(bh));
    chunk_sum_kernel<<<grid, kScanThreads, 0, st>>>(g, nrm, csum);
    cdf_scan_kernel<<<grid, kScanThreads, 0, st>>>(g, nrm, csum, cdf);
    const int64_t draws = bh * g.nodes_total * g.m;
    draw_kernel<<<static_cast<unsigned>((draws + 255) / 256), 256, 0, st>>>(g, nrm, cdf, seed, bh, bh_offset, S, logw);
    return cudaPeekAtLastError() == cudaSuccess ? 4 : -1;
}

}  // namespace ha
