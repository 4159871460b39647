// ha_backward.cu -- gradients of the HyperAttention forward pass (SIMT fp32 kernels).
//
// "HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Key results": the
// speed-ups are quoted for the forward and backward passes). The forward estimate of every row q is a weighted
// softmax over a sparse key set: O_q = sum_k Wn_qk e^{s_qk} v_k / sum_k Wd_qk e^{s_qk}, s_qk = q . k, where
//   * a key in q's sortLSH block (of a level's problem) or in q's exact causal leaf has Wn = Wd = 1,
//   * a uniform sample outside the block has Wd = N/m, and Wn = N/m unless the product with V is row-norm
//     sampled,
//   * a row-norm draw outside the block has Wn = 1/(m p_j) and Wd = 0.
// With the sort and the draws held fixed, L_q = log sum_k Wd_qk e^{s_qk} and g_q = dO_q . O_q:
//   dS_qk = Wn_qk e^{s_qk - L_q} (dO_q . v_k) - Wd_qk e^{s_qk - L_q} g_q,
//   dQ_q += dS_qk k_k,   dK_k += dS_qk q_q,   dV_k += Wn_qk e^{s_qk - L_q} dO_q.
// The forward pass is recomputed first and leaves O (fp32), L and the permutations and draws of every level in
// the workspace. One warp per query row visits the same key set as the forward kernels: the row's dQ stays in
// registers (no other warp of a launch touches it) and dK, dV are accumulated with fp32 atomics.
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kWarps = 8;

template <int DPL>
__device__ __forceinline__ void load_slice(const void *base, int64_t off, int dtype, float (&x)[DPL]) {
#pragma unroll
    for (int c = 0; c < DPL; ++c) x[c] = load_elem(base, off + c, dtype);
}

// One key of row q: log weights ln_wn, ln_wd (-inf: weight 0).
template <int DPL>
struct RowGrad {
    const void *K, *V;
    int dtype;
    float *dK, *dV;
    int64_t head, col;
    float q[DPL], go[DPL], dq[DPL];
    float Lq, gq;

    __device__ void term(int64_t krow, float ln_wn, float ln_wd) {
        float x[DPL];
        load_slice<DPL>(K, head + krow * (DPL * 32) + col, dtype, x);
        float part = 0.0f;
#pragma unroll
        for (int c = 0; c < DPL; ++c) part += q[c] * x[c];
        const float s = warp_sum(part);
        const float pn = ln_wn == -INFINITY ? 0.0f : expf(s + ln_wn - Lq);
        const float pd = ln_wd == -INFINITY ? 0.0f : expf(s + ln_wd - Lq);
        float dov = 0.0f;
        float y[DPL];
        if (ln_wn != -INFINITY) {   // warp-uniform
            load_slice<DPL>(V, head + krow * (DPL * 32) + col, dtype, y);
            float pv = 0.0f;
#pragma unroll
            for (int c = 0; c < DPL; ++c) pv += go[c] * y[c];
            dov = warp_sum(pv);
        }
        const float ds = pn * dov - pd * gq;
        float *dk = dK + head + krow * (DPL * 32) + col;
#pragma unroll
        for (int c = 0; c < DPL; ++c) {
            dq[c] = fmaf(ds, x[c], dq[c]);
            atomicAdd(dk + c, ds * q[c]);
        }
        if (ln_wn != -INFINITY) {
            float *dv = dV + head + krow * (DPL * 32) + col;
#pragma unroll
            for (int c = 0; c < DPL; ++c) atomicAdd(dv + c, pn * go[c]);
        }
    }
};

// g_q = dO_q . O_q, one warp per row
template <int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_rowdot_kernel(const void *__restrict__ dO, int dtype,
                                                                const float *__restrict__ O, int64_t rows,
                                                                float *__restrict__ g) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    float part = 0.0f;
#pragma unroll
    for (int c = 0; c < DPL; ++c) {
        const int64_t i = row * D + lane * DPL + c;
        part += load_elem(dO, i, dtype) * O[i];
    }
    const float t = warp_sum(part);
    if (lane == 0) g[row] = t;
}

// The key terms of one level (the same key sets and weights as the forward level kernels).
template <int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_level_kernel(
    Level lv, const void *__restrict__ Q, const void *__restrict__ K, const void *__restrict__ V,
    const void *__restrict__ dO, int dtype, const int32_t *__restrict__ perm, const int32_t *__restrict__ inv,
    const int32_t *__restrict__ S, int m, int64_t nodes_total, const int32_t *__restrict__ Srn,
    const float *__restrict__ lwrn, const float *__restrict__ L, const float *__restrict__ g, float *dQ, float *dK,
    float *dV) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t N = lv.seg_len;
    if (wg >= lv.bh * lv.nodes * N) return;
    const int64_t prob = wg / N, p = wg % N;
    const int64_t bhi = prob / lv.nodes, node = prob % lv.nodes;
    const int64_t i = p / lv.bp;
    const int64_t node_start = node * lv.node_len;
    const int32_t *permQ = perm + (prob * 2 + 0) * N;
    const int32_t *permK = perm + (prob * 2 + 1) * N;
    const int32_t *invK = inv + (prob * 2 + 1) * N;
    const int64_t qrow = node_start + lv.q_off + permQ[p];

    RowGrad<DPL> rg;
    rg.K = K; rg.V = V; rg.dtype = dtype; rg.dK = dK; rg.dV = dV;
    rg.head = bhi * lv.n * D;
    rg.col = lane * DPL;
    load_slice<DPL>(Q, rg.head + qrow * D + rg.col, dtype, rg.q);
    load_slice<DPL>(dO, rg.head + qrow * D + rg.col, dtype, rg.go);
#pragma unroll
    for (int c = 0; c < DPL; ++c) rg.dq[c] = 0.0f;
    rg.Lq = L[bhi * lv.n + qrow];
    rg.gq = g[bhi * lv.n + qrow];

    for (int64_t j = 0; j < lv.bp; ++j) rg.term(node_start + permK[i * lv.bp + j], 0.0f, 0.0f);
    if (m > 0) {
        const float lw = logf(static_cast<float>(N) / static_cast<float>(m));
        const int64_t set = (bhi * nodes_total + (lv.heap0 + node - 1)) * m;
        for (int u = 0; u < m; ++u) {
            const int32_t kl = S[set + u];
            if (invK[kl] / lv.bp == i) continue;     // counted exactly in the block part
            rg.term(node_start + kl, Srn ? -INFINITY : lw, lw);
        }
        for (int u = 0; Srn && u < m; ++u) {
            const int32_t kl = Srn[set + u];
            if (kl < 0 || invK[kl] / lv.bp == i) continue;
            rg.term(node_start + kl, lwrn[set + u], -INFINITY);
        }
    }
    float *dq = dQ + rg.head + qrow * D + rg.col;
#pragma unroll
    for (int c = 0; c < DPL; ++c) dq[c] += rg.dq[c];   // one warp per row in this launch; launches are ordered
}

// The exact causal leaves: keys [q - q mod leaf, q] with weight 1.
template <int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_leaf_kernel(
    const void *__restrict__ Q, const void *__restrict__ K, const void *__restrict__ V, const void *__restrict__ dO,
    int dtype, int64_t bh, int64_t n, int64_t leaf, const float *__restrict__ L, const float *__restrict__ g,
    float *dQ, float *dK, float *dV) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    if (wg >= bh * n) return;
    const int64_t bhi = wg / n, qrow = wg % n;
    RowGrad<DPL> rg;
    rg.K = K; rg.V = V; rg.dtype = dtype; rg.dK = dK; rg.dV = dV;
    rg.head = bhi * n * D;
    rg.col = lane * DPL;
    load_slice<DPL>(Q, rg.head + qrow * D + rg.col, dtype, rg.q);
    load_slice<DPL>(dO, rg.head + qrow * D + rg.col, dtype, rg.go);
#pragma unroll
    for (int c = 0; c < DPL; ++c) rg.dq[c] = 0.0f;
    rg.Lq = L[wg];
    rg.gq = g[wg];
    for (int64_t k = qrow - qrow % leaf; k <= qrow; ++k) rg.term(k, 0.0f, 0.0f);
    float *dq = dQ + rg.head + qrow * D + rg.col;
#pragma unroll
    for (int c = 0; c < DPL; ++c) dq[c] += rg.dq[c];
}

unsigned grid_of(int64_t warps) { return static_cast<unsigned>((warps + kWarps - 1) / kWarps); }

}  // namespace

int launch_bwd_rowdot(const void *dO, int dtype, const float *O, int64_t rows, int d, float *g, cudaStream_t st) {
    if (d == 64) bwd_rowdot_kernel<64><<<grid_of(rows), kWarps * 32, 0, st>>>(dO, dtype, O, rows, g);
    else if (d == 128) bwd_rowdot_kernel<128><<<grid_of(rows), kWarps * 32, 0, st>>>(dO, dtype, O, rows, g);
    else return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int launch_bwd_level(const Level &lv, const void *Q, const void *K, const void *V, const void *dO, int dtype, int d,
                     const int32_t *perm, const int32_t *inv, const int32_t *S, int m, int64_t nodes_total,
                     const int32_t *Srn, const float *lwrn, const float *L, const float *g, float *dQ, float *dK,
                     float *dV, cudaStream_t st) {
    const unsigned grid = grid_of(lv.bh * lv.nodes * lv.seg_len);
    if (d == 64)
        bwd_level_kernel<64><<<grid, kWarps * 32, 0, st>>>(lv, Q, K, V, dO, dtype, perm, inv, S, m, nodes_total, Srn,
                                                          lwrn, L, g, dQ, dK, dV);
    else if (d == 128)
        bwd_level_kernel<128><<<grid, kWarps * 32, 0, st>>>(lv, Q, K, V, dO, dtype, perm, inv, S, m, nodes_total, Srn,
                                                           lwrn, L, g, dQ, dK, dV);
    else
        return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int launch_bwd_leaf(const void *Q, const void *K, const void *V, const void *dO, int dtype, int64_t bh, int64_t n,
                    int d, int64_t leaf, const float *L, const float *g, float *dQ, float *dK, float *dV,
                    cudaStream_t st) {
    const unsigned grid = grid_of(bh * n);
    if (d == 64)
        bwd_leaf_kernel<64><<<grid, kWarps * 32, 0, st>>>(Q, K, V, dO, dtype, bh, n, leaf, L, g, dQ, dK, dV);
    else if (d == 128)
        bwd_leaf_kernel<128><<<grid, kWarps * 32, 0, st>>>(Q, K, V, dO, dtype, bh, n, leaf, L, g, dQ, dK, dV);
    else
        return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace ha
