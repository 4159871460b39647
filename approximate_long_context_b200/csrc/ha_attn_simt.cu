// ha_attn_simt.cu -- SIMT fp32 attention kernels: the fp32-input path and a tensor-core-free reference
// path for bf16 inputs.
//
// attn_simt_kernel: one warp per query of one level. The query at sorted position p of its problem lies in
// block i = p / b' ("HyperAttention: Long-context Attention in Near-Linear Time", research-map summary,
// "Approach": exact masked row sums inside the aligned diagonal blocks of the sorted order) and sees
//   * every key at sorted positions [i*b', (i+1)*b') with weight 1, and
//   * every sampled column s whose key is NOT in block i (its sorted position / b' != i) with weight N/m
//     (uniform column sampling; in-block columns are already counted exactly).
// One online softmax runs over both sets with the weight folded into the score as + log(N/m), which gives
// O = (N1 + N2) / (D1 + D2) and the log normaliser L = log(D1 + D2). The gather of the permuted rows is
// done here: rows are read through the permutation, no permuted copy is stored.
// With row-norm sampling of the product with V ("Approach": rows of V drawn in proportion to their squared
// norms), the uniform samples feed only the normaliser D2 and the row-norm draws, each with its own log
// weight log(1 / (m p_j)), feed only the numerator N2; both share the running maximum.
//
// causal_base_simt_kernel: exact causal attention (key index <= query index) inside leaves of `leaf` rows,
// then the log-space merge with the off-diagonal parts of every causal level the row belongs to (the
// summary's recursive causal extension and "Limitations": partitioning and merging).
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kWarpsPerCta = 8;

template <int DPL>
struct RowState {
    float mx = -INFINITY;
    float l = 0.0f;
    float o[DPL];
    __device__ RowState() {
#pragma unroll
        for (int c = 0; c < DPL; ++c) o[c] = 0.0f;
    }
    // add one key with score s (already including any log-weight) and value slice v, to the normaliser
    // (TO_L) and/or to the numerator (TO_O)
    template <bool TO_L = true, bool TO_O = true>
    __device__ void add(float s, const float (&v)[DPL]) {
        if (s > mx) {
            const float corr = expf(mx - s);   // 0 when mx = -inf
            l = l * corr + (TO_L ? 1.0f : 0.0f);
#pragma unroll
            for (int c = 0; c < DPL; ++c) o[c] = o[c] * corr + (TO_O ? v[c] : 0.0f);
            mx = s;
        } else {
            const float e = expf(s - mx);
            if (TO_L) l += e;
#pragma unroll
            for (int c = 0; c < DPL; ++c)
                if (TO_O) o[c] += e * v[c];
        }
    }
};

template <int DPL>
__device__ __forceinline__ void load_slice(const void *base, int64_t off, int dtype, float (&x)[DPL]) {
#pragma unroll
    for (int c = 0; c < DPL; ++c) x[c] = load_elem(base, off + c, dtype);
}

template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32) attn_simt_kernel(
    Level lv, const void *__restrict__ Q, const void *__restrict__ K, const void *__restrict__ V, int dtype,
    const int32_t *__restrict__ perm, const int32_t *__restrict__ inv, const int32_t *__restrict__ S, int m,
    int64_t nodes_total, void *__restrict__ O, int out_dtype, float *__restrict__ lse, float *__restrict__ Opart,
    float *__restrict__ Lpart, const int32_t *__restrict__ Srn, const float *__restrict__ lwrn) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
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
    const int64_t head = bhi * lv.n * D;
    const int64_t col = lane * DPL;

    float q[DPL], x[DPL];
    load_slice<DPL>(Q, head + qrow * D + col, dtype, q);
    RowState<DPL> st;

    for (int64_t j = 0; j < lv.bp; ++j) {
        const int64_t krow = node_start + permK[i * lv.bp + j];
        load_slice<DPL>(K, head + krow * D + col, dtype, x);
        float part = 0.0f;
#pragma unroll
        for (int c = 0; c < DPL; ++c) part += q[c] * x[c];
        const float s = warp_sum(part);
        load_slice<DPL>(V, head + krow * D + col, dtype, x);
        st.add(s, x);
    }
    if (m > 0) {
        const float logw = logf(static_cast<float>(N) / static_cast<float>(m));
        const int32_t *Sp = S + (bhi * nodes_total + (lv.heap0 + node - 1)) * m;
        for (int u = 0; u < m; ++u) {
            const int32_t kl = Sp[u];
            if (invK[kl] / lv.bp == i) continue;      // already counted exactly in the block part
            const int64_t krow = node_start + kl;
            load_slice<DPL>(K, head + krow * D + col, dtype, x);
            float part = 0.0f;
#pragma unroll
            for (int c = 0; c < DPL; ++c) part += q[c] * x[c];
            const float s = warp_sum(part) + logw;
            if (Srn) {
                st.add<true, false>(s, x);            // normaliser only
            } else {
                load_slice<DPL>(V, head + krow * D + col, dtype, x);
                st.add(s, x);
            }
        }
    }
    if (Srn && m > 0) {
        const int64_t set = (bhi * nodes_total + (lv.heap0 + node - 1)) * m;
        for (int u = 0; u < m; ++u) {
            const int32_t kl = Srn[set + u];
            if (kl < 0 || invK[kl] / lv.bp == i) continue;
            const int64_t krow = node_start + kl;
            load_slice<DPL>(K, head + krow * D + col, dtype, x);
            float part = 0.0f;
#pragma unroll
            for (int c = 0; c < DPL; ++c) part += q[c] * x[c];
            const float s = warp_sum(part) + lwrn[set + u];
            load_slice<DPL>(V, head + krow * D + col, dtype, x);
            st.add<false, true>(s, x);                // numerator only
        }
    }
    const float inv_l = 1.0f / st.l;
    const float L = st.mx + logf(st.l);
    if (lv.level == 0) {
#pragma unroll
        for (int c = 0; c < DPL; ++c) store_out(O, head + qrow * D + col + c, st.o[c] * inv_l, out_dtype);
        if (lse && lane == 0) lse[bhi * lv.n + qrow] = L;
    } else {
        const int64_t half_n = lv.n / 2;
        const int64_t dense = bhi * half_n + node * N + (qrow - node_start - lv.q_off);
#pragma unroll
        for (int c = 0; c < DPL; ++c) Opart[dense * D + col + c] = st.o[c] * inv_l;
        if (lane == 0) Lpart[dense] = L;
    }
}

template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32) causal_base_simt_kernel(
    const void *__restrict__ Q, const void *__restrict__ K, const void *__restrict__ V, int dtype, int64_t bh,
    int64_t n, int64_t leaf, int levels, const float *__restrict__ Opart, const float *__restrict__ Lpart,
    void *__restrict__ O, int out_dtype, float *__restrict__ Lout) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wg = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
    if (wg >= bh * n) return;
    const int64_t bhi = wg / n, qrow = wg % n;
    const int64_t head = bhi * n * D;
    const int64_t col = lane * DPL;
    float q[DPL], x[DPL];
    load_slice<DPL>(Q, head + qrow * D + col, dtype, q);
    RowState<DPL> st;
    for (int64_t k = qrow - qrow % leaf; k <= qrow; ++k) {
        load_slice<DPL>(K, head + k * D + col, dtype, x);
        float part = 0.0f;
#pragma unroll
        for (int c = 0; c < DPL; ++c) part += q[c] * x[c];
        const float s = warp_sum(part);
        load_slice<DPL>(V, head + k * D + col, dtype, x);
        st.add(s, x);
    }
    // running part (O normalised, log normaliser)
    float Ocur[DPL];
    const float inv_l = 1.0f / st.l;
#pragma unroll
    for (int c = 0; c < DPL; ++c) Ocur[c] = st.o[c] * inv_l;
    float Lcur = st.mx + logf(st.l);
    const int64_t half_n = n / 2;
    for (int lvl = 1; lvl <= levels; ++lvl) {
        const int64_t len = n >> (lvl - 1), half = len / 2;
        const int64_t within = qrow % len;
        if (within < half) continue;                 // not a query of this level's off-diagonal block
        const int64_t dense = static_cast<int64_t>(lvl - 1) * bh * half_n + bhi * half_n + (qrow / len) * half +
                              (within - half);
        const float Lp = Lpart[dense];
        if (Lp == -INFINITY) continue;
        const float M = fmaxf(Lcur, Lp);
        const float a = expf(Lcur - M), b = expf(Lp - M);
        const float inv = 1.0f / (a + b);
#pragma unroll
        for (int c = 0; c < DPL; ++c) Ocur[c] = (a * Ocur[c] + b * Opart[dense * D + col + c]) * inv;
        Lcur = M + logf(a + b);
    }
#pragma unroll
    for (int c = 0; c < DPL; ++c) store_out(O, head + qrow * D + col + c, Ocur[c], out_dtype);
    if (Lout && lane == 0) Lout[wg] = Lcur;   // the row's final log normaliser (for the backward pass)
}

}  // namespace

int launch_attn_simt(const Level &lv, const void *Q, const void *K, const void *V, int dtype, int d,
                     const int32_t *perm, const int32_t *inv, const int32_t *S, int m, int64_t nodes_total,
                     void *O, int out_dtype, float *lse, float *Opart, float *Lpart, cudaStream_t st,
                     const int32_t *Srn, const float *lwrn) {
    const int64_t warps = lv.bh * lv.nodes * lv.seg_len;
    const int64_t grid = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
    if (d == 64)
        attn_simt_kernel<64><<<static_cast<unsigned>(grid), kWarpsPerCta * 32, 0, st>>>(
            lv, Q, K, V, dtype, perm, inv, S, m, nodes_total, O, out_dtype, lse, Opart, Lpart, Srn, lwrn);
    else if (d == 128)
        attn_simt_kernel<128><<<static_cast<unsigned>(grid), kWarpsPerCta * 32, 0, st>>>(
            lv, Q, K, V, dtype, perm, inv, S, m, nodes_total, O, out_dtype, lse, Opart, Lpart, Srn, lwrn);
    else
        return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int launch_causal_base_simt(const void *Q, const void *K, const void *V, int dtype, int64_t bh, int64_t n, int d,
                            int64_t leaf, int levels, const float *Opart, const float *Lpart, void *O,
                            int out_dtype, cudaStream_t st, float *Lout) {
    const int64_t grid = (bh * n + kWarpsPerCta - 1) / kWarpsPerCta;
    if (d == 64)
        causal_base_simt_kernel<64><<<static_cast<unsigned>(grid), kWarpsPerCta * 32, 0, st>>>(
            Q, K, V, dtype, bh, n, leaf, levels, Opart, Lpart, O, out_dtype, Lout);
    else if (d == 128)
        causal_base_simt_kernel<128><<<static_cast<unsigned>(grid), kWarpsPerCta * 32, 0, st>>>(
            Q, K, V, dtype, bh, n, leaf, levels, Opart, Lpart, O, out_dtype, Lout);
    else
        return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace ha
