// ha_diag.cu -- hardness diagnostics of the attention matrix for small problems.
//
// "HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach", "Key
// results", "Limitations"; abstract page): the method's guarantee rests on (1) the max column norm of the
// normalised attention matrix D^-1 A and (2) the ratio of row norms of A once its large entries are removed.
// Readings (the same as the oracle's):
//   alpha = n * max_{j >= first_col} sum_i W_ij^2, W = D^-1 A, A_ij = exp(q_i . k_j);
//   kappa = max_i R_i / min_i R_i, R_i = sum of A_ij over the columns outside row i's sortLSH block (the
//   entries the method computes exactly); 0/0 gives NaN, x/0 gives +inf.
// Both need every entry of A, so they are for small n (the entry point bounds n). Each kernel gives one warp
// one row or one column; scores are fp32 dot products, sums fp32, the reduction in double.
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kDiagWarps = 8;

__device__ __forceinline__ float load_elem(const void *X, int dtype, int64_t idx) {
    if (dtype == 0) {
        const uint16_t b = static_cast<const uint16_t *>(X)[idx];
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    return static_cast<const float *>(X)[idx];
}

// dot of a row staged in shared memory (d floats) with row `row` of X
__device__ __forceinline__ float dot_row(const float *xs, const void *X, int dtype, int64_t row, int d) {
    float acc = 0.0f;
    for (int k = 0; k < d; ++k) acc = fmaf(xs[k], load_elem(X, dtype, row * d + k), acc);
    return acc;
}

// One warp per (problem, query row): max score, normaliser and the sum outside the row's block (both shifted
// by the row max), written as m, D and log R (log R = -inf when nothing lies outside the block).
__global__ void __launch_bounds__(kDiagWarps * 32) diag_rows_kernel(const void *Q, const void *K, int dtype, int64_t n,
                                                                  int d, int64_t bh, const int32_t *inv, int64_t bp,
                                                                  float *m_out, float *d_out, float *logr_out) {
    __shared__ float qs[kDiagWarps][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * kDiagWarps + warp;
    if (g >= bh * n) return;
    const int64_t b = g / n, i = g % n;
    for (int k = lane; k < d; k += 32) qs[warp][k] = load_elem(Q, dtype, g * d + k);
    __syncwarp();
    const int64_t blk_i = inv[(b * 2 + 0) * n + i] / bp;
    float mx = -INFINITY;
    for (int64_t j = lane; j < n; j += 32) mx = fmaxf(mx, dot_row(qs[warp], K, dtype, b * n + j, d));
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float den = 0.0f, rest = 0.0f;
    for (int64_t j = lane; j < n; j += 32) {
        const float e = expf(dot_row(qs[warp], K, dtype, b * n + j, d) - mx);
        den += e;
        if (inv[(b * 2 + 1) * n + j] / bp != blk_i) rest += e;
    }
    for (int off = 16; off > 0; off >>= 1) {
        den += __shfl_xor_sync(0xffffffffu, den, off);
        rest += __shfl_xor_sync(0xffffffffu, rest, off);
    }
    if (lane == 0) {
        m_out[g] = mx;
        d_out[g] = den;
        logr_out[g] = rest > 0.0f ? logf(rest) + mx : -INFINITY;
    }
}

// One warp per (problem, key column j): sum over rows of W_ij^2 = (exp(q_i . k_j - m_i) / D_i)^2.
__global__ void __launch_bounds__(kDiagWarps * 32) diag_cols_kernel(const void *Q, const void *K, int dtype, int64_t n,
                                                                  int d, int64_t bh, const float *m_in,
                                                                  const float *d_in, float *col_out) {
    __shared__ float ks[kDiagWarps][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * kDiagWarps + warp;
    if (g >= bh * n) return;
    const int64_t b = g / n;
    for (int k = lane; k < d; k += 32) ks[warp][k] = load_elem(K, dtype, g * d + k);
    __syncwarp();
    float acc = 0.0f;
    for (int64_t i = lane; i < n; i += 32) {
        const int64_t row = b * n + i;
        const float w = expf(dot_row(ks[warp], Q, dtype, row, d) - m_in[row]) / d_in[row];
        acc = fmaf(w, w, acc);
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) col_out[g] = acc;
}

// One block per problem: alpha = n * max_{j >= first_col} col_j, kappa = exp(max log R - min log R).
__global__ void __launch_bounds__(256) diag_reduce_kernel(int64_t n, int64_t first_col, const float *col,
                                                         const float *logr, double *out) {
    __shared__ float smax[256], rmax[256], rmin[256];
    const int64_t b = blockIdx.x;
    float cm = 0.0f, hi = -INFINITY, lo = INFINITY;
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
        if (j >= first_col) cm = fmaxf(cm, col[b * n + j]);
        const float lr = logr[b * n + j];
        hi = fmaxf(hi, lr);
        lo = fminf(lo, lr);
    }
    smax[threadIdx.x] = cm;
    rmax[threadIdx.x] = hi;
    rmin[threadIdx.x] = lo;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            smax[threadIdx.x] = fmaxf(smax[threadIdx.x], smax[threadIdx.x + s]);
            rmax[threadIdx.x] = fmaxf(rmax[threadIdx.x], rmax[threadIdx.x + s]);
            rmin[threadIdx.x] = fminf(rmin[threadIdx.x], rmin[threadIdx.x + s]);
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[2 * b] = static_cast<double>(n) * static_cast<double>(smax[0]);
        const float h = rmax[0], l = rmin[0];
        double kappa;
        if (h == -INFINITY) kappa = nan("");              // nothing outside any row's block
        else if (l == -INFINITY) kappa = INFINITY;         // some rows have nothing outside their block
        else kappa = exp(static_cast<double>(h) - static_cast<double>(l));
        out[2 * b + 1] = kappa;
    }
}

}  // namespace

int launch_diagnostics(const void *Q, const void *K, int dtype, int64_t bh, int64_t n, int d, const int32_t *inv,
                       int64_t bp, int64_t first_col, float *scratch, double *out, cudaStream_t st) {
    if (d > 128 || n <= 0 || bp <= 0) return -1;
    float *m = scratch, *D = m + bh * n, *logr = D + bh * n, *col = logr + bh * n;
    const int64_t rows = bh * n;
    const unsigned grid = static_cast<unsigned>((rows + kDiagWarps - 1) / kDiagWarps);
    diag_rows_kernel<<<grid, kDiagWarps * 32, 0, st>>>(Q, K, dtype, n, d, bh, inv, bp, m, D, logr);
    diag_cols_kernel<<<grid, kDiagWarps * 32, 0, st>>>(Q, K, dtype, n, d, bh, m, D, col);
    diag_reduce_kernel<<<static_cast<unsigned>(bh), 256, 0, st>>>(n, first_col, col, logr, out);
    return cudaPeekAtLastError() == cudaSuccess ? 3 : -1;
}

}  // namespace ha
