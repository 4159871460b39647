// ha_hash.cu -- sortLSH hashing of the Q and K rows.
//
// "HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach" and
// "Experimental setup": Hamming-sorted LSH): bit j of a row x is [x.P_j > 0] (an exact zero gives 0),
// projection j is bit j (least significant first), and the r-bit code is read as a Gray codeword whose
// rank (the inverse Gray code) orders the buckets so that neighbouring ranks differ in one bit.
//
// Decision precision: each projection and the squared row norm are sequential fp32 fused multiply-add
// chains over k = 0..d-1 from +0, so the sign decision is reproducible bit for bit. A row whose smallest
// |x.P_j| is below 1e-4 * ||x||_2 is flagged as near zero.
//
// Layout: one CTA hashes 128 consecutive rows of the combined index g = ((bh*2 + which)*n + row)
// (which 0 = Q, 1 = K). The rows are staged in shared memory with 16-byte cp.async copies (coalesced;
// the row stride is padded by 16 bytes so that the per-thread row reads do not collide on banks), then
// each thread runs the chains of one row. P is staged transposed ([j][k]) so that the k-loop reads it as
// broadcast float4 loads.
#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kRowsPerCta = 128;

template <int D, int DTYPE>
__global__ void __launch_bounds__(kRowsPerCta) hash_kernel(const void *__restrict__ Q, const void *__restrict__ K,
                                                           int64_t n, int64_t total_rows,
                                                           const float *__restrict__ P, int r,
                                                           uint16_t *__restrict__ rank, uint8_t *__restrict__ near) {
    constexpr int ESZ = DTYPE == 0 ? 2 : 4;
    constexpr int ROW_BYTES = D * ESZ;
    constexpr int STRIDE = ROW_BYTES + 16;
    constexpr int CHUNKS = ROW_BYTES / 16;
    extern __shared__ __align__(16) unsigned char smem[];
    float *PT = reinterpret_cast<float *>(smem);                       // [kMaxR][D]
    unsigned char *tile = smem + kMaxR * D * sizeof(float);            // [kRowsPerCta][STRIDE]

    const int tid = threadIdx.x;
    const int64_t g0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;

    for (int i = tid; i < r * D; i += kRowsPerCta) {
        const int j = i / D, k = i % D;
        PT[j * D + k] = P[k * r + j];
    }
    for (int c = tid; c < kRowsPerCta * CHUNKS; c += kRowsPerCta) {
        const int row = c / CHUNKS, ch = c % CHUNKS;
        const int64_t g = g0 + row;
        if (g < total_rows) {
            const int64_t which = (g / n) & 1, bhi = g / (2 * n), rr = g % n;
            const unsigned char *src = static_cast<const unsigned char *>(which ? K : Q) +
                                       ((bhi * n + rr) * D) * ESZ + ch * 16;
            cp_async_16(tile + row * STRIDE + ch * 16, src);
        }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int64_t g = g0 + tid;
    if (g >= total_rows) return;
    const unsigned char *row = tile + tid * STRIDE;

    float acc[kMaxR];
#pragma unroll
    for (int j = 0; j < kMaxR; ++j) acc[j] = 0.0f;
    float nrm2 = 0.0f;

#pragma unroll 1
    for (int h = 0; h < D / 64; ++h) {
        float x[64];
#pragma unroll
        for (int c = 0; c < 64 * ESZ / 16; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + h * 64 * ESZ + c * 16);
            if (DTYPE == 0) {
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[c * 8 + 2 * e] = __uint_as_float(w[e] << 16);
                    x[c * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
            } else {
                x[c * 4 + 0] = __uint_as_float(v.x);
                x[c * 4 + 1] = __uint_as_float(v.y);
                x[c * 4 + 2] = __uint_as_float(v.z);
                x[c * 4 + 3] = __uint_as_float(v.w);
            }
        }
#pragma unroll
        for (int k = 0; k < 64; ++k) nrm2 = __fmaf_rn(x[k], x[k], nrm2);
#pragma unroll
        for (int j = 0; j < kMaxR; ++j) {
            if (j < r) {
                const float4 *pj = reinterpret_cast<const float4 *>(PT + j * D + h * 64);
#pragma unroll
                for (int k4 = 0; k4 < 16; ++k4) {
                    const float4 p = pj[k4];
                    acc[j] = __fmaf_rn(x[4 * k4 + 0], p.x, acc[j]);
                    acc[j] = __fmaf_rn(x[4 * k4 + 1], p.y, acc[j]);
                    acc[j] = __fmaf_rn(x[4 * k4 + 2], p.z, acc[j]);
                    acc[j] = __fmaf_rn(x[4 * k4 + 3], p.w, acc[j]);
                }
            }
        }
    }

    const float thr = __fmul_rn(1e-4f, __fsqrt_rn(nrm2));
    uint32_t code = 0;
    bool flag = false;
#pragma unroll
    for (int j = 0; j < kMaxR; ++j) {
        if (j < r) {
            code |= (acc[j] > 0.0f ? 1u : 0u) << j;
            flag |= fabsf(acc[j]) < thr;
        }
    }
    // inverse Gray code: prefix XOR of all right shifts (16-bit codes)
    uint32_t g2 = code;
    g2 ^= g2 >> 1;
    g2 ^= g2 >> 2;
    g2 ^= g2 >> 4;
    g2 ^= g2 >> 8;
    rank[g] = static_cast<uint16_t>(g2);
    near[g] = flag ? 1 : 0;
}

template <int D, int DTYPE>
int launch_hash_t(const void *Q, const void *K, int64_t bh, int64_t n, const float *P, int r, uint16_t *rank,
                  uint8_t *near, cudaStream_t st) {
    constexpr int ESZ = DTYPE == 0 ? 2 : 4;
    const size_t smem = kMaxR * D * sizeof(float) + kRowsPerCta * (D * ESZ + 16);
    auto kern = hash_kernel<D, DTYPE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    const int64_t total = 2 * bh * n;
    const int64_t grid = (total + kRowsPerCta - 1) / kRowsPerCta;
    kern<<<static_cast<unsigned>(grid), kRowsPerCta, smem, st>>>(Q, K, n, total, P, r, rank, near);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int launch_hash(const void *Q, const void *K, int dtype, int64_t bh, int64_t n, int d, const float *P, int r,
                uint16_t *rank, uint8_t *near, cudaStream_t st) {
    if (d == 64) return dtype == 0 ? launch_hash_t<64, 0>(Q, K, bh, n, P, r, rank, near, st)
                                   : launch_hash_t<64, 1>(Q, K, bh, n, P, r, rank, near, st);
    if (d == 128) return dtype == 0 ? launch_hash_t<128, 0>(Q, K, bh, n, P, r, rank, near, st)
                                    : launch_hash_t<128, 1>(Q, K, bh, n, P, r, rank, near, st);
    return -1;
}

}  // namespace ha
