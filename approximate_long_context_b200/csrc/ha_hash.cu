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
// Layout: persistent CTAs of 128 threads walk tiles of 128 x RPT consecutive rows of the combined index
// g = ((bh*2 + which)*n + row) (which 0 = Q, 1 = K), RPT rows per thread. Tiles are double-buffered in
// shared memory: the 16-byte cp.async copies of tile i+1 (coalesced; row stride padded by 16 bytes against
// bank conflicts) are in flight while tile i is hashed. P travels as a kernel parameter ([d][r4], r rounded
// up to a multiple of 4): the loops over k and j are unrolled, so every fused multiply-add takes its P[k][j]
// straight from the constant bank, with no load instruction. A thread hashes two rows for d = 64 and one for
// d = 128, so that the unrolled body has the same size for both (with two rows at d = 128 it outgrew the
// instruction cache).
#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

constexpr int kThreads = 128;

// The projection matrix, [D][R4] (columns j >= r are zero).
template <int D, int R4>
struct HashProj {
    float v[D * (R4 > 0 ? R4 : 1)];
};

// RPT rows per thread: a tile is kThreads * RPT consecutive rows; thread i hashes rows i, i + kThreads, ...
template <int D, int DTYPE, int R4, int RPT>
__global__ void __launch_bounds__(kThreads) hash_kernel(const void *__restrict__ Q, const void *__restrict__ K,
                                                        int64_t n, int64_t total_rows,
                                                        const __grid_constant__ HashProj<D, R4> P, int r,
                                                        uint16_t *__restrict__ rank, uint8_t *__restrict__ near) {
    constexpr int kRows = kThreads * RPT;
    constexpr int ESZ = DTYPE == 0 ? 2 : 4;
    constexpr int ROW_BYTES = D * ESZ;
    constexpr int STRIDE = ROW_BYTES + 16;
    constexpr int CHUNKS = ROW_BYTES / 16;
    constexpr int EPC = 16 / ESZ;          // elements per 16-byte chunk
    // R4: r rounded up to a multiple of 4 (compile time, so the unrolled loops carry no conditions); the
    // padded projections multiply zero columns of P and are ignored.
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char *tiles = smem;                                               // [2][kRows][STRIDE]

    const int tid = threadIdx.x;
    const int64_t ntiles = (total_rows + kRows - 1) / kRows;

    // stage one tile with 16-byte copies. A tile inside one segment (the usual case) is kRows * ROW_BYTES
    // contiguous bytes; a tile that straddles segments locates each row (segment = g / n).
    auto stage = [&](int64_t tile, int buf) {
        unsigned char *dst = tiles + buf * (kRows * STRIDE);
        const int64_t g0 = tile * kRows;
        const int64_t seg0 = g0 / n, rr0 = g0 - seg0 * n;
        if (rr0 + kRows <= n) {
            const unsigned char *src = static_cast<const unsigned char *>((seg0 & 1) ? K : Q) +
                                       ((seg0 >> 1) * n + rr0) * ROW_BYTES;
#pragma unroll 4
            for (int i = tid; i < kRows * CHUNKS; i += kThreads) {
                const int row = i / CHUNKS, ch = i % CHUNKS;
                cp_async_16(dst + row * STRIDE + ch * 16, src + static_cast<int64_t>(i) * 16);
            }
        } else {
            const int ch = tid % CHUNKS;
            for (int row = tid / CHUNKS; row < kRows; row += kThreads / CHUNKS) {
                if (g0 + row >= total_rows) break;
                int64_t seg = seg0, rr = rr0 + row;
                while (rr >= n) { rr -= n; ++seg; }
                const int64_t which = seg & 1, bhi = seg >> 1;
                const unsigned char *src = static_cast<const unsigned char *>(which ? K : Q) +
                                           ((bhi * n + rr) * D) * ESZ + ch * 16;
                cp_async_16(dst + row * STRIDE + ch * 16, src);
            }
        }
        cp_async_commit();
    };

    int64_t tile = blockIdx.x;
    if (tile < ntiles) stage(tile, 0);
    int buf = 0;
    for (; tile < ntiles; tile += gridDim.x, buf ^= 1) {
        const int64_t next = tile + gridDim.x;
        if (next < ntiles) {
            stage(next, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();   // tile `buf` visible to every thread

        const unsigned char *rows = tiles + buf * (kRows * STRIDE) + tid * STRIDE;
        float acc[RPT][R4 > 0 ? R4 : 1];
        float nrm2[RPT];
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            nrm2[q] = 0.0f;
#pragma unroll
            for (int j = 0; j < R4; ++j) acc[q][j] = 0.0f;
        }
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            float x[RPT][EPC];
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const uint4 v = *reinterpret_cast<const uint4 *>(rows + q * (kThreads * STRIDE) + c * 16);
                if (DTYPE == 0) {
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[q][2 * e] = __uint_as_float(w[e] << 16);
                        x[q][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                    }
                } else {
                    x[q][0] = __uint_as_float(v.x);
                    x[q][1] = __uint_as_float(v.y);
                    x[q][2] = __uint_as_float(v.z);
                    x[q][3] = __uint_as_float(v.w);
                }
            }
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                const int k = c * EPC + e;
#pragma unroll
                for (int q = 0; q < RPT; ++q) nrm2[q] = __fmaf_rn(x[q][e], x[q][e], nrm2[q]);
#pragma unroll
                for (int j = 0; j < R4; ++j) {
                    const float p = P.v[k * R4 + j];
#pragma unroll
                    for (int q = 0; q < RPT; ++q) acc[q][j] = __fmaf_rn(x[q][e], p, acc[q][j]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            const int64_t g = tile * kRows + q * kThreads + tid;
            if (g >= total_rows) continue;
            const float thr = __fmul_rn(1e-4f, __fsqrt_rn(nrm2[q]));
            uint32_t code = 0;
            bool flag = false;
#pragma unroll
            for (int j = 0; j < R4; ++j) {
                if (j < r) {
                    code |= (acc[q][j] > 0.0f ? 1u : 0u) << j;
                    flag |= fabsf(acc[q][j]) < thr;
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
        __syncthreads();   // everyone is done with tile `buf` before it is refilled
    }
}

int num_sms_hash() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D, int DTYPE, int R4>
int launch_hash_t(const void *Q, const void *K, int64_t bh, int64_t n, const float *P, int r, uint16_t *rank,
                  uint8_t *near, cudaStream_t st) {
    HashProj<D, R4> proj{};
    for (int k = 0; k < D; ++k)
        for (int j = 0; j < r; ++j) proj.v[k * R4 + j] = P[k * r + j];
    constexpr int ESZ = DTYPE == 0 ? 2 : 4;
    // two rows per thread for d = 64, one for d = 128: the unrolled chain body (d x RPT x r fused multiply-adds)
    // then has the same size for both and fits the instruction cache
    constexpr int RPT = D == 64 ? 2 : 1;
    constexpr int kRows = kThreads * RPT;
    const size_t smem = 2 * kRows * (D * ESZ + 16);
    auto kern = hash_kernel<D, DTYPE, R4, RPT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t total = 2 * bh * n;
    const int64_t ntiles = (total + kRows - 1) / kRows;
    const int64_t slots = static_cast<int64_t>(num_sms_hash()) * per_sm;
    const int64_t grid = ntiles < slots ? ntiles : slots;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(Q, K, n, total, proj, r, rank, near);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

template <int D, int DTYPE>
int launch_hash_r(const void *Q, const void *K, int64_t bh, int64_t n, const float *P, int r, uint16_t *rank,
                  uint8_t *near, cudaStream_t st) {
    switch ((r + 3) / 4) {
        case 0: return launch_hash_t<D, DTYPE, 0>(Q, K, bh, n, P, r, rank, near, st);
        case 1: return launch_hash_t<D, DTYPE, 4>(Q, K, bh, n, P, r, rank, near, st);
        case 2: return launch_hash_t<D, DTYPE, 8>(Q, K, bh, n, P, r, rank, near, st);
        case 3: return launch_hash_t<D, DTYPE, 12>(Q, K, bh, n, P, r, rank, near, st);
        default: return launch_hash_t<D, DTYPE, 16>(Q, K, bh, n, P, r, rank, near, st);
    }
}

}  // namespace

// P: [d][r] float in host memory (copied into the launch's parameters).
int launch_hash(const void *Q, const void *K, int dtype, int64_t bh, int64_t n, int d, const float *P, int r,
                uint16_t *rank, uint8_t *near, cudaStream_t st) {
    if (r < 0 || r > kMaxR || (d != 64 && d != 128)) return -1;
    if (d == 64) return dtype == 0 ? launch_hash_r<64, 0>(Q, K, bh, n, P, r, rank, near, st)
                                   : launch_hash_r<64, 1>(Q, K, bh, n, P, r, rank, near, st);
    return dtype == 0 ? launch_hash_r<128, 0>(Q, K, bh, n, P, r, rank, near, st)
                      : launch_hash_r<128, 1>(Q, K, bh, n, P, r, rank, near, st);
}

}  // namespace ha
