// ha_sort.cu -- stable segmented counting sort of the sortLSH ranks.
//
// "HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach"): the
// rows of Q and of K are sorted by their LSH bucket rank. Ties keep the original row order (stable), so the
// sorted order is unique. Every problem of a level has one query segment and one key segment of N rows
// (see ha::Level); segment s = (bh * nodes + node) * 2 + which, which 0 = queries, 1 = keys.
//
// One pass sorts by one radix digit of at most 10 bits; ranks of up to 16 bits take two stable passes
// (least significant digit first). A pass is three launches:
//   count   -- per 2048-row chunk of a segment, a shared-memory histogram of the digit;
//   scan    -- per segment, turn the chunk histograms into the first output position of every
//              (chunk, digit) pair (digit-major, chunks in order), with 1024 / radix threads per digit;
//   scatter -- per chunk, 8 warps each own a contiguous 256-row slice; a warp finds the rows of equal digit
//              inside a 32-row step with one ballot per digit bit and keeps running per-digit counters, so
//              rows leave in their original order within each digit. The chunk is ordered in shared memory
//              first, so that the permutation is written in runs of consecutive slots.
// No kernel waits on another CTA: the three launches replace a look-back scan.
#include "ha_common.cuh"
#include "ha_internal.h"

namespace ha {
namespace {

struct SegView {
    const uint16_t *rank;   // rank of local row 0 of the segment
    int64_t out;            // s * N: first slot of the segment in perm / inv
};

__device__ __forceinline__ SegView seg_view(const Level &lv, const uint16_t *rank, int64_t s) {
    const int64_t which = s & 1;
    const int64_t node = (s >> 1) % lv.nodes;
    const int64_t bhi = (s >> 1) / lv.nodes;
    const int64_t start = node * lv.node_len + (which == 0 ? lv.q_off : 0);
    SegView v;
    v.rank = rank + (bhi * 2 + which) * lv.n + start;
    v.out = s * lv.seg_len;
    return v;
}

__device__ __forceinline__ int digit_of(const SegView &v, const int32_t *in_idx, int64_t p, SortPass ps,
                                        int32_t &row) {
    row = in_idx ? in_idx[v.out + p] : static_cast<int32_t>(p);
    return (static_cast<int>(v.rank[row]) >> ps.shift) & (ps.radix - 1);
}

__global__ void __launch_bounds__(256) sort_count_kernel(Level lv, const uint16_t *__restrict__ rank, SortPass ps,
                                                         const int32_t *__restrict__ in_idx, int32_t *__restrict__ hist,
                                                         int cps) {
    extern __shared__ int cnt[];
    const int64_t s = blockIdx.x / cps;
    const int c = blockIdx.x % cps;
    for (int b = threadIdx.x; b < ps.radix; b += blockDim.x) cnt[b] = 0;
    __syncthreads();
    const SegView v = seg_view(lv, rank, s);
    const int64_t start = static_cast<int64_t>(c) * kSortChunk;
    const int64_t end = min(lv.seg_len, start + kSortChunk);
    for (int64_t p = start + threadIdx.x; p < end; p += blockDim.x) {
        int32_t row;
        atomicAdd(&cnt[digit_of(v, in_idx, p, ps, row)], 1);
    }
    __syncthreads();
    int32_t *h = hist + (s * cps + c) * ps.radix;
    for (int b = threadIdx.x; b < ps.radix; b += blockDim.x) h[b] = cnt[b];
}

// Per segment: the first output position of every (chunk, digit) pair, digit-major and chunks in order. The
// 1024 threads split into G = 1024 / radix groups per digit; group g sums, then numbers, chunks
// [g * cpg, (g + 1) * cpg), so the chunk counts of a digit are read by G threads at once.
__global__ void __launch_bounds__(1024) sort_scan_kernel(int radix, int cps, int32_t *__restrict__ hist) {
    __shared__ int part[1024];                    // [group][digit]: the group's sum, then its first position
    __shared__ int tot[1 << kMaxPassBits];
    const int64_t s = blockIdx.x;
    int32_t *h = hist + s * cps * radix;
    const int G = radix >= 1024 ? 1 : 1024 / radix;
    const int cpg = (cps + G - 1) / G;
    const int b = threadIdx.x % radix, g = threadIdx.x / radix;
    const bool active = g < G;
    const int c0 = g * cpg, c1 = min(cps, c0 + cpg);
    constexpr int U = 16;   // loads in flight together
    if (active) {
        int sum = 0;
        for (int c = c0; c < c1; c += U) {
            int t[U];
#pragma unroll
            for (int u = 0; u < U; ++u) t[u] = c + u < c1 ? h[(c + u) * radix + b] : 0;
#pragma unroll
            for (int u = 0; u < U; ++u) sum += t[u];
        }
        part[g * radix + b] = sum;
    }
    __syncthreads();
    if (threadIdx.x < radix) {   // exclusive over the groups of digit b; the digit's total
        int run = 0;
        for (int gg = 0; gg < G; ++gg) {
            const int t = part[gg * radix + b];
            part[gg * radix + b] = run;
            run += t;
        }
        tot[b] = run;
    }
    __syncthreads();
    // inclusive scan of the digit totals (Hillis-Steele; radix <= blockDim, one digit per thread)
    const int tb = threadIdx.x;
    for (int off = 1; off < radix; off <<= 1) {
        const int add = (tb < radix && tb >= off) ? tot[tb - off] : 0;
        __syncthreads();
        if (tb < radix) tot[tb] += add;
        __syncthreads();
    }
    if (active) {
        int run = (b == 0 ? 0 : tot[b - 1]) + part[g * radix + b];
        for (int c = c0; c < c1; c += U) {
            int t[U];
#pragma unroll
            for (int u = 0; u < U; ++u) t[u] = c + u < c1 ? h[(c + u) * radix + b] : 0;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c + u < c1) {
                    h[(c + u) * radix + b] = run;
                    run += t[u];
                }
        }
    }
}

// Exclusive prefix sum of a[0..R) in place by a block of kSortWarps * 32 threads (R <= 4 * blockDim).
__device__ __forceinline__ void block_exclusive_scan(int *a, int R, int *warp_sums) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (R + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * per;
    int v[4];
    int sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        v[u] = (u < per && b0 + u < R) ? a[b0 + u] : 0;
        sum += v[u];
    }
    int x = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < kSortWarps; ++w) {
            const int t = warp_sums[w];
            warp_sums[w] = run;
            run += t;
        }
    }
    __syncthreads();
    int run = warp_sums[warp] + x - sum;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (u < per && b0 + u < R) a[b0 + u] = run;
        run += v[u];
    }
    __syncthreads();
}

// Per chunk: rank the rows stably by digit (warps own contiguous 256-row slices; within a 32-row step equal
// digits are ranked with __match_any_sync), giving each row its local position in the chunk's digit-sorted
// order and its global position (the digit's first slot for this chunk, from the scan, plus its rank among
// the chunk's rows of that digit). The inverse permutation is written in row order; the permutation is
// written from the digit-sorted order, so that rows of one digit land in consecutive slots.
template <int NBITS>   // log2 of the radix
__global__ void __launch_bounds__(kSortWarps * 32, 4) sort_scatter_kernel(Level lv, const uint16_t *__restrict__ rank,
                                                                       SortPass ps, const int32_t *__restrict__ in_idx,
                                                                       const int32_t *__restrict__ hist, int cps,
                                                                       int32_t *__restrict__ perm,
                                                                       int32_t *__restrict__ inv) {
    extern __shared__ int sm[];
    const int R = ps.radix;
    int *wcnt = sm;                               // [kSortWarps][R]: per-warp digit counts, then local offsets
    int *coff = wcnt + kSortWarps * R;            // [R]: first local position of each digit in the chunk
    int *gbase = coff + R;                        // [R]: first global position of each digit for this chunk
    int *wsum = gbase + R;                        // [kSortWarps]
    int32_t *srow = wsum + kSortWarps;            // [kSortChunk]: rows in local (digit-sorted) order
    int32_t *sgpos = srow + kSortChunk;           // [kSortChunk]: their global positions
    const int64_t s = blockIdx.x / cps;
    const int c = blockIdx.x % cps;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const SegView v = seg_view(lv, rank, s);
    const int64_t start = static_cast<int64_t>(c) * kSortChunk;
    const int64_t end = min(lv.seg_len, start + kSortChunk);
    constexpr int kSlice = kSortChunk / kSortWarps;
    // this chunk's first global slot of each digit (from the scan), loaded early (R <= 4 * blockDim)
    const int32_t *h = hist + (s * cps + c) * R;
    int gb_pref[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int b = threadIdx.x + u * kSortWarps * 32;
        gb_pref[u] = b < R ? h[b] : 0;
    }
    const int64_t lo = min(end, start + static_cast<int64_t>(warp) * kSlice);
    const int64_t hi = min(end, lo + kSlice);
    int *mycnt = wcnt + warp * R;

    // one ranking pass: the slice's digits (loads issued together), each row's rank among the earlier rows of
    // its digit in the slice (kept in registers), and the slice's per-digit counts
    constexpr int STEPS = kSlice / 32;
    int keyv[STEPS], rk[STEPS];
    int32_t rowv[STEPS];
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
        const int64_t p = lo + i * 32 + lane;
        rowv[i] = 0;
        keyv[i] = p < hi ? digit_of(v, in_idx, p, ps, rowv[i]) : -1;
    }
    for (int i = threadIdx.x; i < kSortWarps * R; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
        const int key = keyv[i];
        // the lanes holding the same key: one ballot for validity, one per digit bit
        unsigned peers = __ballot_sync(0xffffffffu, key >= 0);
        if (key < 0) peers = ~peers;
#pragma unroll
        for (int bb = 0; bb < NBITS; ++bb) {
            const bool bit = (key >> bb) & 1;
            const unsigned bal = __ballot_sync(0xffffffffu, bit);
            peers &= bit ? bal : ~bal;
        }
        const int before = key >= 0 ? mycnt[key] : 0;
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) mycnt[key] = before + __popc(peers);
        __syncwarp();
        rk[i] = before + __popc(peers & lt_mask);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int b = threadIdx.x + u * kSortWarps * 32;
        if (b < R) {
            int tot = 0;
            for (int w = 0; w < kSortWarps; ++w) tot += wcnt[w * R + b];
            coff[b] = tot;
            gbase[b] = gb_pref[u];
        }
    }
    __syncthreads();
    block_exclusive_scan(coff, R, wsum);
    for (int b = threadIdx.x; b < R; b += blockDim.x) {
        int run = coff[b];
        for (int w = 0; w < kSortWarps; ++w) {
            const int t = wcnt[w * R + b];
            wcnt[w * R + b] = run;
            run += t;
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
        const int key = keyv[i];
        if (key >= 0) {
            const int lpos = mycnt[key] + rk[i];
            const int gpos = gbase[key] + (lpos - coff[key]);
            if (inv) inv[v.out + rowv[i]] = gpos;
            srow[lpos] = rowv[i];
            sgpos[lpos] = gpos;
        }
    }
    __syncthreads();
    const int nloc = static_cast<int>(end - start);
    for (int lp = threadIdx.x; lp < nloc; lp += blockDim.x) perm[v.out + sgpos[lp]] = srow[lp];
}

template <int NBITS>
bool launch_scatter(int64_t grid, size_t smem, cudaStream_t st, const Level &lv, const uint16_t *rank, SortPass ps,
                    const int32_t *in_idx, const int32_t *hist, int cps, int32_t *perm, int32_t *inv) {
    auto kern = sort_scatter_kernel<NBITS>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return false;
    kern<<<static_cast<unsigned>(grid), kSortWarps * 32, smem, st>>>(lv, rank, ps, in_idx, hist, cps, perm, inv);
    return true;
}

}  // namespace

int launch_sort_pass(const Level &lv, const uint16_t *rank, SortPass ps, const int32_t *in_idx, int32_t *hist,
                     int32_t *perm, int32_t *inv, cudaStream_t st) {
    if (ps.radix < 1 || ps.radix > (1 << kMaxPassBits)) return -1;
    const int64_t nseg = lv.bh * lv.nodes * 2;
    const int cps = static_cast<int>((lv.seg_len + kSortChunk - 1) / kSortChunk);
    const int64_t grid = nseg * cps;
    sort_count_kernel<<<static_cast<unsigned>(grid), 256, ps.radix * sizeof(int), st>>>(lv, rank, ps, in_idx, hist, cps);
    sort_scan_kernel<<<static_cast<unsigned>(nseg), 1024, 0, st>>>(ps.radix, cps, hist);
    const size_t smem = (static_cast<size_t>(kSortWarps + 2) * ps.radix + kSortWarps + 2 * kSortChunk) * sizeof(int);
    int nbits = 0;
    while ((1 << nbits) < ps.radix) ++nbits;
    int ok = 0;
    switch (nbits) {
        case 0: ok = launch_scatter<0>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 1: ok = launch_scatter<1>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 2: ok = launch_scatter<2>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 3: ok = launch_scatter<3>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 4: ok = launch_scatter<4>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 5: ok = launch_scatter<5>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 6: ok = launch_scatter<6>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 7: ok = launch_scatter<7>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 8: ok = launch_scatter<8>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        case 9: ok = launch_scatter<9>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
        default: ok = launch_scatter<10>(grid, smem, st, lv, rank, ps, in_idx, hist, cps, perm, inv); break;
    }
    if (!ok) return -1;
    return cudaPeekAtLastError() == cudaSuccess ? 3 : -1;
}

}  // namespace ha
