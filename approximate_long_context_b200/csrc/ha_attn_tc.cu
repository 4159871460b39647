// ha_attn_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) attention kernels for bf16 inputs.
//
// Two modes share one persistent kernel:
//
//  LEVEL: the HyperAttention problem of one level ("HyperAttention: Long-context Attention in Near-Linear
//  Time", research-map summary, "Approach"). A work item is a pair of 128-query tiles of one sorted block
//  i. Its key stream is the b'/128 chunks of key block i (exact block part) followed by ceil(m/128) chunks
//  of the sampled columns (uniform sample part; columns whose key lies in block i, and padding past m, are
//  masked; the others carry the weight N/m as + log2(N/m) on the base-2 score). Rows are fetched through
//  the sort permutations with TMA tile::gather4 loads straight into 128-byte-swizzled shared memory, so no
//  permuted copy of Q, K or V exists. One online softmax over both parts gives O = (N1+N2)/(D1+D2); the
//  epilogue writes each row to its original position (the merge and un-permute), or, for causal levels,
//  the fp32 part and its log normaliser.
//
//  CAUSAL: exact causal attention inside leaves of c rows (the summary's recursive causal extension: the
//  base case), followed by the log-space merge with the parts of every causal level the row belongs to
//  ("Limitations": partitioning and merging). A work item is a pair of query tiles of one leaf; tile g sees
//  key chunks 0..g, the diagonal chunk with the inclusive causal mask. Items run heaviest first.
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warp 0      loader: Q tiles, K/V chunks (ring of NST stages), sample masks;
//   warp 1      MMA issuer (lane 0): S = Q K^T into TMEM, O += P V with P read from TMEM;
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: a thread owns one query row (TMEM lane),
//               reads S, keeps the running max and sum, writes P (bf16) over S in TMEM, rescales O when the
//               running max grows by more than 2^8, and runs the epilogue.
// TMEM (512 columns): S/P of tile t at columns [128 t, 128 t + 128), O of tile t at [256 + d t, 256 + d t + d).
// Every mbarrier wait is bounded; on expiry the kernel sets the status bit, the other warps give up, the
// loader waits (bounded) for its copies in flight, and TMEM is freed before exit.
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"
#include "ha_sm100.cuh"

namespace ha {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kMaxLevels = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the running max grows by more than this

enum { MODE_LEVEL = 0, MODE_CAUSAL = 1 };

struct TcArgs {
    int mode;
    int64_t n, bh;
    // LEVEL
    Level lv;
    const int32_t *perm, *inv, *S;
    int m;
    int64_t nodes_total;
    int nb, ns;            // block chunks, sample chunks
    int tiles_per_block, pairs_per_block;
    float lw2;             // log2(N / m)
    // CAUSAL
    int64_t leaf, nleaves;
    int levels, tiles_per_leaf, pairs_per_leaf;
    const float *Opart_r, *Lpart_r;
    // outputs
    void *O;
    int out_dtype;
    float *lse, *Opart_w, *Lpart_w;
    int *status;
    int64_t items;
};

struct Item {
    bool valid[2];
    int nc[2];          // key chunks of each tile
    int nc_max;
    // LEVEL
    int64_t prob, blk, bhi, node;
    int pair;
    // CAUSAL
    int64_t leaf_start;   // global row (bhi * n + leaf offset)
    int gt[2];            // tile index within the leaf
};

__device__ __forceinline__ Item decode(const TcArgs &a, int64_t it) {
    Item x{};
    if (a.mode == MODE_LEVEL) {
        const int64_t nblk = a.lv.seg_len / a.lv.bp;
        const int64_t per_prob = nblk * a.pairs_per_block;
        x.prob = it / per_prob;
        const int64_t rem = it % per_prob;
        x.blk = rem / a.pairs_per_block;
        x.pair = static_cast<int>(rem % a.pairs_per_block);
        x.bhi = x.prob / a.lv.nodes;
        x.node = x.prob % a.lv.nodes;
        for (int t = 0; t < 2; ++t) {
            x.valid[t] = x.pair * 2 + t < a.tiles_per_block;
            x.nc[t] = a.nb + a.ns;
        }
        x.nc_max = a.nb + a.ns;
    } else {
        const int64_t per_pair = a.bh * a.nleaves;
        const int pair = a.pairs_per_leaf - 1 - static_cast<int>(it / per_pair);   // heaviest first
        const int64_t rem = it % per_pair;
        x.bhi = rem / a.nleaves;
        const int64_t w = rem % a.nleaves;
        x.leaf_start = x.bhi * a.n + w * a.leaf;
        x.pair = pair;
        x.nc_max = 0;
        for (int t = 0; t < 2; ++t) {
            x.gt[t] = pair * 2 + t;
            x.valid[t] = x.gt[t] < a.tiles_per_leaf;
            x.nc[t] = x.valid[t] ? x.gt[t] + 1 : 0;
            x.nc_max = max(x.nc_max, x.nc[t]);
        }
    }
    return x;
}

template <int D>
struct Smem {
    static constexpr int kSlabs = D / 64;
    static constexpr int kTileBytes = 128 * D * 2;              // one 128-row tile of bf16
    static constexpr int kStages = D == 64 ? 4 : 2;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + 2 * kTileBytes;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kMask = kV + kStages * kTileBytes;
    static constexpr int kBars = kMask + kStages * 16;
    // barrier indices
    static constexpr int bQFull = 0, bQEmpty = 2, bKFull = 4, bVFull = bKFull + kStages,
                         bKVEmpty = bVFull + kStages, bMaskFull = bKVEmpty + kStages, bSFull = bMaskFull + kStages,
                         bPFull = bSFull + 2, bOReady = bPFull + 2, bOFree = bOReady + 2, bDrain = bOFree + 2,
                         kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
};

__device__ __forceinline__ void flag_status(int *status) {
    if (status) atomicOr(status, kStatusTimeout);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const TcArgs a) {
    using L = Smem<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kAbort);
    uint32_t *mask_words = reinterpret_cast<uint32_t *>(sm + L::kMask);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 32) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(L::bQFull + t), 1);
            mbar_init(bar(L::bQEmpty + t), 1);
            mbar_init(bar(L::bSFull + t), 1);
            mbar_init(bar(L::bPFull + t), 128);
            mbar_init(bar(L::bOReady + t), 1);
            mbar_init(bar(L::bOFree + t), 128);
        }
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar(L::bKFull + s), 1);
            mbar_init(bar(L::bVFull + s), 1);
            mbar_init(bar(L::bKVEmpty + s), 1);
            mbar_init(bar(L::bMaskFull + s), 1);
        }
        mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + L::kTmemSlot, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + L::kTmemSlot);

    const int64_t first = blockIdx.x, stride = gridDim.x;

    if (warp == 0) {
        // ------------------------------------------------------------------ loader
        int64_t g = 0;
        int qcnt[2] = {0, 0};
        bool ok = true;
        for (int64_t it = first; it < a.items && ok; it += stride) {
            const Item x = decode(a, it);
            // query tiles
            for (int t = 0; t < 2 && ok; ++t) {
                if (!x.valid[t]) continue;
                if (qcnt[t] > 0 && !mbar_wait(bar(L::bQEmpty + t), (qcnt[t] - 1) & 1, abort_flag)) { ok = false; break; }
                int rows[4];
                if (a.mode == MODE_LEVEL) {
                    const int64_t N = a.lv.seg_len;
                    const int32_t *pq = a.perm + (x.prob * 2) * N + x.blk * a.lv.bp + (x.pair * 2 + t) * 128;
                    const int64_t qbase = x.bhi * a.n + x.node * a.lv.node_len + a.lv.q_off;
                    const int4 v4 = *reinterpret_cast<const int4 *>(pq + 4 * lane);
                    rows[0] = static_cast<int>(qbase + v4.x); rows[1] = static_cast<int>(qbase + v4.y);
                    rows[2] = static_cast<int>(qbase + v4.z); rows[3] = static_cast<int>(qbase + v4.w);
                } else {
                    const int64_t r0 = x.leaf_start + x.gt[t] * 128 + 4 * lane;
                    for (int j = 0; j < 4; ++j) rows[j] = static_cast<int>(r0 + j);
                }
                if (lane == 0) mbar_arrive_expect_tx(bar(L::bQFull + t), L::kTileBytes);
                __syncwarp();
                const uint32_t dst = sbase + L::kQ + t * L::kTileBytes + lane * 512;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_gather4(dst + sl * 16384, &tmQ, sl * 64, rows[0], rows[1], rows[2], rows[3], bar(L::bQFull + t));
                ++qcnt[t];
            }
            if (!ok) break;
            // key / value chunks
            for (int c = 0; c < x.nc_max; ++c, ++g) {
                const int slot = static_cast<int>(g % L::kStages);
                const int64_t round = g / L::kStages;
                if (round > 0 && !mbar_wait(bar(L::bKVEmpty + slot), (round - 1) & 1, abort_flag)) { ok = false; break; }
                int rows[4];
                uint32_t excl = 0;   // bit j: column 4*lane + j masked
                if (a.mode == MODE_LEVEL) {
                    const int64_t N = a.lv.seg_len;
                    const int64_t kbase = x.bhi * a.n + x.node * a.lv.node_len;
                    if (c < a.nb) {
                        const int32_t *pk = a.perm + (x.prob * 2 + 1) * N + x.blk * a.lv.bp + c * 128;
                        const int4 v4 = *reinterpret_cast<const int4 *>(pk + 4 * lane);
                        rows[0] = static_cast<int>(kbase + v4.x); rows[1] = static_cast<int>(kbase + v4.y);
                        rows[2] = static_cast<int>(kbase + v4.z); rows[3] = static_cast<int>(kbase + v4.w);
                    } else {
                        const int32_t *Sp = a.S + (x.bhi * a.nodes_total + (a.lv.heap0 + x.node - 1)) * a.m;
                        const int32_t *ik = a.inv + (x.prob * 2 + 1) * N;
                        for (int j = 0; j < 4; ++j) {
                            const int u = (c - a.nb) * 128 + 4 * lane + j;
                            if (u < a.m) {
                                const int32_t s = Sp[u];
                                rows[j] = static_cast<int>(kbase + s);
                                if (ik[s] / a.lv.bp == x.blk) excl |= 1u << j;
                            } else {
                                rows[j] = static_cast<int>(kbase);
                                excl |= 1u << j;
                            }
                        }
                    }
                } else {
                    const int64_t r0 = x.leaf_start + static_cast<int64_t>(c) * 128 + 4 * lane;
                    for (int j = 0; j < 4; ++j) rows[j] = static_cast<int>(r0 + j);
                }
                uint32_t words[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) words[j] = __ballot_sync(0xffffffffu, (excl >> j) & 1u);
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) mask_words[slot * 4 + j] = words[j];
                    mbar_arrive(bar(L::bMaskFull + slot));
                    mbar_arrive_expect_tx(bar(L::bKFull + slot), L::kTileBytes);
                }
                __syncwarp();
                const uint32_t kdst = sbase + L::kK + slot * L::kTileBytes + lane * 512;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_gather4(kdst + sl * 16384, &tmK, sl * 64, rows[0], rows[1], rows[2], rows[3], bar(L::bKFull + slot));
                if (lane == 0) mbar_arrive_expect_tx(bar(L::bVFull + slot), L::kTileBytes);
                __syncwarp();
                const uint32_t vdst = sbase + L::kV + slot * L::kTileBytes + lane * 512;
#pragma unroll
                for (int sl = 0; sl < L::kSlabs; ++sl)
                    tma_gather4(vdst + sl * 16384, &tmV, sl * 64, rows[0], rows[1], rows[2], rows[3], bar(L::bVFull + slot));
            }
        }
        if (!ok) flag_status(a.status);
        // copies still in flight land before the CTA exits: wait (bounded) for the last round of each slot
        // and the last Q load of each tile
        volatile int no_abort = 0;
        for (int s = 0; s < L::kStages; ++s) {
            const int64_t uses = g > s ? (g - 1 - s) / L::kStages + 1 : 0;   // rounds issued on slot s
            if (uses > 0) {
                mbar_wait(bar(L::bKFull + s), (uses - 1) & 1, &no_abort, 200000000ull);
                mbar_wait(bar(L::bVFull + s), (uses - 1) & 1, &no_abort, 200000000ull);
            }
        }
        for (int t = 0; t < 2; ++t)
            if (qcnt[t] > 0) mbar_wait(bar(L::bQFull + t), (qcnt[t] - 1) & 1, &no_abort, 200000000ull);
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            int64_t g = 0;
            int qcnt[2] = {0, 0}, pcnt[2] = {0, 0}, ocnt[2] = {0, 0};
            bool ok = true;
            auto issue_s = [&](int t, int slot) {
                const uint32_t qa = sbase + L::kQ + t * L::kTileBytes;
                const uint32_t ka = sbase + L::kK + slot * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tmem + t * 128, smem_desc(qa + off, 16, 1024), smem_desc(ka + off, 16, 1024), idesc_qk,
                           kk > 0 ? 1u : 0u);
                }
            };
            for (int64_t it = first; it < a.items && ok; it += stride) {
                const Item x = decode(a, it);
                {
                    const int slot0 = static_cast<int>(g % L::kStages);
                    if (!mbar_wait(bar(L::bKFull + slot0), (g / L::kStages) & 1, abort_flag)) { ok = false; break; }
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (!x.valid[t]) continue;
                        if (!mbar_wait(bar(L::bQFull + t), qcnt[t] & 1, abort_flag)) { ok = false; break; }
                        ++qcnt[t];
                        tc_fence_after();
                        issue_s(t, slot0);
                        mma_commit(bar(L::bSFull + t));
                        if (x.nc[t] == 1) mma_commit(bar(L::bQEmpty + t));
                    }
                    if (!ok) break;
                }
                for (int c = 0; c < x.nc_max && ok; ++c) {
                    const int64_t gc = g + c;
                    const int slot = static_cast<int>(gc % L::kStages);
                    if (!mbar_wait(bar(L::bVFull + slot), (gc / L::kStages) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    for (int t = 0; t < 2; ++t) {
                        if (!x.valid[t] || c >= x.nc[t]) continue;
                        if (!mbar_wait(bar(L::bPFull + t), pcnt[t] & 1, abort_flag)) { ok = false; break; }
                        ++pcnt[t];
                        if (c == 0 && ocnt[t] > 0 &&
                            !mbar_wait(bar(L::bOFree + t), (ocnt[t] - 1) & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t va = sbase + L::kV + slot * L::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tmem + 256 + t * D, tmem + t * 128 + kk * 8, smem_desc(va + kk * 2048, 16384, 1024),
                                   idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(bar(L::bOReady + t));
                        if (c + 1 < x.nc[t]) {
                            const int64_t gn = gc + 1;
                            const int slot1 = static_cast<int>(gn % L::kStages);
                            if (!mbar_wait(bar(L::bKFull + slot1), (gn / L::kStages) & 1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                            issue_s(t, slot1);
                            mma_commit(bar(L::bSFull + t));
                            if (c + 1 == x.nc[t] - 1) mma_commit(bar(L::bQEmpty + t));
                        }
                    }
                    if (!ok) break;
                    mma_commit(bar(L::bKVEmpty + slot));
                }
                g += x.nc_max;
                for (int t = 0; t < 2; ++t)
                    if (x.valid[t]) ++ocnt[t];
            }
            if (!ok) flag_status(a.status);
            // drain: every MMA issued so far has completed before TMEM is released
            mma_commit(bar(L::bDrain));
            volatile int no_abort = 0;
            mbar_wait(bar(L::bDrain), 0, &no_abort, 200000000ull);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ softmax + epilogue
        const int t = (warp - 4) >> 2;
        const int q = warp & 3;                      // TMEM lane quarter
        const int r = q * 32 + lane;                 // row within the tile
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t tS = trow + t * 128;
        const uint32_t tO = trow + 256 + t * D;
        int64_t g = 0;
        int scnt = 0, pvcnt = 0;
        bool ok = true;
        for (int64_t it = first; it < a.items && ok; it += stride) {
            const Item x = decode(a, it);
            if (!x.valid[t]) { g += x.nc_max; continue; }
            float m_run = -INFINITY, l = 0.0f;
            for (int c = 0; c < x.nc[t]; ++c) {
                const int64_t gc = g + c;
                const int slot = static_cast<int>(gc % L::kStages);
                if (!mbar_wait(bar(L::bSFull + t), scnt & 1, abort_flag)) { ok = false; break; }
                ++scnt;
                const bool samp = a.mode == MODE_LEVEL && c >= a.nb;
                const bool diag = a.mode == MODE_CAUSAL && c == x.gt[t];
                uint32_t mw[4] = {0u, 0u, 0u, 0u};
                if (samp) {
                    if (!mbar_wait(bar(L::bMaskFull + slot), (gc / L::kStages) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
                    for (int j = 0; j < 4; ++j) mw[j] = mask_words[slot * 4 + j];
                }
                tc_fence_after();
                const float w2 = samp ? a.lw2 : 0.0f;
                // pass 1: chunk max of the valid columns
                float smax = -INFINITY;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t v[32];
                    tmem_ld32(tS + j * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = j * 32 + e;
                        const bool masked = (samp && ((mw[col & 3] >> (col >> 2)) & 1u)) || (diag && col > r);
                        if (!masked) smax = fmaxf(smax, __uint_as_float(v[e]));
                    }
                }
                const float xmax = smax == -INFINITY ? -INFINITY : fmaf(smax, kLog2e, w2);
                const float m_new = xmax > m_run + kRescaleLog2 ? xmax : m_run;
                const bool grow = m_new != m_run;
                if (grow) {
                    const float alpha = ex2_approx(m_run - m_new);   // 0 when m_run = -inf
                    l *= alpha;
                }
                // rescale O (warp-uniform: lanes whose max did not grow scale by 1)
                if (c > 0 && __any_sync(0xffffffffu, grow)) {
                    const float alpha = grow ? ex2_approx(m_run - m_new) : 1.0f;
                    if (!mbar_wait(bar(L::bOReady + t), (pvcnt - 1) & 1, abort_flag)) { ok = false; }
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t v[32];
                        tmem_ld32(tO + j * 32, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                        tmem_st32(tO + j * 32, v);
                    }
                    tmem_st_wait();
                }
                m_run = m_new;
                // pass 2: P = 2^(x - m_run) in bf16 over S, row sum of the rounded values
                const float off = w2 - m_run;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t v[32];
                    tmem_ld32(tS + j * 32, v);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c0 = j * 32 + 2 * e, c1 = c0 + 1;
                        const bool k0 = (samp && ((mw[c0 & 3] >> (c0 >> 2)) & 1u)) || (diag && c0 > r);
                        const bool k1 = (samp && ((mw[c1 & 3] >> (c1 >> 2)) & 1u)) || (diag && c1 > r);
                        const float p0 = k0 ? 0.0f : ex2_approx(fmaf(__uint_as_float(v[2 * e]), kLog2e, off));
                        const float p1 = k1 ? 0.0f : ex2_approx(fmaf(__uint_as_float(v[2 * e + 1]), kLog2e, off));
                        pk[e] = pack_bf16x2(p0, p1);
                        l += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
                    }
                    tmem_st16(tS + j * 16, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(L::bPFull + t));
                ++pvcnt;
            }
            if (!ok) break;
            // epilogue: wait for the last P V of this tile, then write the row
            if (!mbar_wait(bar(L::bOReady + t), (pvcnt - 1) & 1, abort_flag)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float Lrow = (m_run + __log2f(l)) * kLn2;   // natural log of the row's normaliser
            if (a.mode == MODE_LEVEL) {
                const int64_t N = a.lv.seg_len;
                const int64_t pos = x.blk * a.lv.bp + (x.pair * 2 + t) * 128 + r;
                const int64_t qloc = a.perm[(x.prob * 2) * N + pos];
                if (a.lv.level == 0) {
                    const int64_t orow = x.bhi * a.n + a.lv.q_off + x.node * a.lv.node_len + qloc;
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t v[32];
                        tmem_ld32(tO + j * 32, v);
                        tmem_ld_wait();
                        if (a.out_dtype == 0) {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.O) + orow * D + j * 32);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                uint4 w;
                                w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * inv_l, __uint_as_float(v[8 * e + 1]) * inv_l);
                                w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * inv_l, __uint_as_float(v[8 * e + 3]) * inv_l);
                                w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * inv_l, __uint_as_float(v[8 * e + 5]) * inv_l);
                                w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * inv_l, __uint_as_float(v[8 * e + 7]) * inv_l);
                                dst[e] = w;
                            }
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.O) + orow * D + j * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv_l, __uint_as_float(v[4 * e + 1]) * inv_l,
                                                     __uint_as_float(v[4 * e + 2]) * inv_l, __uint_as_float(v[4 * e + 3]) * inv_l);
                        }
                    }
                    if (a.lse) a.lse[orow] = Lrow;
                } else {
                    const int64_t dense = x.bhi * (a.n / 2) + x.node * N + qloc;
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t v[32];
                        tmem_ld32(tO + j * 32, v);
                        tmem_ld_wait();
                        float4 *dst = reinterpret_cast<float4 *>(a.Opart_w + dense * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(v[4 * e]) * inv_l, __uint_as_float(v[4 * e + 1]) * inv_l,
                                                 __uint_as_float(v[4 * e + 2]) * inv_l, __uint_as_float(v[4 * e + 3]) * inv_l);
                    }
                    a.Lpart_w[dense] = Lrow;
                }
            } else {
                // exact causal leaf part merged with the level parts of this row (log space)
                const int64_t orow = x.leaf_start + x.gt[t] * 128 + r;
                const int64_t bhi = x.bhi, qrow = orow - bhi * a.n;
                const int64_t half_n = a.n / 2;
                float wts[kMaxLevels];
                uint32_t idx[kMaxLevels];
                int np = 0;
                float Lmax = Lrow;
                for (int lvl = 1; lvl <= a.levels && np < kMaxLevels; ++lvl) {
                    const int64_t len = a.n >> (lvl - 1), half = len / 2, within = qrow % len;
                    if (within < half) continue;
                    const int64_t dense = static_cast<int64_t>(lvl - 1) * a.bh * half_n + bhi * half_n +
                                          (qrow / len) * half + (within - half);
                    const float Lp = a.Lpart_r[dense];
                    if (Lp == -INFINITY) continue;
                    wts[np] = Lp;
                    idx[np] = static_cast<uint32_t>(dense);
                    Lmax = fmaxf(Lmax, Lp);
                    ++np;
                }
                const float wb = __expf(Lrow - Lmax);
                float tot = wb;
                for (int i = 0; i < np; ++i) {
                    wts[i] = __expf(wts[i] - Lmax);
                    tot += wts[i];
                }
                const float inv_tot = 1.0f / tot;
                const float cb = wb * inv_l * inv_tot;
#pragma unroll
                for (int j = 0; j < D / 32; ++j) {
                    uint32_t v[32];
                    tmem_ld32(tO + j * 32, v);
                    tmem_ld_wait();
                    float acc[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(v[e]) * cb;
                    for (int i = 0; i < np; ++i) {
                        const float wi = wts[i] * inv_tot;
                        const float4 *src = reinterpret_cast<const float4 *>(a.Opart_r + static_cast<int64_t>(idx[i]) * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 p = src[e];
                            acc[4 * e] += wi * p.x; acc[4 * e + 1] += wi * p.y;
                            acc[4 * e + 2] += wi * p.z; acc[4 * e + 3] += wi * p.w;
                        }
                    }
                    if (a.out_dtype == 0) {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.O) + orow * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint4 w;
                            w.x = pack_bf16x2(acc[8 * e + 0], acc[8 * e + 1]);
                            w.y = pack_bf16x2(acc[8 * e + 2], acc[8 * e + 3]);
                            w.z = pack_bf16x2(acc[8 * e + 4], acc[8 * e + 5]);
                            w.w = pack_bf16x2(acc[8 * e + 6], acc[8 * e + 7]);
                            dst[e] = w;
                        }
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.O) + orow * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(L::bOFree + t));
            g += x.nc_max;
        }
        if (!ok) flag_status(a.status);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------- host side

bool make_gather_map(CUtensorMap *map, const void *base, int64_t rows, int d) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t estr[2] = {1, 1};
    const CUresult rc = cuTensorMapEncodeTiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
                                               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS;
}

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D>
int launch_tc(const void *Q, const void *K, const void *V, const TcArgs &args, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const int64_t rows = args.bh * args.n;
    if (!make_gather_map(&mq, Q, rows, D) || !make_gather_map(&mk, K, rows, D) || !make_gather_map(&mv, V, rows, D))
        return -1;
    const size_t smem = Smem<D>::kBytes + 1024;
    auto kern = attn_tc_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    const int64_t grid = args.items < num_sms() ? args.items : num_sms();
    if (grid <= 0) return 0;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(mq, mk, mv, args);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int dispatch(int d, const void *Q, const void *K, const void *V, const TcArgs &args, cudaStream_t st) {
    if (d == 64) return launch_tc<64>(Q, K, V, args, st);
    if (d == 128) return launch_tc<128>(Q, K, V, args, st);
    return -2;
}

}  // namespace

int launch_attn_tc(const Level &lv, const void *Q, const void *K, const void *V, int d, const int32_t *perm,
                   const int32_t *inv, const int32_t *S, int m, int64_t nodes_total, void *O, int out_dtype,
                   float *lse, float *Opart, float *Lpart, int *status, cudaStream_t st) {
    if ((d != 64 && d != 128) || lv.bp % 128 != 0 || lv.bh * lv.n >= (int64_t(1) << 31)) return -2;
    TcArgs a{};
    a.mode = MODE_LEVEL;
    a.n = lv.n;
    a.bh = lv.bh;
    a.lv = lv;
    a.perm = perm;
    a.inv = inv;
    a.S = S;
    a.m = m;
    a.nodes_total = nodes_total;
    a.nb = lv.bp / 128;
    a.ns = (m + 127) / 128;
    a.tiles_per_block = lv.bp / 128;
    a.pairs_per_block = (a.tiles_per_block + 1) / 2;
    a.lw2 = m > 0 ? log2f(static_cast<float>(lv.seg_len) / static_cast<float>(m)) : 0.0f;
    a.O = O;
    a.out_dtype = out_dtype;
    a.lse = lse;
    a.Opart_w = Opart;
    a.Lpart_w = Lpart;
    a.status = status;
    a.items = lv.bh * lv.nodes * (lv.seg_len / lv.bp) * a.pairs_per_block;
    return dispatch(d, Q, K, V, a, st);
}

int launch_causal_base_tc(const void *Q, const void *K, const void *V, int64_t bh, int64_t n, int d, int64_t leaf,
                          int levels, const float *Opart, const float *Lpart, void *O, int out_dtype, int *status,
                          cudaStream_t st) {
    if ((d != 64 && d != 128) || leaf % 128 != 0 || n % leaf != 0 || levels > kMaxLevels ||
        bh * n >= (int64_t(1) << 31) || static_cast<int64_t>(levels) * bh * (n / 2) >= (int64_t(1) << 32))
        return -2;
    TcArgs a{};
    a.mode = MODE_CAUSAL;
    a.n = n;
    a.bh = bh;
    a.leaf = leaf;
    a.nleaves = n / leaf;
    a.levels = levels;
    a.tiles_per_leaf = static_cast<int>(leaf / 128);
    a.pairs_per_leaf = (a.tiles_per_leaf + 1) / 2;
    a.Opart_r = Opart;
    a.Lpart_r = Lpart;
    a.O = O;
    a.out_dtype = out_dtype;
    a.status = status;
    a.items = bh * a.nleaves * a.pairs_per_leaf;
    return dispatch(d, Q, K, V, a, st);
}

}  // namespace ha
