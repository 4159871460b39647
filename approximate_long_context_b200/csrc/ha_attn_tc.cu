// ha_attn_tc.cu -- tensor-core (tcgen05 / TMEM) attention kernels for bf16 inputs.
//
// Two modes share one persistent kernel:
//
//  LEVEL: the HyperAttention problem of one level ("HyperAttention: Long-context Attention in Near-Linear
//  Time", research-map summary, "Approach"). A work item is a pair of 128-query tiles of one sorted block
//  i. Its key stream is the b'/128 chunks of key block i (exact block part) followed by ceil(m/128) chunks
//  of sampled columns (uniform sample part). The loader compacts the sample list per item: columns whose
//  key lies in block i are already counted exactly and are dropped, the rest keep their order and carry
//  the weight N/m (+ log2(N/m) on the base-2 score); only the tail of the last sample chunk is masked.
//  Rows are read through the sort permutations (the gather) with 16-byte cp.async copies straight into
//  the 128-byte-swizzled layout the tensor core reads, so no permuted copy of Q, K or V exists. One online
//  softmax over both parts gives O = (N1+N2)/(D1+D2); the epilogue writes each row to its original position
//  (the merge and un-permute), or, for causal levels, the fp32 part and its log normaliser.
//
//  LEVEL_RN: LEVEL with row-norm sampling of the product with V ("Approach": rows of V drawn with probability
//  proportional to their squared norms, weight 1/(m p_j)). The key stream gains ceil(m/128) chunks of the
//  row-norm draws outside block i, each column with its own log2 weight; the uniform sample chunks feed only
//  the normaliser (their P.V products are not issued and their V rows not loaded) and the row-norm chunks
//  only the numerator, so O = (N1 + N2') / (D1 + D2).
//
//  CAUSAL: exact causal attention inside leaves of c rows (the summary's recursive causal extension: the
//  base case), merged in log space with the parts of every causal level the row belongs to
//  ("Limitations": partitioning and merging). A work item is a pair of query tiles of one leaf; query tile
//  g sees key chunks 0..g, the last one with the inclusive causal mask. Items run heaviest first.
//
// Work unit of the MMA and softmax roles: a "pair" (query tile t, key chunk c) of 128 x 128 scores. The
// pairs of an item run c-major, t-minor; j counts pairs over a CTA's items. S of pair j lives in TMEM buffer
// j mod R of a ring of R = 2 buffers of 128 columns. d = 64: the softmax writes P (bf16) to a TMEM buffer of
// its tile, and S of pair j + 2 is issued as soon as the softmax has read S of pair j. d = 128: P overwrites
// the first 64 columns of its S buffer, and S of pair j + 2 is issued right after the P.V products of pairs j
// (and j + 1, in groups of two) that read them. The P.V product reads P from TMEM. (On this part an M=128,
// K=16 MMA costs about the same for N = 64 and N = 128, so 128-key chunks halve the cost of the score
// products.)
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warp 0      K loader: 128-row chunks into a ring of NST stages, per-item sample list; publishes each
//               stage's row list for
//   warp 3      V loader: the V rows of the same chunks;
//   warp 2      Q loader: the two query tiles of an item (QB buffers per tile);
//   warp 1      MMA issuer (lane 0);
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: a thread owns one query row (TMEM lane),
//               keeps the running max and sum, rescales O only when the running max grows by more than 2^8,
//               and runs the epilogue.
// Loaders copy with cp.async and arrive on the stage barrier when their copies complete.
// TMEM (512 columns): S ring at [0, 256); d = 64: P of tile t at [256 + 64 t, 320 + 64 t), O of tile t at
// [384 + 64 t, 448 + 64 t); d = 128: O of tile t at [256 + 128 t, 384 + 128 t).
// Every mbarrier wait is bounded; on expiry the kernel sets the status bit, the other warps give up, the
// loaders wait for their copies, the MMA issuer drains the tensor core, and TMEM is freed before exit.
#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"
#include "ha_attn_items.cuh"

namespace ha {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kThreads = 384;

template <int D>
struct Cfg {
    // d = 64: P in TMEM buffers of its own (one per tile), so that the score tile of pair k + R may overwrite
    // S of pair k as soon as the softmax has read it, before P of pair k exists (TMEM: 2 x 128 S columns,
    // 2 x 64 P columns, 2 x 64 O columns). d = 128 writes P over its S (TMEM: 2 x 128 S, 2 x 128 O).
    static constexpr bool kSepP = D == 64;
    static constexpr int R = 2;                        // S ring buffers
    static constexpr int QB = D == 64 ? 2 : 1;         // Q buffers per tile
    static constexpr int NST = D == 64 ? 4 : 2;        // K/V stages
    // P.V products issued per group before the score products that reuse their buffers: two keep a score
    // product from queueing right behind the P.V that reads its buffer (a tensor-pipe stall; d = 128 is bound
    // by the pipe), one gives the second tile its next score tile sooner (d = 64 is bound by the softmax)
    static constexpr int kGroup = D == 64 ? 1 : 2;
    static constexpr int SEG = D == 64 ? 128 : 64;     // bytes per row segment of the staged output stores
    // d = 64: the epilogue stages its output rows in the item's own Q buffer (dead once the tile's last score
    // product has completed; the Q loader refills it only after the epilogue); d = 128 has a stage of its own
    static constexpr bool kStageInQ = D == 64;
    static constexpr int kPCol = R * 128;              // P of tile t at [kPCol + 64 t, kPCol + 64 (t + 1)) (kSepP)
    static constexpr int kOCol = R * 128 + (kSepP ? 128 : 0);   // first O column
    static constexpr int kTileBytes = 128 * D * 2;     // 128 rows of bf16 (a Q tile, a K or a V chunk)
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + 2 * QB * kTileBytes;
    static constexpr int kV = kK + NST * kTileBytes;
    static constexpr int kList = kV + NST * kTileBytes;                    // compacted samples of the item
    static constexpr int kCacheS = kList + kMaxSampleList * 4;             // samples of the current problem
    static constexpr int kCacheB = kCacheS + kMaxSampleList * 4;           // their sorted key block
    static constexpr int kKPerm = kCacheB + kMaxSampleList * 4;            // key rows of the item's block
    static constexpr int kQPerm = kKPerm + kMaxBlock * 4;                  // query rows of one tile
    static constexpr int kRows = kQPerm + 128 * 4;                         // global rows of each stage
    // LEVEL_RN (m <= kMaxSampleListRn): the uniform samples take entries [0, m) of the list and the caches, the
    // row-norm draws [m, 2m); the upper halves hold the draws' log2 weights per problem (cache), per item (list)
    // and per stage column
    static constexpr int kCacheW = kCacheS + (kMaxSampleList / 2) * 4;
    static constexpr int kListW = kList + (kMaxSampleList / 2) * 4;
    static constexpr int kStageW = kCacheB + (kMaxSampleList / 2) * 4;
    static constexpr int kZeroW = kCacheW + kMaxSampleListRn * 4;         // 128 zero weights (block chunks)
    static constexpr int kWord = kRows + NST * 128 * 4;
    static constexpr int kStage = (kWord + NST * 4 + 64 + 15) / 16 * 16;   // 8 softmax warps x 32 rows x SEG
    static constexpr int kBars = kStage + (kStageInQ ? 0 : 8 * 32 * SEG);
    static constexpr int bQFull = 0, bQEmpty = bQFull + 2 * QB, bKVFull = bQEmpty + 2 * QB,
                         bKVEmpty = bKVFull + NST, bWordFull = bKVEmpty + NST, bRowsFull = bWordFull + NST,
                         bSFull = bRowsFull + NST,
                         bPFull = bSFull + R, bPVDone = bPFull + R, bPVDoneT = bPVDone + R, bOFree = bPVDoneT + 4,
                         bDrain = bOFree + 2, bQStage = bDrain + 2, bSFree = bQStage + 2 * QB, bPFullT = bSFree + R,
                         bNever = bPFullT + 2, kNumBars = bNever + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static_assert(kBars % 8 == 0, "mbarriers need 8-byte alignment");
    static_assert(kStage % 16 == 0, "16-byte stage pieces");
    static_assert(!kStageInQ || 4 * 32 * SEG <= kTileBytes, "a tile's four warps stage in its Q buffer");
    static_assert(kBytes + 1024 <= 232448, "shared memory budget");
    static_assert(2 * kMaxSampleListRn <= kMaxSampleList / 2 && NST * 128 <= kMaxSampleList / 2 &&
                      kMaxSampleListRn + 128 <= kMaxSampleList / 2,
                  "row-norm entries fit in the lower halves, their weights in the upper halves");
    static_assert(kOCol + 2 * D <= 512, "TMEM budget");
};

// about 4% faster than one instance for both modes).
template <int D, int MODE, bool HOOK>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const TcArgs a) {
    using C = Cfg<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    auto bar = [&](int i) -> uint32_t { return sbase + C::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::kAbort);
    int *words = reinterpret_cast<int *>(sm + C::kWord);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (MODE == MODE_LEVEL_RN && threadIdx.x < kKC) reinterpret_cast<float *>(sm + C::kZeroW)[threadIdx.x] = 0.0f;
    if (threadIdx.x == 32) {
        for (int i = 0; i < 2 * C::QB; ++i) {
            mbar_init(bar(C::bQFull + i), 32);     // the Q loader's lanes (copy completion)
            mbar_init(bar(C::bQEmpty + i), 1);
            mbar_init(bar(C::bQStage + i), 128);   // the tile's softmax threads, after an epilogue staged there
        }
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(bar(C::bKVFull + s), 64);    // the K and V loader warps' lanes (copy completion)
            mbar_init(bar(C::bRowsFull + s), 1);
            mbar_init(bar(C::bKVEmpty + s), 1);
            mbar_init(bar(C::bWordFull + s), 1);
        }
        for (int b = 0; b < C::R; ++b) {
            mbar_init(bar(C::bSFull + b), 1);
            mbar_init(bar(C::bPFull + b), 128);
            mbar_init(bar(C::bSFree + b), 128);    // kSepP: the softmax threads of the pair's tile have read S
        }
        for (int b = 0; b < C::R; ++b) mbar_init(bar(C::bPVDone + b), 1);
        for (int i = 0; i < 4; ++i) mbar_init(bar(C::bPVDoneT + i), 1);
        for (int t = 0; t < 2; ++t) mbar_init(bar(C::bPFullT + t), 128);   // kSepP: P of a tile's pair written
        mbar_init(bar(C::bNever), 1);              // nothing arrives: the test hook's wait never completes
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(C::bDrain + t), 1);
            mbar_init(bar(C::bOFree + t), 128);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + C::kTmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + C::kTmemSlot);

    // LEVEL items all cost the same: each CTA takes a contiguous range, so consecutive items share a problem
    // and its cached samples. CAUSAL items are ordered heaviest first and dealt round-robin.
    int64_t first, last, stride;
    if (is_level(MODE)) {
        const int64_t per = (a.items + gridDim.x - 1) / gridDim.x;
        first = static_cast<int64_t>(blockIdx.x) * per;
        last = min(a.items, first + per);
        stride = 1;
    } else {
        first = blockIdx.x;
        last = a.items;
        stride = gridDim.x;
    }


    // Q tiles: tile t of an item into Q buffer qc mod QB of that tile, after the buffer's previous user (the
    // tile's score products and, with the epilogue staged there, its epilogue) is done with it
    int qc0 = 0, qc1 = 0;
    auto load_q_tile = [&](const Item &x, int t) -> bool {
        int32_t *qperm = reinterpret_cast<int32_t *>(sm + C::kQPerm);
        int &qc = t == 0 ? qc0 : qc1;
        const int qb = qc % C::QB;
        const int use = qc / C::QB;
        if (use > 0 && !mbar_wait(bar(C::bQEmpty + t * C::QB + qb), (use - 1) & 1, abort_flag)) return false;
        if (C::kStageInQ && use > 0 && !mbar_wait(bar(C::bQStage + t * C::QB + qb), (use - 1) & 1, abort_flag))
            return false;
        const uint32_t base = sbase + C::kQ + (t * C::QB + qb) * C::kTileBytes;
        int64_t qbase;
        const bool through_perm = is_level(MODE);
        if (through_perm) {
            // the tile's 128 query rows: one 16-byte load per lane, staged in shared memory
            const int32_t *pq = a.perm + (x.prob * 2) * a.lv.seg_len + x.blk * a.lv.bp + (x.pair * 2 + t) * 128;
            __syncwarp();
            reinterpret_cast<int4 *>(qperm)[lane] = reinterpret_cast<const int4 *>(pq)[lane];
            check_indices(qperm, 128, a.lv.seg_len, a.status, lane);
            __syncwarp();
            qbase = x.bhi * a.n + x.node * a.lv.node_len + a.lv.q_off;
        } else {
            qbase = x.leaf_start + static_cast<int64_t>(t == 0 ? x.gt0 : x.gt1) * 128;
        }
        if (through_perm) gather_rows<D, true>(base, a.Q, qbase, qperm, lane);
        else gather_rows<D, false>(base, a.Q, qbase, qperm, lane);
        cp_async_arrive(bar(C::bQFull + t * C::QB + qb));
        ++qc;
        return true;
    };

    if (warp == 2) {
        // ------------------------------------------------------------------ Q loader
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride) {
            const Item x = decode<MODE>(a, it);
            if (x.v0) ok = load_q_tile(x, 0);
            if (ok && x.v1) ok = load_q_tile(x, 1);
        }
        cp_wait<0>();
        if (!ok) flag_status(a.status);
    } else if (warp == 0) {
        // ------------------------------------------------------------------ K/V loader
        const unsigned lt_mask = (1u << lane) - 1u;
        int32_t *slist = reinterpret_cast<int32_t *>(sm + C::kList);
        int32_t *cache_s = reinterpret_cast<int32_t *>(sm + C::kCacheS);
        int32_t *cache_b = reinterpret_cast<int32_t *>(sm + C::kCacheB);
        int32_t *kperm = reinterpret_cast<int32_t *>(sm + C::kKPerm);
        int32_t *stage_rows = reinterpret_cast<int32_t *>(sm + C::kRows);
        float *cache_w = reinterpret_cast<float *>(sm + C::kCacheW);
        float *list_w = reinterpret_cast<float *>(sm + C::kListW);
        float *stage_w = reinterpret_cast<float *>(sm + C::kStageW);
        int64_t cached_prob = -1;
        uint32_t g = 0;
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride) {
            const Item x = decode<MODE>(a, it);
            // key rows of block blk and the compacted sample list of this item: the sampled columns whose key
            // lies outside block blk, in sample order (from the per-problem cache of samples and their blocks)
            int cnt = 0, cnt_rn = 0;
            int64_t kbase = 0;
            if (is_level(MODE)) {
                kbase = x.bhi * a.n + x.node * a.lv.node_len;
                const int32_t *pkg = a.perm + (x.prob * 2 + 1) * a.lv.seg_len + x.blk * a.lv.bp;
                __syncwarp();
                for (int i = lane; i < a.lv.bp / 4; i += 32)
                    reinterpret_cast<int4 *>(kperm)[i] = reinterpret_cast<const int4 *>(pkg)[i];
                check_indices(kperm, a.lv.bp, a.lv.seg_len, a.status, lane);
                if (a.ns > 0) {
                    if (x.prob != cached_prob) {
                        const int32_t *Sp = a.S + (x.bhi * a.nodes_total + (a.lv.heap0 + x.node - 1)) * a.m;
                        const int32_t *ik = a.inv + (x.prob * 2 + 1) * a.lv.seg_len;
                        __syncwarp();
                        for (int u = lane; u < a.m; u += 32)
                            cache_s[u] = checked_index(Sp[u], a.lv.seg_len, a.status);
                        __syncwarp();
                        for (int u = lane; u < a.m; u += 32) cache_b[u] = ik[cache_s[u]] / a.lv.bp;
                        if (MODE == MODE_LEVEL_RN) {
                            // row-norm draws of this problem behind the uniform samples; -1 (no draw) never kept
                            const int64_t so = (x.bhi * a.nodes_total + (a.lv.heap0 + x.node - 1)) * a.m;
                            for (int u = lane; u < a.m; u += 32) {
                                const int32_t sr = a.Srn[so + u];   // -1: no draw
                                cache_s[a.m + u] = sr < 0 ? sr : checked_index(sr, a.lv.seg_len, a.status);
                                cache_w[u] = a.lwrn[so + u] * kLog2e;
                            }
                            __syncwarp();
                            for (int u = lane; u < a.m; u += 32) {
                                const int32_t sr = cache_s[a.m + u];
                                cache_b[a.m + u] = sr < 0 ? -1 : ik[sr] / a.lv.bp;
                            }
                        }
                        cached_prob = x.prob;
                    }
                    __syncwarp();
                    for (int base = 0; base < a.m; base += 32) {
                        const int u = base + lane;
                        const bool keep = u < a.m && cache_b[u] != x.blk;
                        const unsigned bal = __ballot_sync(0xffffffffu, keep);
                        if (keep) slist[cnt + __popc(bal & lt_mask)] = cache_s[u];
                        cnt += __popc(bal);
                    }
                    if (MODE == MODE_LEVEL_RN) {
                        for (int base = 0; base < a.m; base += 32) {
                            const int u = base + lane;
                            const bool keep = u < a.m && cache_s[a.m + u] >= 0 && cache_b[a.m + u] != x.blk;
                            const unsigned bal = __ballot_sync(0xffffffffu, keep);
                            if (keep) {
                                const int at = cnt_rn + __popc(bal & lt_mask);
                                slist[a.m + at] = cache_s[a.m + u];
                                list_w[at] = cache_w[u];
                            }
                            cnt_rn += __popc(bal);
                        }
                    }
                }
                __syncwarp();
            }
            for (int c = 0; c < x.nc_max; ++c, ++g) {
                const int slot = static_cast<int>(g % C::NST);
                const uint32_t round = g / C::NST;
                if (round > 0 && !mbar_wait(bar(C::bKVEmpty + slot), (round - 1) & 1, abort_flag)) { ok = false; break; }
                int valid_cols = kKC;
                // 0: block chunk (through the key permutation), 1: sample chunk, 2: contiguous, 3: row-norm chunk
                int kind;
                int u0 = 0;
                if (is_level(MODE)) {
                    if (c < a.nb) {
                        kind = 0;
                    } else if (c < a.nb + a.ns) {
                        kind = 1;
                        u0 = (c - a.nb) * kKC;
                        valid_cols = min(kKC, max(0, cnt - u0));
                    } else {
                        kind = 3;
                        u0 = (c - a.nb - a.ns) * kKC;
                        valid_cols = min(kKC, max(0, cnt_rn - u0));
                        if (MODE == MODE_LEVEL_RN) {
                            for (int row = lane; row < kKC; row += 32)
                                stage_w[slot * kKC + row] = row + u0 < cnt_rn ? list_w[u0 + row] : 0.0f;
                            __syncwarp();
                        }
                    }
                } else {
                    kind = 2;
                }
                if (lane == 0) {
                    words[slot] = valid_cols;
                    mbar_arrive(bar(C::bWordFull + slot));
                }
                // the chunk's 128 global rows, published for the V loader
                const int64_t cbase = is_level(MODE) ? kbase : x.leaf_start + static_cast<int64_t>(c) * kKC;
                int32_t *rows = stage_rows + slot * 128;
                for (int row = lane; row < kKC; row += 32) {
                    int32_t loc;
                    if (kind == 0) loc = kperm[c * kKC + row];
                    else if (kind == 1) loc = row + u0 < cnt ? slist[u0 + row] : 0;
                    else if (kind == 3) loc = row + u0 < cnt_rn ? slist[a.m + u0 + row] : 0;
                    else loc = row;
                    rows[row] = static_cast<int32_t>(cbase + loc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::bRowsFull + slot));
                const uint32_t kb = sbase + C::kK + slot * C::kTileBytes;
                gather_rows<D, true>(kb, a.K, 0, rows, lane);
                cp_async_arrive(bar(C::bKVFull + slot));
            }
        }
        cp_wait<0>();
        if (!ok) flag_status(a.status);
    } else if (warp == 3) {
        // ------------------------------------------------------------------ V loader
        // follows the K loader's chunk sequence: waits for each stage's row list, copies the V rows
        const int32_t *stage_rows = reinterpret_cast<const int32_t *>(sm + C::kRows);
        uint32_t g = 0;
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride) {
            const Item x = decode<MODE>(a, it);
            for (int c = 0; c < x.nc_max; ++c, ++g) {
                const int slot = static_cast<int>(g % C::NST);
                if (!mbar_wait(bar(C::bRowsFull + slot), (g / C::NST) & 1, abort_flag)) { ok = false; break; }
                if (MODE == MODE_LEVEL_RN && c >= a.nb && c < a.nb + a.ns) {
                    // uniform samples feed only the normaliser: no P.V product reads this stage's V
                    mbar_arrive(bar(C::bKVFull + slot));
                    continue;
                }
                const int32_t *rows = stage_rows + slot * 128;
                const uint32_t vb = sbase + C::kV + slot * C::kTileBytes;
                gather_rows<D, true>(vb, a.V, 0, rows, lane);
                cp_async_arrive(bar(C::bKVFull + slot));
            }
        }
        cp_wait<0>();
        if (!ok) flag_status(a.status);
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (score and P.V products)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, kKC, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            // descriptors are built once; an MMA only adds a byte offset >> 4 to the start-address field
            const uint64_t dq0 = smem_desc(sbase + C::kQ, 16, 1024);
            const uint64_t dk0 = smem_desc(sbase + C::kK, 16, 1024);
            const uint64_t dv0 = smem_desc(sbase + C::kV, 128 * 128, 1024);
            // An item in flight: its chunks/pairs offsets, the Q buffer of each tile (-1: not yet waited for)
            // and how many of its score tiles are already issued. Score tiles run ahead across item
            // boundaries: once the current item has issued all of its S products, the next item's first
            // ones go out while the current item's last P.V products wait for their P.
            struct Flight {
                Item x;
                uint32_t g, kp;
                int qb0, qb1;
                int pre;
            };
            int oc0 = 0, oc1 = 0;
            uint32_t pvn0 = 0, pvn1 = 0;   // P.V products issued per tile
            bool ok = true;
            // wait for (blocking) or test (non-blocking) the Q tile of tile t of item f; false if not ready
            auto get_q = [&](Flight &f, int t, bool block) -> bool {
                int &qb = t == 0 ? f.qb0 : f.qb1;
                if (qb >= 0) return true;
                int &qc = t == 0 ? qc0 : qc1;
                const uint32_t b = bar(C::bQFull + t * C::QB + qc % C::QB);
                const uint32_t par = (qc / C::QB) & 1;
                if (block) {
                    if (!mbar_wait(b, par, abort_flag)) { ok = false; return false; }
                } else if (!mbar_try_wait(b, par)) {
                    return false;
                }
                qb = qc % C::QB;
                ++qc;
                return true;
            };
            auto issue_s = [&](Flight &f, int k) -> bool {
                int t, c;
                pair_tc(f.x, k, t, c);
                const uint32_t gc = f.g + c;
                const int slot = static_cast<int>(gc % C::NST);
                if (!mbar_wait(bar(C::bKVFull + slot), (gc / C::NST) & 1, abort_flag)) return false;
                tc_fence_after();
                const int buf = static_cast<int>((f.kp + static_cast<uint32_t>(k)) % C::R);
                const int qb = t == 0 ? f.qb0 : f.qb1;
                const uint64_t dq = dq0 + static_cast<uint64_t>(((t * C::QB + qb) * C::kTileBytes) >> 4);
                const uint64_t dk = dk0 + static_cast<uint64_t>((slot * C::kTileBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
                    mma_ss(tmem + buf * 128, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(C::bSFull + buf));
                // last score tile of this query tile in this item: its Q buffer may be refilled
                if (c == (t == 0 ? f.x.nc0 : f.x.nc1) - 1) mma_commit(bar(C::bQEmpty + t * C::QB + qb));
                ++f.pre;
                return true;
            };
            Flight cur{}, nxt{};
            bool have_next = false;
            if (first < last) {
                cur.x = decode<MODE>(a, first);
                cur.g = 0; cur.kp = 0; cur.qb0 = -1; cur.qb1 = -1; cur.pre = 0;
            }
            for (int64_t it = first; it < last && ok; it += stride) {
                const Item &x = cur.x;
                const int np = x.npairs;
                // score tiles of this item not yet issued by the previous item's look-ahead
                for (int k = cur.pre; k < np && k < C::R && ok; ++k) {
                    int t, c;
                    pair_tc(x, k, t, c);
                    if (!get_q(cur, t, true)) break;
                    ok = issue_s(cur, k);
                }
                have_next = it + stride < last;
                if (have_next) {
                    nxt.x = decode<MODE>(a, it + stride);
                    nxt.g = cur.g + x.nc_max;
                    nxt.kp = cur.kp + np;
                    nxt.qb0 = -1; nxt.qb1 = -1; nxt.pre = 0;
                }
                bool look = have_next;   // look-ahead into the next item still possible
                // the score tile R pairs ahead, in this item or (look-ahead) in the next one
                auto issue_ahead = [&](int ka) {
                    if (ka < np) {
                        ok = issue_s(cur, ka);
                    } else if (look) {
                        const int kn = ka - np;
                        if (kn == nxt.pre && kn < nxt.x.npairs) {
                            int tn, cn;
                            pair_tc(nxt.x, kn, tn, cn);
                            // with one Q buffer per tile, the next Q is loaded only after this item's last S:
                            // take it only if it is already there
                            if (get_q(nxt, tn, C::QB > 1)) ok = issue_s(nxt, kn);
                            else look = false;
                        } else {
                            look = false;
                        }
                    }
                };
                for (int k = 0; k < np && ok; ++k) {
                    int t, c;
                    pair_tc(x, k, t, c);
                    const uint32_t gc = cur.g + c;
                    const int slot = static_cast<int>(gc % C::NST);
                    const uint32_t kk_all = cur.kp + static_cast<uint32_t>(k);
                    const int buf = static_cast<int>(kk_all % C::R);
                    uint32_t &pvn = t == 0 ? pvn0 : pvn1;
                    if (C::kSepP) {
                        // S of pair k has been read: its buffer takes the score tile R pairs ahead
                        if (!mbar_wait(bar(C::bSFree + buf), (kk_all / C::R) & 1, abort_flag)) { ok = false; break; }
                        issue_ahead(k + C::R);
                        if (!ok) break;
                        if (!mbar_wait(bar(C::bPFullT + t), pvn & 1, abort_flag)) { ok = false; break; }
                    } else if (!mbar_wait(bar(C::bPFull + buf), (kk_all / C::R) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int oc = t == 0 ? oc0 : oc1;
                    if (c == 0 && oc > 0 && !mbar_wait(bar(C::bOFree + t), (oc - 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    // V of chunk c arrived with K (one barrier per stage), which S of this pair waited for
                    const uint64_t dv = dv0 + static_cast<uint64_t>((slot * C::kTileBytes) >> 4);
                    const uint32_t od = tmem + C::kOCol + t * D;
                    // LEVEL_RN: the uniform sample chunks have no P.V product (the commits below still arrive)
                    const bool pv = MODE != MODE_LEVEL_RN || c < a.nb || c >= a.nb + a.ns;
                    if (pv) {
#pragma unroll
                        for (int kk = 0; kk < kKC / 16; ++kk) {
                            const uint32_t pa =
                                C::kSepP ? tmem + C::kPCol + t * 64 + kk * 8 : tmem + buf * 128 + kk * 8;
                            mma_ts(od, pa, dv + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                                   (c > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    // the tile's n-th P.V arrives on barrier 2t + (n & 1), phase n >> 1 (with P apart, this also
                    // frees the tile's P buffer)
                    mma_commit(bar(C::bPVDoneT + 2 * t + (pvn & 1)));
                    ++pvn;
                    // the chunk's stage is free once every tile that uses it has issued its P.V
                    const bool last_user = t == 1 || c >= x.nc1;
                    if (last_user) mma_commit(bar(C::bKVEmpty + slot));
                    // P over S: the ring buffers of this pair group (kGroup = 2: pairs k-1 and k, or k alone at an
                    // odd end) are free again: fill them with the score tiles R pairs ahead
                    if (!C::kSepP && (C::kGroup == 1 || (k & 1) || k == np - 1)) {
                        for (int kg = (C::kGroup == 2 && (k & 1)) ? k - 1 : k; kg <= k && ok; ++kg) issue_ahead(kg + C::R);
                    }
                }
                if (x.v0) ++oc0;
                if (x.v1) ++oc1;
                if (have_next) cur = nxt;
            }
            if (!ok) flag_status(a.status);
            mma_commit(bar(C::bDrain));   // every MMA issued so far completes before TMEM is released
            volatile int no_abort = 0;
            mbar_wait(bar(C::bDrain), 0, &no_abort, 200000000ull);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ softmax + epilogue
        const int t = (warp - 4) >> 2;
        const int q = warp & 3;                      // TMEM lane quarter
        const int r = q * 32 + lane;                 // row within the tile
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t tO = trow + C::kOCol + t * D;
        uint32_t kp = 0, g = 0;
        uint32_t pvt = 0;                            // P.V products of this tile before the current item
        int qn = 0;                                  // items of this tile so far (its Q buffer is qn mod QB)
        bool ok = true;
        // test hook (its own instance: the check alone, even outside the chunk loop, measured about 15% slower
        // on the long workload): the first wait targets a barrier nothing completes; it runs out, sets the
        // abort flag, and every role stops
        if (HOOK && a.stall_ns > 0 && first < last &&
            !mbar_wait(bar(C::bNever), 0, abort_flag, static_cast<uint64_t>(a.stall_ns)))
            ok = false;
        for (int64_t it = first; it < last && ok; it += stride) {
            const Item x = decode<MODE>(a, it);
            const bool my_valid = t == 0 ? x.v0 : x.v1;
            const int my_nc = t == 0 ? x.nc0 : x.nc1;
            const int my_gt = t == 0 ? x.gt0 : x.gt1;
            if (!my_valid) { kp += x.npairs; g += x.nc_max; continue; }
            int64_t qloc = 0;
            if (is_level(MODE)) {
                const int64_t pos = x.blk * a.lv.bp + (x.pair * 2 + t) * 128 + r;
                // consumed by the epilogue
                qloc = checked_index(a.perm[(x.prob * 2) * a.lv.seg_len + pos], a.lv.seg_len, a.status);
            }
            float m_run = -INFINITY, l = 0.0f;
            for (int c = 0; c < my_nc; ++c) {
                const uint32_t k = kp + static_cast<uint32_t>(pair_index(x, t, c));
                const int buf = static_cast<int>(k % C::R);
                const uint32_t tS = trow + buf * 128;
                if (!mbar_wait(bar(C::bSFull + buf), (k / C::R) & 1, abort_flag)) { ok = false; break; }
                // column bound: columns > bound are masked (bound >= 127: none)
                int bound = kKC - 1;
                float w2 = 0.0f;
                // LEVEL_RN: uniform sample chunks add to the normaliser only (no P is written), row-norm chunks
                // (per-column log2 weights) to the numerator only
                bool to_l = true, to_o = true;
                // LEVEL_RN: every chunk's scores get per-column log2 weights, wcol[col] + w2 (zero for block
                // chunks, log2(N/m) for uniform sample chunks, the draws' weights for row-norm chunks), so that
                // the softmax runs one code path for all chunk kinds
                const float *wcol = reinterpret_cast<const float *>(sm + C::kZeroW);
                if (is_level(MODE)) {
                    if (c >= a.nb) {
                        const uint32_t gc = g + c;
                        const int slot = static_cast<int>(gc % C::NST);
                        if (!mbar_wait(bar(C::bWordFull + slot), (gc / C::NST) & 1, abort_flag)) { ok = false; break; }
                        bound = words[slot] - 1;
                        if (MODE != MODE_LEVEL_RN || c < a.nb + a.ns) {
                            w2 = a.lw2;
                            to_o = MODE != MODE_LEVEL_RN;
                        } else {
                            wcol = reinterpret_cast<const float *>(sm + C::kStageW) + slot * kKC;
                            to_l = false;
                        }
                    }
                } else {
                    bound = MODE == MODE_DENSE ? kKC - 1 : my_gt * 128 + r - c * kKC;
                }
                tc_fence_after();
                const bool masked = __any_sync(0xffffffffu, bound < kKC - 1);
                // pass 1: row max, 64 columns at a time (registers stay below the spill limit)
                float smax = -INFINITY;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t va[32], vb[32];
                    tmem_ld32(tS + h * 64, va);
                    tmem_ld32(tS + h * 64 + 32, vb);
                    tmem_ld_wait();
                    if (masked) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (h * 64 + e > bound) va[e] = 0xff800000u;   // -inf
                            if (h * 64 + 32 + e > bound) vb[e] = 0xff800000u;
                        }
                    }
                    if (MODE == MODE_LEVEL_RN) {
                        // weighted base-2 scores (a masked -inf stays -inf); smax then holds the weighted max
                        const float4 *w4 = reinterpret_cast<const float4 *>(wcol + h * 64);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 wa = w4[e], wb = w4[8 + e];
                            va[4 * e] = __float_as_uint(fmaf(__uint_as_float(va[4 * e]), kLog2e, wa.x + w2));
                            va[4 * e + 1] = __float_as_uint(fmaf(__uint_as_float(va[4 * e + 1]), kLog2e, wa.y + w2));
                            va[4 * e + 2] = __float_as_uint(fmaf(__uint_as_float(va[4 * e + 2]), kLog2e, wa.z + w2));
                            va[4 * e + 3] = __float_as_uint(fmaf(__uint_as_float(va[4 * e + 3]), kLog2e, wa.w + w2));
                            vb[4 * e] = __float_as_uint(fmaf(__uint_as_float(vb[4 * e]), kLog2e, wb.x + w2));
                            vb[4 * e + 1] = __float_as_uint(fmaf(__uint_as_float(vb[4 * e + 1]), kLog2e, wb.y + w2));
                            vb[4 * e + 2] = __float_as_uint(fmaf(__uint_as_float(vb[4 * e + 2]), kLog2e, wb.z + w2));
                            vb[4 * e + 3] = __float_as_uint(fmaf(__uint_as_float(vb[4 * e + 3]), kLog2e, wb.w + w2));
                        }
                    }
                    float mx0 = __uint_as_float(va[0]), mx1 = __uint_as_float(vb[0]);
#pragma unroll
                    for (int e = 1; e < 32; ++e) {
                        mx0 = fmaxf(mx0, __uint_as_float(va[e]));
                        mx1 = fmaxf(mx1, __uint_as_float(vb[e]));
                    }
                    smax = fmaxf(smax, fmaxf(mx0, mx1));
                }
                const float xmax = smax == -INFINITY ? -INFINITY
                                   : MODE == MODE_LEVEL_RN ? smax
                                                                                : fmaf(smax, kLog2e, w2);
                const float m_new = xmax > m_run + kRescaleLog2 ? xmax : m_run;
                const bool grow = m_new != m_run;
                const float alpha = grow ? ex2_approx(m_run - m_new) : 1.0f;   // 0 when m_run = -inf
                l *= alpha;
                if (c > 0 && __any_sync(0xffffffffu, grow)) {
                    // O holds P.V of chunks 0..c-1: wait for the last of them (chunk c-1) before scaling it
                    const uint32_t nprev = pvt + static_cast<uint32_t>(c) - 1;
                    if (!mbar_wait(bar(C::bPVDoneT + 2 * t + (nprev & 1)), (nprev >> 1) & 1, abort_flag)) ok = false;
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t o[32];
                        tmem_ld32(tO + j * 32, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tO + j * 32, o);
                    }
                    tmem_st_wait();
                }
                m_run = m_new;
                const float off = w2 - m_run;
                float l0 = 0.0f, l1 = 0.0f;
                // pass 2: P = 2^(x - m_run) in bf16, 64 columns: over the first 64 columns of the S buffer (keys
                // 0-63 land in columns 0-31, already read; keys 64-127 in columns 32-63, read by the first half),
                // or (kSepP) into the tile's P buffer once the tile's previous P.V has read it
                const uint32_t tP = C::kSepP ? trow + C::kPCol + t * 64 : tS;
                if (C::kSepP && pvt + static_cast<uint32_t>(c) > 0) {
                    const uint32_t nprev = pvt + static_cast<uint32_t>(c) - 1;
                    if (!mbar_wait(bar(C::bPVDoneT + 2 * t + (nprev & 1)), (nprev >> 1) & 1, abort_flag)) ok = false;
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t va[32], vb[32];
                    tmem_ld32(tS + h * 64, va);
                    tmem_ld32(tS + h * 64 + 32, vb);
                    tmem_ld_wait();
                    if (C::kSepP && h == 1) {
                        // all of S has been read: the buffer may take the next score tile
                        tc_fence_before();
                        mbar_arrive(bar(C::bSFree + buf));
                    }
                    if (masked) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (h * 64 + e > bound) va[e] = 0xff800000u;
                            if (h * 64 + 32 + e > bound) vb[e] = 0xff800000u;
                        }
                    }
                    uint32_t pk[32];
                    if (MODE == MODE_LEVEL_RN) {
                        // P = 2^(x log2 e + w_col + w2 - m_run)
                        const float4 *w4 = reinterpret_cast<const float4 *>(wcol + h * 64);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 wa = w4[e], wb = w4[8 + e];
                            const float a0 = ex2_approx(fmaf(__uint_as_float(va[4 * e]), kLog2e, wa.x + off));
                            const float a1 = ex2_approx(fmaf(__uint_as_float(va[4 * e + 1]), kLog2e, wa.y + off));
                            const float a2 = ex2_approx(fmaf(__uint_as_float(va[4 * e + 2]), kLog2e, wa.z + off));
                            const float a3 = ex2_approx(fmaf(__uint_as_float(va[4 * e + 3]), kLog2e, wa.w + off));
                            const float b0 = ex2_approx(fmaf(__uint_as_float(vb[4 * e]), kLog2e, wb.x + off));
                            const float b1 = ex2_approx(fmaf(__uint_as_float(vb[4 * e + 1]), kLog2e, wb.y + off));
                            const float b2 = ex2_approx(fmaf(__uint_as_float(vb[4 * e + 2]), kLog2e, wb.z + off));
                            const float b3 = ex2_approx(fmaf(__uint_as_float(vb[4 * e + 3]), kLog2e, wb.w + off));
                            l0 += (a0 + a1) + (a2 + a3);
                            l1 += (b0 + b1) + (b2 + b3);
                            pk[2 * e] = pack_bf16x2(a0, a1);
                            pk[2 * e + 1] = pack_bf16x2(a2, a3);
                            pk[16 + 2 * e] = pack_bf16x2(b0, b1);
                            pk[16 + 2 * e + 1] = pack_bf16x2(b2, b3);
                        }
                    } else {
                        // scale-and-offset and sums as packed f32x2 instructions, the exponentials on the MUFU unit
                        const uint64_t sc = f2_pack(kLog2e, kLog2e), of = f2_pack(off, off);
                        uint64_t sa = f2_pack(0.0f, 0.0f), sb = sa;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float2 xa =
                                f2_unpack(f2_fma(f2_pack(__uint_as_float(va[2 * e]), __uint_as_float(va[2 * e + 1])), sc, of));
                            const float2 xb =
                                f2_unpack(f2_fma(f2_pack(__uint_as_float(vb[2 * e]), __uint_as_float(vb[2 * e + 1])), sc, of));
                            const float p0 = ex2_approx(xa.x), p1 = ex2_approx(xa.y);
                            const float p2 = ex2_approx(xb.x), p3 = ex2_approx(xb.y);
                            sa = f2_add(sa, f2_pack(p0, p1));
                            sb = f2_add(sb, f2_pack(p2, p3));
                            pk[e] = pack_bf16x2(p0, p1);
                            pk[16 + e] = pack_bf16x2(p2, p3);
                        }
                        const float2 ta = f2_unpack(sa), tb = f2_unpack(sb);
                        l0 += ta.x + ta.y;
                        l1 += tb.x + tb.y;
                    }
                    if (to_o) tmem_st32(tP + h * 32, pk);
                }
                if (to_l) l += l0 + l1;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(C::kSepP ? C::bPFullT + t : C::bPFull + buf));
            }
            if (!ok) break;
            // epilogue: wait for the tile's last P.V of this item, then write the row
            const uint32_t nlast = pvt + static_cast<uint32_t>(my_nc) - 1;
            if (!mbar_wait(bar(C::bPVDoneT + 2 * t + (nlast & 1)), (nlast >> 1) & 1, abort_flag)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            pvt += static_cast<uint32_t>(my_nc);
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float Lrow = (m_run + __log2f(l)) * kLn2;   // natural log of the row's normaliser
            const int qbuf = t * C::QB + qn % C::QB;
            unsigned char *stage = C::kStageInQ ? sm + C::kQ + qbuf * C::kTileBytes + q * (32 * C::SEG)
                                                : sm + C::kStage + (warp - 4) * (32 * C::SEG);
            auto o_scaled = [&](float scale) {
                return [&, scale](int j, float (&v)[32]) {
                    uint32_t o[32];
                    tmem_ld32(tO + j * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * scale;
                };
            };
            if (is_level(MODE)) {
                const int64_t N = a.lv.seg_len;
                if (a.lv.level == 0) {
                    const int64_t orow = x.bhi * a.n + a.lv.q_off + x.node * a.lv.node_len + qloc;
                    const int esz = a.out_dtype == 0 ? 2 : 4;
                    unsigned char *drow = static_cast<unsigned char *>(a.O) + orow * D * esz;
                    warp_write_rows<D, C::SEG>(stage, drow, a.out_dtype == 0, lane, o_scaled(inv_l));
                    if (a.lse) a.lse[orow] = Lrow;
                } else {
                    const int64_t dense = x.bhi * (a.n / 2) + x.node * N + qloc;
                    unsigned char *drow = reinterpret_cast<unsigned char *>(a.Opart_w + dense * D);
                    warp_write_rows<D, C::SEG>(stage, drow, false, lane, o_scaled(inv_l));
                    a.Lpart_w[dense] = Lrow;
                }
            } else {
                // exact causal leaf part merged with the level parts of this row (log space)
                const int64_t orow = x.leaf_start + static_cast<int64_t>(my_gt) * 128 + r;
                const int64_t bhi = x.bhi, qrow = orow - bhi * a.n;
                const int64_t half_n = a.n / 2;
                // the level parts this row belongs to: level l holds the row when it lies in the lower half of
                // its node
                auto part_index = [&](int lvl, int64_t &dense) -> bool {
                    const int64_t len = a.n >> (lvl - 1), half = len / 2, within = qrow % len;
                    if (within < half) return false;
                    dense = static_cast<int64_t>(lvl - 1) * a.bh * half_n + bhi * half_n + (qrow / len) * half +
                            (within - half);
                    return true;
                };
                float Lmax = Lrow;
                for (int lvl = 1; lvl <= a.levels; ++lvl) {
                    int64_t dense;
                    if (part_index(lvl, dense)) Lmax = fmaxf(Lmax, a.Lpart_r[dense]);
                }
                const float wb = __expf(Lrow - Lmax);
                float tot = wb;
                for (int lvl = 1; lvl <= a.levels; ++lvl) {
                    int64_t dense;
                    if (part_index(lvl, dense)) tot += __expf(a.Lpart_r[dense] - Lmax);   // exp(-inf) = 0
                }
                const float inv_tot = 1.0f / tot;
                const float cb = wb * inv_l * inv_tot;
                auto merged = [&](int j, float (&acc)[32]) {
                    uint32_t o[32];
                    tmem_ld32(tO + j * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(o[e]) * cb;
                    for (int lvl = 1; lvl <= a.levels; ++lvl) {
                        int64_t dense;
                        if (!part_index(lvl, dense)) continue;
                        const float Lp = a.Lpart_r[dense];
                        if (Lp == -INFINITY) continue;
                        const float wi = __expf(Lp - Lmax) * inv_tot;
                        const float4 *src = reinterpret_cast<const float4 *>(a.Opart_r + dense * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 p = src[e];
                            acc[4 * e] += wi * p.x; acc[4 * e + 1] += wi * p.y;
                            acc[4 * e + 2] += wi * p.z; acc[4 * e + 3] += wi * p.w;
                        }
                    }
                };
                const int esz = a.out_dtype == 0 ? 2 : 4;
                unsigned char *drow = static_cast<unsigned char *>(a.O) + orow * D * esz;
                warp_write_rows<D, C::SEG>(stage, drow, a.out_dtype == 0, lane, merged);
            }
            if (C::kStageInQ) {
                // the stage writes are ordered before the tensor core's later reads of the refilled buffer
                fence_proxy_async_smem();
                mbar_arrive(bar(C::bQStage + qbuf));   // the Q buffer may be refilled
            }
            ++qn;
            tc_fence_before();
            mbar_arrive(bar(C::bOFree + t));
            kp += x.npairs;
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

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D, int MODE, bool HOOK = false>
int launch_tc(const void *Q, const void *K, const void *V, TcArgs args, cudaStream_t st) {
    args.Q = static_cast<const uint16_t *>(Q);
    args.K = static_cast<const uint16_t *>(K);
    args.V = static_cast<const uint16_t *>(V);
    const size_t smem = Cfg<D>::kBytes + 1024;
    auto kern = attn_tc_kernel<D, MODE, HOOK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    const int64_t grid = args.items < num_sms() ? args.items : num_sms();
    if (grid <= 0) return 0;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(args);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

int dispatch(int d, const void *Q, const void *K, const void *V, const TcArgs &args, cudaStream_t st) {
    {
        // the single-tile kernel of ha_attn_pp.cu for the modes and head dims it covers
        TcArgs pa = args;
        pa.Q = static_cast<const uint16_t *>(Q);
        pa.K = static_cast<const uint16_t *>(K);
        pa.V = static_cast<const uint16_t *>(V);
        const int k = launch_attn_pp(d, pa, num_sms(), st);
        if (k != -2) return k;
    }
    const bool level = args.mode == MODE_LEVEL;
    const bool dense = args.mode == MODE_DENSE;
    if (args.mode == MODE_LEVEL_RN) {
        if (d == 64) return launch_tc<64, MODE_LEVEL_RN>(Q, K, V, args, st);
        if (d == 128) return launch_tc<128, MODE_LEVEL_RN>(Q, K, V, args, st);
        return -2;
    }
    if (level && args.stall_ns > 0) {   // the test hook's instance
        if (d == 64) return launch_tc<64, MODE_LEVEL, true>(Q, K, V, args, st);
        if (d == 128) return launch_tc<128, MODE_LEVEL, true>(Q, K, V, args, st);
        return -2;
    }
    if (d == 64) {
        if (level) return launch_tc<64, MODE_LEVEL>(Q, K, V, args, st);
        return dense ? launch_tc<64, MODE_DENSE>(Q, K, V, args, st) : launch_tc<64, MODE_CAUSAL>(Q, K, V, args, st);
    }
    if (d == 128) {
        if (level) return launch_tc<128, MODE_LEVEL>(Q, K, V, args, st);
        return dense ? launch_tc<128, MODE_DENSE>(Q, K, V, args, st) : launch_tc<128, MODE_CAUSAL>(Q, K, V, args, st);
    }
    return -2;
}

}  // namespace

int launch_attn_tc(const Level &lv, const void *Q, const void *K, const void *V, int d, const int32_t *perm,
                   const int32_t *inv, const int32_t *S, int m, int64_t nodes_total, void *O, int out_dtype,
                   float *lse, float *Opart, float *Lpart, int *status, cudaStream_t st, int64_t stall_ns,
                   const int32_t *Srn, const float *lwrn) {
    const bool rn = Srn != nullptr && m > 0;
    if ((d != 64 && d != 128) || lv.bp % 128 != 0 || lv.bp > kMaxBlock || m > (rn ? kMaxSampleListRn : kMaxSampleList) ||
        lv.bh * lv.n >= (int64_t(1) << 31))
        return -2;
    TcArgs a{};
    a.mode = rn ? MODE_LEVEL_RN : MODE_LEVEL;
    a.Srn = rn ? Srn : nullptr;
    a.lwrn = rn ? lwrn : nullptr;
    a.n = lv.n;
    a.bh = lv.bh;
    a.lv = lv;
    a.perm = perm;
    a.inv = inv;
    a.S = S;
    a.m = m;
    a.nodes_total = nodes_total;
    a.nb = lv.bp / kKC;
    a.ns = (m + kKC - 1) / kKC;
    a.nr = rn ? a.ns : 0;
    a.tiles_per_block = lv.bp / 128;
    a.pairs_per_block = (a.tiles_per_block + 1) / 2;
    a.lw2 = m > 0 ? log2f(static_cast<float>(lv.seg_len) / static_cast<float>(m)) : 0.0f;
    a.O = O;
    a.out_dtype = out_dtype;
    a.lse = lse;
    a.Opart_w = Opart;
    a.Lpart_w = Lpart;
    a.status = status;
    a.stall_ns = stall_ns;
    a.items = lv.bh * lv.nodes * (lv.seg_len / lv.bp) * a.pairs_per_block;
    a.per_outer = static_cast<uint32_t>((lv.seg_len / lv.bp) * a.pairs_per_block);
    if (a.items >= (int64_t(1) << 31)) return -2;
    return dispatch(d, Q, K, V, a, st);
}

int launch_causal_base_tc(const void *Q, const void *K, const void *V, int64_t bh, int64_t n, int d, int64_t leaf,
                          int levels, const float *Opart, const float *Lpart, void *O, int out_dtype, int *status,
                          cudaStream_t st, int64_t stall_ns) {
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
    a.stall_ns = stall_ns;
    a.items = bh * a.nleaves * a.pairs_per_leaf;
    a.per_outer = static_cast<uint32_t>(bh * a.nleaves);
    if (a.items >= (int64_t(1) << 31)) return -2;
    return dispatch(d, Q, K, V, a, st);
}

int launch_exact_tc(const void *Q, const void *K, const void *V, int64_t bh, int64_t n, int d, int causal, void *O,
                    int out_dtype, int *status, cudaStream_t st) {
    if ((d != 64 && d != 128) || n <= 0 || n % 128 != 0 || bh * n >= (int64_t(1) << 31)) return -2;
    TcArgs a{};
    a.mode = causal ? MODE_CAUSAL : MODE_DENSE;
    a.n = n;
    a.bh = bh;
    a.leaf = n;
    a.nleaves = 1;
    a.levels = 0;
    a.tiles_per_leaf = static_cast<int>(n / 128);
    a.pairs_per_leaf = (a.tiles_per_leaf + 1) / 2;
    a.O = O;
    a.out_dtype = out_dtype;
    a.status = status;
    a.stall_ns = 0;
    a.items = bh * a.pairs_per_leaf;
    a.per_outer = static_cast<uint32_t>(bh);
    if (a.items >= (int64_t(1) << 31)) return -2;
    return dispatch(d, Q, K, V, a, st);
}

}  // namespace ha
