// ha_attn_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) attention kernels for bf16 inputs.
//
// Two modes share one persistent kernel:
//
//  LEVEL: the HyperAttention problem of one level ("HyperAttention: Long-context Attention in Near-Linear
//  Time", research-map summary, "Approach"). A work item is a pair of 128-query tiles of one sorted block
//  i. Its key stream is the b'/64 chunks of key block i (exact block part) followed by ceil(m/64) chunks
//  of sampled columns (uniform sample part). The loader compacts the sample list per item: columns whose
//  key lies in block i are already counted exactly and are dropped, the rest keep their order and carry
//  the weight N/m (+ log2(N/m) on the base-2 score); only the tail of the last sample chunk is masked.
//  Rows are fetched through the sort permutations with TMA tile::gather4 loads straight into
//  128-byte-swizzled shared memory, so no permuted copy of Q, K or V exists. One online softmax over both
//  parts gives O = (N1+N2)/(D1+D2); the epilogue writes each row to its original position (merge and
//  un-permute), or, for causal levels, the fp32 part and its log normaliser.
//
//  CAUSAL: exact causal attention inside leaves of c rows (the summary's recursive causal extension: the
//  base case), merged in log space with the parts of every causal level the row belongs to
//  ("Limitations": partitioning and merging). A work item is a pair of query tiles of one leaf; query tile
//  g sees key chunks 0..2g+1, the last two with the inclusive causal mask. Items run heaviest first.
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warp 0      loader: Q tiles, K/V chunks of 64 rows (ring of NST stages), per-item sample list;
//   warp 1      MMA issuer (lane 0): S = Q K^T into TMEM (two S buffers per tile, so the next chunk's
//               scores are computed while the softmax works on the current one), O += P V with P in TMEM;
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: a thread owns one query row (TMEM lane),
//               reads its 64 scores once, keeps the running max and sum, writes P (bf16) over S, rescales O
//               only when the running max grows by more than 2^8, and runs the epilogue.
// TMEM (512 columns): S buffers of tile t at [128 t, 128 t + 64) and [128 t + 64, 128 t + 128) (P occupies
// the first 32 columns of its buffer), O of tile t at [256 + d t, 256 + d t + d).
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
constexpr int kKC = 64;                 // keys per chunk
constexpr int kMaxLevels = 16;
constexpr int kMaxSampleList = 1024;    // sampled columns per problem handled by the tensor-core path
constexpr int kMaxBlock = 1024;         // rows per sorted block handled by the tensor-core path
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the running max grows by more than this

enum { MODE_LEVEL = 0, MODE_CAUSAL = 1 };

struct TcArgs {
    int mode;
    const uint16_t *Q, *K, *V;   // bf16 [bh * n][d]
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
    int nc[2];            // key chunks of each tile
    int nc_max;
    // LEVEL
    int64_t prob, blk, bhi, node;
    int pair;
    // CAUSAL
    int64_t leaf_start;   // global row of the leaf's first row (bhi * n + leaf offset)
    int gt[2];            // query tile index within the leaf
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
        x.leaf_start = x.bhi * a.n + (rem % a.nleaves) * a.leaf;
        x.pair = pair;
        x.nc_max = 0;
        for (int t = 0; t < 2; ++t) {
            x.gt[t] = pair * 2 + t;
            x.valid[t] = x.gt[t] < a.tiles_per_leaf;
            x.nc[t] = x.valid[t] ? 2 * x.gt[t] + 2 : 0;
            x.nc_max = max(x.nc_max, x.nc[t]);
        }
    }
    return x;
}

template <int D>
struct Smem {
    static constexpr int kSlabs = D / 64;
    static constexpr int kTileBytes = 128 * D * 2;       // one 128-row Q tile (bf16)
    static constexpr int kChunkBytes = kKC * D * 2;      // one 64-row K or V chunk
    static constexpr int kStages = D == 64 ? 8 : 4;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + 2 * kTileBytes;
    static constexpr int kV = kK + kStages * kChunkBytes;
    static constexpr int kList = kV + kStages * kChunkBytes;             // compacted samples of the item
    static constexpr int kCacheS = kList + kMaxSampleList * 4;           // samples of the current problem
    static constexpr int kCacheB = kCacheS + kMaxSampleList * 4;         // their sorted key block
    static constexpr int kKPerm = kCacheB + kMaxSampleList * 4;          // key rows of the item's block
    static constexpr int kQPerm = kKPerm + kMaxBlock * 4;                // query rows of one tile
    static constexpr int kWord = kQPerm + 128 * 4;
    static constexpr int kBars = kWord + kStages * 4 + 64;   // keep 8-byte alignment with slack
    static constexpr int bQFull = 0, bQEmpty = 2, bKVFull = 4,
                         bKVEmpty = bKVFull + kStages, bWordFull = bKVEmpty + kStages, bSFull = bWordFull + kStages,
                         bPFull = bSFull + 4, bOReady = bPFull + 4, bOFinal = bOReady + 2, bOFree = bOFinal + 2,
                         bDrain = bOFree + 2, kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static_assert(kBars % 8 == 0, "mbarriers need 8-byte alignment");
};

__device__ __forceinline__ void flag_status(int *status) {
    if (status) atomicOr(status, kStatusTimeout);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const TcArgs a) {
    using L = Smem<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kAbort);
    int *words = reinterpret_cast<int *>(sm + L::kWord);
    int32_t *slist = reinterpret_cast<int32_t *>(sm + L::kList);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 32) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(L::bQFull + t), 32);     // the Q loader warp
            mbar_init(bar(L::bQEmpty + t), 1);
            mbar_init(bar(L::bOReady + t), 1);
            mbar_init(bar(L::bOFinal + t), 1);
            mbar_init(bar(L::bOFree + t), 128);
            for (int b = 0; b < 2; ++b) {
                mbar_init(bar(L::bSFull + 2 * t + b), 1);
                mbar_init(bar(L::bPFull + 2 * t + b), 128);
            }
        }
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar(L::bKVFull + s), 32);    // the K/V loader warp
            mbar_init(bar(L::bKVEmpty + s), 1);
            mbar_init(bar(L::bWordFull + s), 1);
        }
        mbar_init(bar(L::bDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + L::kTmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + L::kTmemSlot);

    // LEVEL items all cost the same: each CTA takes a contiguous range, so consecutive items share a problem
    // and its cached samples. CAUSAL items are ordered heaviest first and dealt round-robin.
    int64_t first, last, stride;
    if (a.mode == MODE_LEVEL) {
        const int64_t per = (a.items + gridDim.x - 1) / gridDim.x;
        first = static_cast<int64_t>(blockIdx.x) * per;
        last = min(a.items, first + per);
        stride = 1;
    } else {
        first = blockIdx.x;
        last = a.items;
        stride = gridDim.x;
    }

    if (warp == 0 || warp == 2) {
        // ------------------------------------------------------------------ loaders
        // warp 2 copies the Q tiles of each item, warp 0 streams the K/V chunks. Rows move as 16-byte cp.async
        // copies, PPR lanes per row, into the 128-byte-swizzled layout the tensor core reads (16-byte piece j
        // of row r sits at piece j ^ (r & 7)); when a warp's copies have landed it fences them to the async
        // proxy and its 32 lanes arrive on the stage's barrier.
        constexpr int PPR = D / 8;             // 16-byte pieces per row
        constexpr int RPI = 32 / PPR;          // rows per warp instruction
        const int rsub = lane / PPR, piece = lane % PPR;
        const int slab = piece >> 3, jp = piece & 7;
        bool ok = true;
        if (warp == 2) {
            int32_t *qperm = reinterpret_cast<int32_t *>(sm + L::kQPerm);
            int qcnt0 = 0, qcnt1 = 0;
            for (int64_t it = first; it < last && ok; it += stride) {
                const Item x = decode(a, it);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!ok || !x.valid[t]) continue;
                    int &qc = t == 0 ? qcnt0 : qcnt1;
                    if (qc > 0 && !mbar_wait(bar(L::bQEmpty + t), (qc - 1) & 1, abort_flag)) { ok = false; continue; }
                    const uint32_t base = sbase + L::kQ + t * L::kTileBytes;
                    int64_t qbase;
                    const bool through_perm = a.mode == MODE_LEVEL;
                    if (through_perm) {
                        // the tile's 128 query rows, one 16-byte load per lane, staged in shared memory
                        const int32_t *pq = a.perm + (x.prob * 2) * a.lv.seg_len + x.blk * a.lv.bp + (x.pair * 2 + t) * 128;
                        __syncwarp();
                        reinterpret_cast<int4 *>(qperm)[lane] = reinterpret_cast<const int4 *>(pq)[lane];
                        __syncwarp();
                        qbase = x.bhi * a.n + x.node * a.lv.node_len + a.lv.q_off;
                    } else {
                        qbase = x.leaf_start + x.gt[t] * 128;
                    }
#pragma unroll 8
                    for (int r0 = 0; r0 < 128; r0 += RPI) {
                        const int row = r0 + rsub;
                        const int64_t grow = qbase + (through_perm ? qperm[row] : row);
                        cp_async16(base + slab * 16384 + row * 128 + ((jp ^ (row & 7)) << 4), a.Q + grow * D + piece * 8);
                    }
                    cp_commit();
                    cp_wait<0>();
                    fence_proxy_async_smem();
                    mbar_arrive(bar(L::bQFull + t));
                    ++qc;
                }
            }
        } else {
            const unsigned lt_mask = (1u << lane) - 1u;
            int32_t *cache_s = reinterpret_cast<int32_t *>(sm + L::kCacheS);
            int32_t *cache_b = reinterpret_cast<int32_t *>(sm + L::kCacheB);
            int32_t *kperm = reinterpret_cast<int32_t *>(sm + L::kKPerm);
            int64_t cached_prob = -1;
            int64_t g = 0;
            // commit groups whose barrier arrival is still owed (oldest first); a chunk's arrival is made
            // once kLag newer groups have been issued, or when the stream drains
            constexpr int kLag = 2;
            uint32_t f0 = 0, f1 = 0, f2 = 0;
            int fn = 0;
            auto push = [&](uint32_t b) {
                cp_commit();
                if (fn == 0) f0 = b; else if (fn == 1) f1 = b; else f2 = b;
                ++fn;
                if (fn > kLag) {
                    cp_wait<kLag>();
                    fence_proxy_async_smem();
                    mbar_arrive(f0);
                    f0 = f1;
                    f1 = f2;
                    --fn;
                }
            };
            for (int64_t it = first; it < last && ok; it += stride) {
                const Item x = decode(a, it);
                // compacted sample list of this item: the sampled columns whose key lies outside block blk,
                // in sample order (from the per-problem cache of samples and their sorted blocks)
                int cnt = 0;
                int64_t kbase = 0;
                const int32_t *pk = nullptr;
                if (a.mode == MODE_LEVEL) {
                    kbase = x.bhi * a.n + x.node * a.lv.node_len;
                    const int32_t *pkg = a.perm + (x.prob * 2 + 1) * a.lv.seg_len + x.blk * a.lv.bp;
                    __syncwarp();
                    for (int i = lane; i < a.lv.bp / 4; i += 32)
                        reinterpret_cast<int4 *>(kperm)[i] = reinterpret_cast<const int4 *>(pkg)[i];
                    pk = kperm;
                    if (a.ns > 0) {
                        if (x.prob != cached_prob) {
                            const int32_t *Sp = a.S + (x.bhi * a.nodes_total + (a.lv.heap0 + x.node - 1)) * a.m;
                            const int32_t *ik = a.inv + (x.prob * 2 + 1) * a.lv.seg_len;
                            __syncwarp();
                            for (int u = lane; u < a.m; u += 32) cache_s[u] = Sp[u];
                            __syncwarp();
                            for (int u = lane; u < a.m; u += 32) cache_b[u] = ik[cache_s[u]] / a.lv.bp;
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
                    }
                    __syncwarp();
                }
                for (int c = 0; c < x.nc_max; ++c, ++g) {
                    const int slot = static_cast<int>(g % L::kStages);
                    const int64_t round = g / L::kStages;
                    if (round > 0 && !mbar_wait(bar(L::bKVEmpty + slot), (round - 1) & 1, abort_flag)) { ok = false; break; }
                    int valid_cols = kKC;
                    int kind;   // 0: block chunk (through the key permutation), 1: sample chunk, 2: contiguous
                    int u0 = 0;
                    if (a.mode == MODE_LEVEL) {
                        if (c < a.nb) {
                            kind = 0;
                        } else {
                            kind = 1;
                            u0 = (c - a.nb) * kKC;
                            valid_cols = min(kKC, max(0, cnt - u0));
                        }
                    } else {
                        kind = 2;
                    }
                    if (lane == 0) {
                        words[slot] = valid_cols;
                        mbar_arrive(bar(L::bWordFull + slot));
                    }
                    const uint32_t kb = sbase + L::kK + slot * L::kChunkBytes;
                    const uint32_t vb = sbase + L::kV + slot * L::kChunkBytes;
                    const int64_t cbase = a.mode == MODE_LEVEL ? kbase : x.leaf_start + static_cast<int64_t>(c) * kKC;
#pragma unroll 8
                    for (int r0 = 0; r0 < kKC; r0 += RPI) {
                        const int row = r0 + rsub;
                        int32_t loc;
                        if (kind == 0) loc = pk[c * kKC + row];
                        else if (kind == 1) loc = u0 + row < cnt ? slist[u0 + row] : 0;
                        else loc = row;
                        const int64_t goff = (cbase + loc) * D + piece * 8;
                        const uint32_t off = slab * (kKC * 128) + row * 128 + ((jp ^ (row & 7)) << 4);
                        cp_async16(kb + off, a.K + goff);
                        cp_async16(vb + off, a.V + goff);
                    }
                    push(bar(L::bKVFull + slot));
                }
            }
            // owed arrivals: every copy lands before the CTA moves on or exits
            cp_wait<0>();
            fence_proxy_async_smem();
            if (fn > 0) mbar_arrive(f0);
            if (fn > 1) mbar_arrive(f1);
            if (fn > 2) mbar_arrive(f2);
        }
        if (!ok) flag_status(a.status);
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, kKC, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            int64_t g = 0;
            int qcnt0 = 0, qcnt1 = 0, ocnt0 = 0, ocnt1 = 0, pb00 = 0, pb01 = 0, pb10 = 0, pb11 = 0;
            bool ok = true;
            auto tS = [&](int t, int b) -> uint32_t { return tmem + t * 128 + b * 64; };
            auto issue_s = [&](int t, int b, int slot) {
                const uint32_t qa = sbase + L::kQ + t * L::kTileBytes;
                const uint32_t ka = sbase + L::kK + slot * L::kChunkBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t koff = (kk >> 2) * (kKC * 128) + (kk & 3) * 32;
                    mma_ss(tS(t, b), smem_desc(qa + qoff, 16, 1024), smem_desc(ka + koff, 16, 1024), idesc_qk,
                           kk > 0 ? 1u : 0u);
                }
            };
            auto wait_k = [&](int64_t gc) -> bool {
                return mbar_wait(bar(L::bKVFull + static_cast<int>(gc % L::kStages)), (gc / L::kStages) & 1, abort_flag);
            };
            for (int64_t it = first; it < last && ok; it += stride) {
                const Item x = decode(a, it);
                // first two score chunks of each tile
                for (int c0 = 0; c0 < 2 && ok; ++c0) {
                    if (c0 >= x.nc_max) break;
                    if (!wait_k(g + c0)) { ok = false; break; }
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!x.valid[t] || c0 >= x.nc[t]) continue;
                        if (c0 == 0) {
                            int &qc = t == 0 ? qcnt0 : qcnt1;
                            if (!mbar_wait(bar(L::bQFull + t), qc & 1, abort_flag)) { ok = false; break; }
                            ++qc;
                        }
                        tc_fence_after();
                        issue_s(t, c0, static_cast<int>((g + c0) % L::kStages));
                        mma_commit(bar(L::bSFull + 2 * t + c0));
                        if (c0 == x.nc[t] - 1) mma_commit(bar(L::bQEmpty + t));
                    }
                }
                for (int c = 0; c < x.nc_max && ok; ++c) {
                    const int64_t gc = g + c;
                    const int slot = static_cast<int>(gc % L::kStages);
                    if (!mbar_wait(bar(L::bKVFull + slot), (gc / L::kStages) & 1, abort_flag)) { ok = false; break; }
                    const int b = c & 1;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!ok || !x.valid[t] || c >= x.nc[t]) continue;
                        int &pc = t == 0 ? (b ? pb01 : pb00) : (b ? pb11 : pb10);
                        if (!mbar_wait(bar(L::bPFull + 2 * t + b), pc & 1, abort_flag)) { ok = false; continue; }
                        ++pc;
                        const int oc = t == 0 ? ocnt0 : ocnt1;
                        if (c == 0 && oc > 0 && !mbar_wait(bar(L::bOFree + t), (oc - 1) & 1, abort_flag)) { ok = false; continue; }
                        tc_fence_after();
                        const uint32_t va = sbase + L::kV + slot * L::kChunkBytes;
#pragma unroll
                        for (int kk = 0; kk < kKC / 16; ++kk)
                            mma_ts(tmem + 256 + t * D, tS(t, b) + kk * 8, smem_desc(va + kk * 2048, kKC * 128, 1024),
                                   idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(bar(L::bOReady + t));
                        if (c == x.nc[t] - 1) mma_commit(bar(L::bOFinal + t));
                    }
                    if (!ok) break;
                    // chunk c is consumed once these P.V products finish: release its stage before waiting for
                    // chunk c + 2, whose arrival may depend on that stage
                    mma_commit(bar(L::bKVEmpty + slot));
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!ok || !x.valid[t] || c + 2 >= x.nc[t]) continue;
                        if (!wait_k(gc + 2)) { ok = false; continue; }
                        tc_fence_after();
                        issue_s(t, b, static_cast<int>((gc + 2) % L::kStages));
                        mma_commit(bar(L::bSFull + 2 * t + b));
                        if (c + 2 == x.nc[t] - 1) mma_commit(bar(L::bQEmpty + t));
                    }
                    if (!ok) break;
                }
                g += x.nc_max;
                if (x.valid[0]) ++ocnt0;
                if (x.valid[1]) ++ocnt1;
            }
            if (!ok) flag_status(a.status);
            mma_commit(bar(L::bDrain));   // every MMA issued so far completes before TMEM is released
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
        const uint32_t tO = trow + 256 + t * D;
        int64_t g = 0;
        int sb0 = 0, sb1 = 0, pvcnt = 0, fin = 0;
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride) {
            const Item x = decode(a, it);
            const bool my_valid = t == 0 ? x.valid[0] : x.valid[1];
            const int my_nc = t == 0 ? x.nc[0] : x.nc[1];
            const int my_gt = t == 0 ? x.gt[0] : x.gt[1];
            if (!my_valid) { g += x.nc_max; continue; }
            int64_t qloc = 0;
            if (a.mode == MODE_LEVEL) {
                const int64_t pos = x.blk * a.lv.bp + (x.pair * 2 + t) * 128 + r;
                qloc = a.perm[(x.prob * 2) * a.lv.seg_len + pos];   // consumed by the epilogue
            }
            float m_run = -INFINITY, l = 0.0f;
            for (int c = 0; c < my_nc; ++c) {
                const int64_t gc = g + c;
                const int b = c & 1;
                const uint32_t tS = trow + t * 128 + b * 64;
                if (!mbar_wait(bar(L::bSFull + 2 * t + b), (b ? sb1 : sb0) & 1, abort_flag)) { ok = false; break; }
                if (b) ++sb1; else ++sb0;
                // column bound: columns > bound are masked (bound >= 63: none)
                int bound = kKC - 1;
                float w2 = 0.0f;
                if (a.mode == MODE_LEVEL) {
                    if (c >= a.nb) {
                        const int slot = static_cast<int>(gc % L::kStages);
                        if (!mbar_wait(bar(L::bWordFull + slot), (gc / L::kStages) & 1, abort_flag)) { ok = false; break; }
                        bound = words[slot] - 1;
                        w2 = a.lw2;
                    }
                } else {
                    bound = my_gt * 128 + r - c * kKC;
                }
                tc_fence_after();
                uint32_t va[32], vb[32];   // scores of columns 0-31 and 32-63 (registers; indices are constants)
                tmem_ld32(tS, va);
                tmem_ld32(tS + 32, vb);
                tmem_ld_wait();
                if (__any_sync(0xffffffffu, bound < kKC - 1)) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        if (e > bound) va[e] = 0xff800000u;   // -inf
                        if (e + 32 > bound) vb[e] = 0xff800000u;
                    }
                }
                float mx0 = __uint_as_float(va[0]), mx1 = __uint_as_float(va[1]);
                float mx2 = __uint_as_float(vb[0]), mx3 = __uint_as_float(vb[1]);
#pragma unroll
                for (int e = 2; e < 32; e += 2) {
                    mx0 = fmaxf(mx0, __uint_as_float(va[e]));
                    mx1 = fmaxf(mx1, __uint_as_float(va[e + 1]));
                    mx2 = fmaxf(mx2, __uint_as_float(vb[e]));
                    mx3 = fmaxf(mx3, __uint_as_float(vb[e + 1]));
                }
                const float smax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
                const float xmax = smax == -INFINITY ? -INFINITY : fmaf(smax, kLog2e, w2);
                const float m_new = xmax > m_run + kRescaleLog2 ? xmax : m_run;
                const bool grow = m_new != m_run;
                const float alpha = grow ? ex2_approx(m_run - m_new) : 1.0f;   // 0 when m_run = -inf
                l *= alpha;
                if (c > 0 && __any_sync(0xffffffffu, grow)) {
                    // O holds P.V of chunks 0..c-1; the last of them (PV of chunk c-1) may still be running
                    if (!mbar_wait(bar(L::bOReady + t), (pvcnt - 1) & 1, abort_flag)) ok = false;
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
                uint32_t pk[32];
                float l0 = 0.0f, l1 = 0.0f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(va[2 * e]), kLog2e, off));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(va[2 * e + 1]), kLog2e, off));
                    const float p2 = ex2_approx(fmaf(__uint_as_float(vb[2 * e]), kLog2e, off));
                    const float p3 = ex2_approx(fmaf(__uint_as_float(vb[2 * e + 1]), kLog2e, off));
                    l0 += p0 + p1;
                    l1 += p2 + p3;
                    pk[e] = pack_bf16x2(p0, p1);
                    pk[16 + e] = pack_bf16x2(p2, p3);
                }
                l += l0 + l1;
                tmem_st32(tS, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(L::bPFull + 2 * t + b));
                ++pvcnt;
            }
            if (!ok) break;
            // epilogue: wait for the tile's last P.V of this item, then write the row
            if (!mbar_wait(bar(L::bOFinal + t), fin & 1, abort_flag)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            ++fin;
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float Lrow = (m_run + __log2f(l)) * kLn2;   // natural log of the row's normaliser
            if (a.mode == MODE_LEVEL) {
                const int64_t N = a.lv.seg_len;
                if (a.lv.level == 0) {
                    const int64_t orow = x.bhi * a.n + a.lv.q_off + x.node * a.lv.node_len + qloc;
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t o[32];
                        tmem_ld32(tO + j * 32, o);
                        tmem_ld_wait();
                        if (a.out_dtype == 0) {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.O) + orow * D + j * 32);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                uint4 w;
                                w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv_l, __uint_as_float(o[8 * e + 1]) * inv_l);
                                w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv_l, __uint_as_float(o[8 * e + 3]) * inv_l);
                                w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv_l, __uint_as_float(o[8 * e + 5]) * inv_l);
                                w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv_l, __uint_as_float(o[8 * e + 7]) * inv_l);
                                dst[e] = w;
                            }
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.O) + orow * D + j * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                                     __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
                        }
                    }
                    if (a.lse) a.lse[orow] = Lrow;
                } else {
                    const int64_t dense = x.bhi * (a.n / 2) + x.node * N + qloc;
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        uint32_t o[32];
                        tmem_ld32(tO + j * 32, o);
                        tmem_ld_wait();
                        float4 *dst = reinterpret_cast<float4 *>(a.Opart_w + dense * D + j * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                                 __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
                    }
                    a.Lpart_w[dense] = Lrow;
                }
            } else {
                // exact causal leaf part merged with the level parts of this row (log space)
                const int64_t orow = x.leaf_start + my_gt * 128 + r;
                const int64_t bhi = x.bhi, qrow = orow - bhi * a.n;
                const int64_t half_n = a.n / 2;
                // the level parts this row belongs to: level l holds the row when it lies in the lower half of its node
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
#pragma unroll
                for (int j = 0; j < D / 32; ++j) {
                    uint32_t o[32];
                    tmem_ld32(tO + j * 32, o);
                    tmem_ld_wait();
                    float acc[32];
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

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D>
int launch_tc(const void *Q, const void *K, const void *V, TcArgs args, cudaStream_t st) {
    args.Q = static_cast<const uint16_t *>(Q);
    args.K = static_cast<const uint16_t *>(K);
    args.V = static_cast<const uint16_t *>(V);
    const size_t smem = Smem<D>::kBytes + 1024;
    auto kern = attn_tc_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    const int64_t grid = args.items < num_sms() ? args.items : num_sms();
    if (grid <= 0) return 0;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(args);
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
    if ((d != 64 && d != 128) || lv.bp % 128 != 0 || lv.bp > kMaxBlock || m > kMaxSampleList ||
        lv.bh * lv.n >= (int64_t(1) << 31))
        return -2;
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
    a.nb = lv.bp / kKC;
    a.ns = (m + kKC - 1) / kKC;
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
