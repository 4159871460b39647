// ha_attn_pp.cu -- tensor-core (tcgen05 / TMEM) attention of the levels (block and sampled columns, merged), for
// d = 64 and d = 128: one 128-query tile per work item, double-buffered score and probability tiles, two softmax
// warpgroups on the two column halves of every chunk.
//
// The work is the same as in ha_attn_tc.cu ("HyperAttention: Long-context Attention in Near-Linear Time",
// research-map summary, "Approach"): the queries of a sorted block attend exactly to the block's keys and, with the
// weight N/m, to the uniformly sampled columns whose key lies outside the block (LEVEL). One online softmax per row
// over all parts gives O = (N1 + N2) / (D1 + D2). The schedule, and the measurements on this part that chose it:
//
//   * A work item is ONE 128-query tile. Its key chunks (the compacted sample chunks first, then the block chunks, so
//     that the running max is usually set by the weighted samples and rarely grows later) form one stream. The score
//     tile of chunk k goes to TMEM buffer S_(k mod 2) and its probabilities to P_(k mod 2), so the score product of
//     chunk k + 1 runs on the tensor core while the softmax works on chunk k, and the P.V product of chunk k while
//     the softmax works on chunk k + 1: no warp waits on the "scores -> softmax -> P.V -> next scores" chain, which
//     costs about 1.3K cycles of barrier and MMA latency per chunk on this part.
//   * The exponentials (MUFU unit, 16 per clock per SM) bound the softmax. Two warpgroups share every chunk: warp w
//     handles rows 32 (w mod 4) .. 32 (w mod 4) + 31 and column half h = (w - 4) / 4, so each sub-partition runs two
//     softmax warps. The halves of a row exchange their partial maxima through shared memory (a 64-thread named
//     barrier per lane quarter) and keep partial sums, which the epilogue adds. The exponent's scale and offset and
//     the row sums run as packed f32x2 instructions.
//   * The MMA issuer, per chunk k: wait for P(k), issue O += P(k) V(k), then the score product of chunk k + 2 into
//     the buffer that chunk k has just released; each commit of a score product therefore also covers the P.V
//     product of two chunks back, so a P buffer is always free when its next scores arrive. A row is re-based only
//     when its max grows by more than 2^8; O is then scaled after the previous chunk's P.V product has completed.
//   * One warp builds, an item ahead, the global key rows of every chunk of the item (through the key permutation,
//     and the sampled columns whose key lies outside the block, compacted) and the item's count of kept samples;
//     the K and V loaders then only copy rows, and the softmax takes its masking from the count.
//   * A warpgroup of its own runs the epilogue (normalise, write each row to its original position, or write a causal
//     level's part). d = 64: the accumulator is double-buffered by item, and the epilogue reads it into registers and
//     releases it before it writes, so the next item's first P.V product never waits on it. d = 128: one accumulator
//     (TMEM holds no second one), released once the epilogue has read the row.
//
// CTA layout (512 threads, one CTA per SM, persistent):
//   warp 0       K loader,
//   warp 1       MMA issuer (lane 0),
//   warp 2       row-list builder and Q loader,
//   warp 3       V loader,
//   warps 4-7    softmax of column half 0, warps 8-11 softmax of column half 1 (warp w reads TMEM lanes
//                32 (w mod 4) .. 32 (w mod 4) + 31),
//   warps 12-15  epilogue.
// Loaders copy rows with 16-byte cp.async into the 128-byte-swizzled layout the tensor core reads and arrive on the
// stage's K or V barrier when their copies complete. Stages: 4 (d = 64) or 2 (d = 128); with two, a K stage is
// refilled as soon as its chunk's score product has completed, a V stage once its P.V product has. Registers per
// thread: softmax kRegsSoftmax, the others kRegsOther (4 x 128 threads x 128 at launch).
// TMEM (512 columns): S_b at [128 b, 128 b + 128), P_b at [256 + 64 b, ...) (column half h at + 32 h), O accumulator j
// at [384 + d j, 384 + d (j + 1)) (b = 0, 1; j < 2 for d = 64, j = 0 for d = 128).
// Every mbarrier wait is bounded; on expiry the kernel sets the status bit, every role gives up, the loaders wait for
// their copies, the MMA issuer drains the tensor core, and TMEM is freed before exit.
#include "ha_attn_items.cuh"

namespace ha {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kSTThreads = 512;
constexpr int kRegsSoftmax = 152;   // each softmax warpgroup
constexpr int kRegsOther = 104;     // loader/issuer and epilogue warpgroups
static_assert(128 * (2 * kRegsSoftmax + 2 * kRegsOther) == kSTThreads * 128,
              "the warpgroups' budgets add up to the launch's registers");
constexpr int kCK = 128;            // keys per chunk
constexpr int kMaxItemChunks = kMaxBlock / kCK + kMaxSampleList / kCK;   // block chunks + sample chunks of an item

template <int D_>
struct STCfg {
    static constexpr int D = D_;
    static constexpr int QB = D == 64 ? 2 : 1;         // Q buffers
    static constexpr int NST = D == 64 ? 4 : 2;        // K/V stages of kCK rows
    static constexpr int OB = D == 64 ? 2 : 1;         // O accumulators (item i uses i mod OB)
    static constexpr int kQBytes = 128 * D * 2;        // a Q tile
    static constexpr int kCBytes = kCK * D * 2;        // a K or V chunk
    static constexpr int kPCol = 256;                  // P_b at kPCol + 64 b
    static constexpr int kOCol = 384;                  // O accumulator j at kOCol + D j
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + QB * kQBytes;
    static constexpr int kV = kK + NST * kCBytes;
    static constexpr int kStage = kV + NST * kCBytes;                     // 4 epilogue warps x 32 rows x 128 bytes
    static constexpr int kList = kStage + 4 * 32 * 128;                   // compacted samples of the block
    static constexpr int kCacheS = kList + kMaxSampleList * 4;            // samples of the current problem
    static constexpr int kCacheB = kCacheS + kMaxSampleList * 4;          // their sorted key block
    static constexpr int kKPerm = kCacheB + kMaxSampleList * 4;           // key rows of the current block
    static constexpr int kQPerm = kKPerm + kMaxBlock * 4;                 // query rows of one tile
    static constexpr int kIList = kQPerm + 128 * 4;                       // [item parity]: global key rows per chunk
    static constexpr int kICnt = kIList + 2 * kMaxItemChunks * kCK * 4;   // [item parity]: kept samples of the item
    static constexpr int kStats = kICnt + 16;                             // [item parity][half][row]: max, sum
    static constexpr int kXch = kStats + 2 * 2 * 128 * 8;                 // [chunk parity][half][row]: partial maxima
    static constexpr int kBars = kXch + 2 * 2 * 128 * 4;
    static constexpr int bQFull = 0, bQEmpty = bQFull + QB, bKFull = bQEmpty + QB, bVFull = bKFull + NST,
                         bKVEmpty = bVFull + NST,
                         bListFull = bKVEmpty + NST, bListEmpty = bListFull + 2,
                         bSFull = bListEmpty + 2,
                         bPFull = bSFull + 2, bOReady = bPFull + 2, bOFree = bOReady + 2,
                         bStatsReady = bOFree + 2, bStatsFree = bStatsReady + 2, bDrain = bStatsFree + 2,
                         kNumBars = bDrain + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kBytes = kAbort + 4;
    static_assert(kBars % 8 == 0, "mbarriers need 8-byte alignment");
    static_assert(kStage % 16 == 0 && kStats % 8 == 0, "alignment of the stage and the stats");
    static_assert(kBytes + 1024 <= 232448, "shared memory budget");
    static_assert(kOCol + OB * D <= 512, "TMEM budget");
};

// One 128-query tile. LEVEL: tile `tile` of sorted block blk of problem prob = (bhi, node); CAUSAL: query tile gt of
// a leaf (items heaviest first); DENSE: query tile gt of a sequence.
struct Tile {
    int nc;                 // key chunks
    uint32_t prob, blk, bhi, node, tile;
    int64_t leaf_start;     // CAUSAL / DENSE: global row of the leaf's first row
    int gt;
};

// Item index -> tile; per_outer = tiles per problem (LEVEL) or per query-tile index (CAUSAL, DENSE); nb, ns = block
// and sample chunks of kCK keys (LEVEL). Item counts and their factors are below 2^31 (checked on the host), so the
// divisions are 32-bit.
template <int MODE>
__device__ __forceinline__ Tile decode_tile(const TcArgs &a, int64_t it64) {
    Tile x{};
    const uint32_t it = static_cast<uint32_t>(it64);
    const uint32_t per = a.per_outer;
    if (is_level(MODE)) {
        const uint32_t prob = it / per;
        const uint32_t rem = it - prob * per;
        const uint32_t tpb = static_cast<uint32_t>(a.tiles_per_block);
        const uint32_t blk = rem / tpb;
        const uint32_t nodes = static_cast<uint32_t>(a.lv.nodes);
        x.prob = prob;
        x.blk = blk;
        x.tile = rem - blk * tpb;
        x.bhi = prob / nodes;
        x.node = prob - x.bhi * nodes;
        x.nc = a.nb + a.ns;
    } else {
        const uint32_t po = it / per;
        const uint32_t rem = it - po * per;
        const uint32_t nl = static_cast<uint32_t>(a.nleaves);
        x.bhi = rem / nl;
        x.leaf_start = static_cast<int64_t>(x.bhi) * a.n + static_cast<int64_t>(rem - x.bhi * nl) * a.leaf;
        if (MODE == MODE_CAUSAL) {
            x.gt = a.tiles_per_leaf - 1 - static_cast<int>(po);   // heaviest first
            x.nc = x.gt + 1;
        } else {
            x.gt = static_cast<int>(po);
            x.nc = a.tiles_per_leaf;
        }
    }
    return x;
}

// P = 2^(s log2(e) + off) over this half's 64 columns, rounded to bf16 pairs; returns the row sum of P (of the fp32
// values). The scale-and-offset and the sums run as packed f32x2 instructions (half the issue slots of scalar ones);
// the exponentials on the MUFU unit. Masked columns (s = -inf) give 2^-inf = 0.
__device__ __forceinline__ float exp_half(const uint32_t (&v)[64], float off, uint32_t (&pk)[32]) {
    const uint64_t sc = f2_pack(kLog2e, kLog2e), of = f2_pack(off, off);
    uint64_t la = f2_pack(0.0f, 0.0f), lb = la;
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc, of));
        const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
        const uint64_t p = f2_pack(p0, p1);
        if (e & 2) lb = f2_add(lb, p);
        else la = f2_add(la, p);
        pk[e / 2] = pack_bf16x2(p0, p1);
    }
    const float2 l2 = f2_unpack(f2_add(la, lb));
    return l2.x + l2.y;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kSTThreads, 1) attn_st_kernel(const TcArgs a) {
    using C = STCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    auto bar = [&](int i) -> uint32_t { return sbase + C::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::kAbort);
    int *icnt = reinterpret_cast<int *>(sm + C::kICnt);
    float2 *stats = reinterpret_cast<float2 *>(sm + C::kStats);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 32) {
        for (int i = 0; i < C::QB; ++i) {
            mbar_init(bar(C::bQFull + i), 32);     // the Q loader's lanes (copy completion)
            mbar_init(bar(C::bQEmpty + i), 1);     // commit after the tile's last score product
        }
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(bar(C::bKFull + s), 32);     // the K loader's lanes (copy completion)
            mbar_init(bar(C::bVFull + s), 32);     // the V loader's lanes
            mbar_init(bar(C::bKVEmpty + s), 1);    // commit after the chunk's P.V product
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::bListFull + i), 1);   // the list builder: an item's key rows and column counts written
            mbar_init(bar(C::bListEmpty + i), 10); // the K and V loaders and the 8 softmax warps: done with the list
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(C::bSFull + b), 1);      // commit after a score product into S_b
            mbar_init(bar(C::bPFull + b), 256);    // both softmax warpgroups: their halves of P_b written
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::bOReady + i), 1);     // commit after an item's last P.V product (item parity i)
            mbar_init(bar(C::bOFree + i), 128);    // the epilogue threads: the accumulator of parity i read
            mbar_init(bar(C::bStatsReady + i), 256);   // both softmax warpgroups: row max and sum written
            mbar_init(bar(C::bStatsFree + i), 128);    // the epilogue threads: row max and sum read
        }
        mbar_init(bar(C::bDrain), 1);
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

    // LEVEL items all cost the same: each CTA takes a contiguous range, so consecutive items share a block and a
    // problem (and their key rows and samples). CAUSAL and DENSE items are dealt round-robin, heaviest first.
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

    // Each warpgroup sets its register budget at the top of its own branch, so that the budget holds for all code
    // of the branch.
    if (warp < 4) {
        setmaxnreg_dec<kRegsOther>();
        if (warp == 2) {
            // -------------------------------------------------------------- list builder and Q loader
            // Per item i: the global key rows of all its chunks and their valid column counts into list slot
            // i mod 2 (once the loaders are done with item i - 2), then the query tile into Q buffer i mod QB (once
            // the buffer's previous tile has issued its last score product). The lists run an item ahead of the
            // loaders, so the loaders only copy rows.
            const unsigned lt_mask = (1u << lane) - 1u;
            int32_t *slist = reinterpret_cast<int32_t *>(sm + C::kList);
            int32_t *cache_s = reinterpret_cast<int32_t *>(sm + C::kCacheS);
            int32_t *cache_b = reinterpret_cast<int32_t *>(sm + C::kCacheB);
            int32_t *kperm = reinterpret_cast<int32_t *>(sm + C::kKPerm);
            int32_t *qperm = reinterpret_cast<int32_t *>(sm + C::kQPerm);
            int64_t cached_prob = -1, cached_blk = -1;
            int cnt = 0;
            uint32_t ni = 0;
            bool ok = true;
            for (int64_t it = first; it < last && ok; it += stride, ++ni) {
                const Tile x = decode_tile<MODE>(a, it);
                const int ls = static_cast<int>(ni & 1);
                // CAUSAL and DENSE read contiguous key rows: no list
                if (is_level(MODE) && ni >= 2 &&
                    !mbar_wait_inl(bar(C::bListEmpty + ls), ((ni >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                int32_t *ilist = reinterpret_cast<int32_t *>(sm + C::kIList) + ls * (kMaxItemChunks * kCK);
                int64_t kbase = 0;
                if (is_level(MODE)) {
                    kbase = static_cast<int64_t>(x.bhi) * a.n + static_cast<int64_t>(x.node) * a.lv.node_len;
                    const int64_t key_blk = static_cast<int64_t>(x.prob) * (a.lv.seg_len / a.lv.bp) + x.blk;
                    if (key_blk != cached_blk) {
                        const int32_t *pkg = a.perm + (static_cast<int64_t>(x.prob) * 2 + 1) * a.lv.seg_len +
                                             static_cast<int64_t>(x.blk) * a.lv.bp;
                        __syncwarp();
                        for (int i = lane; i < a.lv.bp / 4; i += 32)
                            reinterpret_cast<int4 *>(kperm)[i] = reinterpret_cast<const int4 *>(pkg)[i];
                        check_indices(kperm, a.lv.bp, a.lv.seg_len, a.status, lane);
                        cnt = 0;
                        if (a.m > 0) {
                            if (static_cast<int64_t>(x.prob) != cached_prob) {
                                const int32_t *Sp =
                                    a.S + (static_cast<int64_t>(x.bhi) * a.nodes_total + (a.lv.heap0 + x.node - 1)) * a.m;
                                const int32_t *ik = a.inv + (static_cast<int64_t>(x.prob) * 2 + 1) * a.lv.seg_len;
                                __syncwarp();
                                for (int u = lane; u < a.m; u += 32)
                                    cache_s[u] = checked_index(Sp[u], a.lv.seg_len, a.status);
                                __syncwarp();
                                for (int u = lane; u < a.m; u += 32) cache_b[u] = ik[cache_s[u]] / a.lv.bp;
                                cached_prob = x.prob;
                            }
                            // the block's sampled columns whose key lies outside it, in sample order
                            __syncwarp();
                            for (int base = 0; base < a.m; base += 32) {
                                const int u = base + lane;
                                const bool keep = u < a.m && cache_b[u] != static_cast<int32_t>(x.blk);
                                const unsigned bal = __ballot_sync(0xffffffffu, keep);
                                if (keep) slist[cnt + __popc(bal & lt_mask)] = cache_s[u];
                                cnt += __popc(bal);
                            }
                        }
                        cached_blk = key_blk;
                        __syncwarp();
                    }
                }
                if (is_level(MODE)) {
                    // LEVEL: chunks [0, ns) are sample chunks (their tails, past the block's count, point at the first
                    // key row and are masked), [ns, ns + nb) block chunks
                    for (int c = 0; c < x.nc; ++c) {
                        const bool sample = is_level(MODE) && c < a.ns;
                        const int u0 = c * kCK;
                        const int64_t cbase = is_level(MODE) ? kbase : x.leaf_start + static_cast<int64_t>(c) * kCK;
#pragma unroll
                        for (int rr = 0; rr < kCK / 32; ++rr) {
                            const int row = rr * 32 + lane;
                            int32_t loc;
                            if (!is_level(MODE)) loc = row;
                            else if (sample) loc = row + u0 < cnt ? slist[u0 + row] : 0;
                            else loc = kperm[(c - a.ns) * kCK + row];
                            ilist[c * kCK + row] = static_cast<int32_t>(cbase + loc);
                        }
                    }
                    if (lane == 0) icnt[ls] = is_level(MODE) ? cnt : 0;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::bListFull + ls));
                }
                // the query tile
                const int qb = static_cast<int>(ni % C::QB), use = static_cast<int>(ni / C::QB);
                if (use > 0 && !mbar_wait_inl(bar(C::bQEmpty + qb), (use - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t base = sbase + C::kQ + qb * C::kQBytes;
                if (is_level(MODE)) {
                    const int32_t *pq = a.perm + (static_cast<int64_t>(x.prob) * 2) * a.lv.seg_len +
                                        static_cast<int64_t>(x.blk) * a.lv.bp + x.tile * 128;
                    __syncwarp();
                    reinterpret_cast<int4 *>(qperm)[lane] = reinterpret_cast<const int4 *>(pq)[lane];
                    check_indices(qperm, 128, a.lv.seg_len, a.status, lane);
                    __syncwarp();
                    gather_rows<D, true>(base, a.Q,
                                         static_cast<int64_t>(x.bhi) * a.n + static_cast<int64_t>(x.node) * a.lv.node_len +
                                             a.lv.q_off,
                                         qperm, lane);
                } else {
                    gather_rows<D, false>(base, a.Q, x.leaf_start + static_cast<int64_t>(x.gt) * 128, qperm, lane);
                }
                cp_async_arrive(bar(C::bQFull + qb));
            }
            cp_wait<0>();
            if (!ok) flag_status(a.status);
        } else if (warp == 0 || warp == 3) {
            // -------------------------------------------------------------- K loader (warp 0), V loader (warp 3)
            // chunk g of the CTA (over all items) goes to stage g mod NST once the stage's previous chunk has
            // completed its products; rows from the item's list.
            const bool is_k = warp == 0;
            const uint16_t *src = is_k ? a.K : a.V;
            const uint32_t dst0 = sbase + (is_k ? C::kK : C::kV);
            uint32_t g = 0, ni = 0;
            bool ok = true;
            for (int64_t it = first; it < last && ok; it += stride, ++ni) {
                const Tile x = decode_tile<MODE>(a, it);
                const int ls = static_cast<int>(ni & 1);
                if (is_level(MODE) && !mbar_wait_inl(bar(C::bListFull + ls), (ni >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int32_t *ilist = reinterpret_cast<const int32_t *>(sm + C::kIList) + ls * (kMaxItemChunks * kCK);
                for (int c = 0; c < x.nc; ++c, ++g) {
                    const int slot = static_cast<int>(g % C::NST);
                    const uint32_t round = g / C::NST;
                    // a stage is free once its previous chunk's products have read it. With two stages the K rows
                    // are free as soon as that chunk's score product has completed (its commit to S_((g-2) mod 2)),
                    // which lets K run a chunk ahead of the P.V products; otherwise both wait for the P.V product.
                    bool free_ok = true;
                    if (round > 0) {
                        if (is_k && C::NST == 2) {
                            const uint32_t gp = g - 2;
                            free_ok = mbar_wait_inl(bar(C::bSFull + (gp & 1)), (gp >> 1) & 1, abort_flag);
                        } else {
                            free_ok = mbar_wait_inl(bar(C::bKVEmpty + slot), (round - 1) & 1, abort_flag);
                        }
                    }
                    if (!free_ok) {
                        ok = false;
                        break;
                    }
                    if (is_level(MODE))
                        gather_rows<D, true, kCK>(dst0 + slot * C::kCBytes, src, 0, ilist + c * kCK, lane);
                    else
                        gather_rows<D, false, kCK>(dst0 + slot * C::kCBytes, src,
                                                   x.leaf_start + static_cast<int64_t>(c) * kCK, ilist, lane);
                    cp_async_arrive(bar((is_k ? C::bKFull : C::bVFull) + slot));
                }
                // the row indices are in registers once the copies are issued: the list slot may be rebuilt
                __syncwarp();
                if (is_level(MODE) && ok && lane == 0) mbar_arrive(bar(C::bListEmpty + ls));
            }
            cp_wait<0>();
            if (!ok) flag_status(a.status);
        } else if (lane == 0) {
            // -------------------------------------------------------------- MMA issuer (warp 1, lane 0)
            constexpr uint32_t idesc_qk = idesc_bf16(128, kCK, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            // descriptors are built once; an MMA only adds a byte offset >> 4 to the start-address field
            const uint64_t dq0 = smem_desc(sbase + C::kQ, 16, 1024);
            const uint64_t dk0 = smem_desc(sbase + C::kK, 16, 1024);
            const uint64_t dv0 = smem_desc(sbase + C::kV, kCK * 128, 1024);
            bool ok = true;
            // score-product cursor: item it_s (tile xs), its chunk cs, chunks issued ks, Q buffers taken qc
            int64_t it_s = first;
            Tile xs{};
            if (it_s < last) xs = decode_tile<MODE>(a, it_s);
            int cs = 0, qc = 0, qb_s = 0;
            uint32_t ks = 0;
            auto issue_next_s = [&]() -> bool {
                if (it_s >= last) return true;
                if (cs == 0) {
                    qb_s = qc % C::QB;
                    if (!mbar_wait_inl(bar(C::bQFull + qb_s), (qc / C::QB) & 1, abort_flag)) return false;
                    ++qc;
                }
                const int slot = static_cast<int>(ks % C::NST);
                if (!mbar_wait_inl(bar(C::bKFull + slot), (ks / C::NST) & 1, abort_flag)) return false;
                tc_fence_after();
                const int b = static_cast<int>(ks & 1);
                const uint64_t dq = dq0 + static_cast<uint64_t>((qb_s * C::kQBytes) >> 4);
                const uint64_t dk = dk0 + static_cast<uint64_t>((slot * C::kCBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // k-step kk: 16 columns inside 64-column slab kk / 4 (slabs of 128 rows x 128 bytes)
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
                    mma_ss(tmem + kCK * b, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(C::bSFull + b));
                ++ks;
                if (++cs == xs.nc) {
                    mma_commit(bar(C::bQEmpty + qb_s));   // the tile's last score product: its Q buffer may refill
                    cs = 0;
                    it_s += stride;
                    if (it_s < last) xs = decode_tile<MODE>(a, it_s);
                }
                return true;
            };
            ok = issue_next_s() && issue_next_s();
            uint32_t k = 0, ni = 0;
            for (int64_t it = first; it < last && ok; it += stride, ++ni) {
                const Tile x = decode_tile<MODE>(a, it);
                const int ob = static_cast<int>(ni % C::OB);
                const uint32_t ouse = ni / C::OB;
                for (int c = 0; c < x.nc && ok; ++c, ++k) {
                    const int b = static_cast<int>(k & 1);
                    const int slot = static_cast<int>(k % C::NST);
                    if (!mbar_wait_inl(bar(C::bPFull + b), (k >> 1) & 1, abort_flag)) { ok = false; break; }
                    // the item's first P.V product overwrites accumulator ob: the epilogue must have read the previous
                    // item that used it (item ni - OB)
                    if (c == 0 && ouse > 0 && !mbar_wait_inl(bar(C::bOFree + ob), (ouse - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_inl(bar(C::bVFull + slot), (k / C::NST) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dv = dv0 + static_cast<uint64_t>((slot * C::kCBytes) >> 4);
                    const uint32_t od = tmem + C::kOCol + D * ob;
#pragma unroll
                    for (int kk = 0; kk < kCK / 16; ++kk)
                        mma_ts(od, tmem + C::kPCol + 64 * b + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4),
                               idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
                    if (c == x.nc - 1) mma_commit(bar(C::bOReady + ob));
                    mma_commit(bar(C::bKVEmpty + slot));   // both products of chunk k have been issued
                    ok = issue_next_s();                   // chunk k + 2 into buffer k mod 2
                }
            }
            if (!ok) flag_status(a.status);
            mma_commit(bar(C::bDrain));   // every MMA issued so far completes before TMEM is released
            volatile int no_abort = 0;
            mbar_wait_inl(bar(C::bDrain), 0, &no_abort, 200000000ull);
        }
        __syncwarp();
    } else if (warp < 12) {
        setmaxnreg_inc<kRegsSoftmax>();
        // ------------------------------------------------------------------ softmax of column half h
        const int h = (warp - 4) >> 2;               // column half: keys 64 h .. 64 h + 63 of every chunk
        const int q = warp & 3;                      // TMEM lane quarter
        const int r = q * 32 + lane;                 // row within the tile
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
        float *xch = reinterpret_cast<float *>(sm + C::kXch);
        uint32_t k = 0, ni = 0;
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride, ++ni) {
            const Tile x = decode_tile<MODE>(a, it);
            const int ip = static_cast<int>(ni & 1);
            // this half's share (D / 2 columns) of the row's accumulator
            const uint32_t tO = trow + C::kOCol + D * static_cast<int>(ni % C::OB) + (D / 2) * h;
            float m_run = -INFINITY, l = 0.0f;       // running max (base 2, weight included) and this half's sum
            // the item's count of kept samples (the valid columns of its sample chunks), from its list slot
            int cnt = 0;
            if (is_level(MODE)) {
                const int ls = static_cast<int>(ni & 1);
                if (!mbar_wait_inl(bar(C::bListFull + ls), (ni >> 1) & 1, abort_flag)) ok = false;
                if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                cnt = icnt[ls];
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::bListEmpty + ls));
            }
            for (int c = 0; c < x.nc; ++c, ++k) {
                const int b = static_cast<int>(k & 1);
                if (!mbar_wait_inl(bar(C::bSFull + b), (k >> 1) & 1, abort_flag)) { ok = false; break; }
                // columns > bound are masked (bound >= 63: none in this half); w2: log2 weight of the chunk's columns
                int bound = kCK - 1;
                float w2 = 0.0f;
                if (is_level(MODE)) {
                    if (c < a.ns) {
                        bound = min(kCK, max(0, cnt - c * kCK)) - 1;
                        w2 = a.lw2;
                    }
                } else if (MODE == MODE_CAUSAL) {
                    bound = x.gt * 128 + r - c * kCK;
                }
                bound -= 64 * h;
                tc_fence_after();
                const uint32_t tS = trow + kCK * b + 64 * h;
                uint32_t v[64];
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                tmem_ld_wait();
                const bool masked = __any_sync(0xffffffffu, bound < 63);
                if (masked) {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        if (e > bound) v[e] = 0xff800000u;   // -inf
                }
                float mx;
                {
                    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 64; e += 4) {
                        m0 = fmax3(m0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        m1 = fmax3(m1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                    }
                    mx = fmaxf(m0, m1);
                }
                // the row's max over both halves
                xch[((k & 1) * 2 + h) * 128 + r] = mx;
                named_barrier_sync(1 + q, 64);
                mx = fmaxf(mx, xch[((k & 1) * 2 + (h ^ 1)) * 128 + r]);
                const float xmax = mx == -INFINITY ? -INFINITY : fmaf(mx, kLog2e, w2);
                const float m_new = (c == 0 || xmax > m_run + kRescaleLog2) ? xmax : m_run;
                // alpha scales the earlier sum and O (0 when there were none, or all their columns were masked)
                const float alpha = c == 0 ? 0.0f : (m_new == m_run ? 1.0f : ex2_approx(m_run - m_new));
                const bool rescale = c > 0 && __any_sync(0xffffffffu, m_new != m_run);
                m_run = m_new;
                const float off = m_run == -INFINITY ? 0.0f : w2 - m_run;
                // P = 2^(s log2(e) + w2 - m_run); masked columns give 2^-inf = 0
                uint32_t pk[32];
                const float ls = exp_half(v, off, pk);
                l = l * alpha + ls;
                // P_b is free: the score product of this chunk was issued after the P.V product that last read it
                // (chunk k - 2), and its commit covered that product
                tmem_st32(trow + C::kPCol + 64 * b + 32 * h, pk);
                if (rescale) {
                    // O holds the P.V products of the item's chunks before this one: wait for the last (chunk k - 1;
                    // the commit that frees its K/V stage follows it), then scale this half's D / 2 of its columns
                    const uint32_t kp = k - 1;
                    if (!mbar_wait_inl(bar(C::bKVEmpty + kp % C::NST), (kp / C::NST) & 1, abort_flag)) ok = false;
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int p32 = 0; p32 < D / 64; ++p32) {
                        uint32_t o[32];
                        tmem_ld32(tO + 32 * p32, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tO + 32 * p32, o);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(C::bPFull + b));
            }
            if (!ok) break;
            // the row's max and this half's sum for the epilogue (slot of the item's parity, free once item ni - 2's
            // were read)
            if (ni >= 2 && !mbar_wait_inl(bar(C::bStatsFree + ip), ((ni >> 1) - 1) & 1, abort_flag)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            stats[(ip * 2 + h) * 128 + r] = make_float2(m_run, l);
            mbar_arrive(bar(C::bStatsReady + ip));
        }
        if (!ok) flag_status(a.status);
    } else {
        setmaxnreg_dec<kRegsOther>();
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
        unsigned char *stage = sm + C::kStage + q * (32 * 128);
        uint32_t ni = 0;
        bool ok = true;
        for (int64_t it = first; it < last && ok; it += stride, ++ni) {
            const Tile x = decode_tile<MODE>(a, it);
            const int ip = static_cast<int>(ni & 1);
            const uint32_t par = (ni >> 1) & 1;
            int64_t qloc = 0;
            if (is_level(MODE)) {
                const int64_t pos = static_cast<int64_t>(x.blk) * a.lv.bp + x.tile * 128 + r;
                qloc = checked_index(a.perm[(static_cast<int64_t>(x.prob) * 2) * a.lv.seg_len + pos], a.lv.seg_len,
                                     a.status);
            }
            const int ob = static_cast<int>(ni % C::OB);
            if (!mbar_wait_inl(bar(C::bStatsReady + ip), par, abort_flag)) ok = false;
            if (ok && !mbar_wait_inl(bar(C::bOReady + ob), (ni / C::OB) & 1, abort_flag)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            const float2 st0 = stats[(ip * 2) * 128 + r], st1 = stats[(ip * 2 + 1) * 128 + r];
            mbar_arrive(bar(C::bStatsFree + ip));
            tc_fence_after();
            // both halves share the running max; the row's sum is the halves' sum
            const float lsum = st0.y + st1.y;
            const float inv_l = 1.0f / lsum;
            const float Lrow = (st0.x + __log2f(lsum)) * kLn2;   // natural log of the row's normaliser
            const uint32_t tOr = trow + C::kOCol + D * ob;
            // the row times `scale`: 16 columns [16 g, 16 g + 16) at a time
            auto merged16 = [&](int g, float scale, float (&vv)[16]) {
                uint32_t o[16];
                tmem_ld16(tOr + 16 * g, o);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) vv[e] = __uint_as_float(o[e]) * scale;
            };
            if (MODE != MODE_CAUSAL && !(is_level(MODE) && a.lv.level > 0) && a.out_dtype == 0) {
                // bf16 output rows, 64 columns (128 bytes, one store segment) at a time. d = 64: the merged row is
                // packed into registers and the accumulator released before the store; d = 128: the accumulator is
                // released after the second half has been read.
                const int64_t orow = is_level(MODE) ? static_cast<int64_t>(x.bhi) * a.n + a.lv.q_off +
                                                          static_cast<int64_t>(x.node) * a.lv.node_len + qloc
                                                    : x.leaf_start + static_cast<int64_t>(x.gt) * 128 + r;
                unsigned char *drow = static_cast<unsigned char *>(a.O) + orow * D * 2;
#pragma unroll
                for (int hs = 0; hs < D / 64; ++hs) {
                    uint4 seg[8];
#pragma unroll
                    for (int g4 = 0; g4 < 4; ++g4) {
                        float vv[16];
                        merged16(4 * hs + g4, inv_l, vv);
                        seg[2 * g4] = make_uint4(pack_bf16x2(vv[0], vv[1]), pack_bf16x2(vv[2], vv[3]),
                                                 pack_bf16x2(vv[4], vv[5]), pack_bf16x2(vv[6], vv[7]));
                        seg[2 * g4 + 1] = make_uint4(pack_bf16x2(vv[8], vv[9]), pack_bf16x2(vv[10], vv[11]),
                                                     pack_bf16x2(vv[12], vv[13]), pack_bf16x2(vv[14], vv[15]));
                    }
                    if (hs == D / 64 - 1) {
                        tc_fence_before();
                        mbar_arrive(bar(C::bOFree + ob));
                    }
                    warp_store_segment<128>(stage, drow, 128 * hs, seg, lane);
                }
                if (is_level(MODE) && a.lse) a.lse[orow] = Lrow;
            } else if (MODE != MODE_CAUSAL) {
                // fp32 rows (level 0) or parts (causal levels): 16 merged columns at a time through the stage
                int64_t orow;
                unsigned char *drow;
                if (is_level(MODE) && a.lv.level > 0) {
                    orow = static_cast<int64_t>(x.bhi) * (a.n / 2) + static_cast<int64_t>(x.node) * a.lv.seg_len + qloc;
                    drow = reinterpret_cast<unsigned char *>(a.Opart_w + orow * D);
                    a.Lpart_w[orow] = Lrow;
                } else {
                    orow = is_level(MODE) ? static_cast<int64_t>(x.bhi) * a.n + a.lv.q_off +
                                                static_cast<int64_t>(x.node) * a.lv.node_len + qloc
                                          : x.leaf_start + static_cast<int64_t>(x.gt) * 128 + r;
                    drow = static_cast<unsigned char *>(a.O) + orow * D * 4;
                    if (is_level(MODE) && a.lse) a.lse[orow] = Lrow;
                }
#pragma unroll 1
                for (int g = 0; g < D / 16; ++g) {
                    float vv[16];
                    merged16(g, inv_l, vv);
                    uint4 seg[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        seg[i] = make_uint4(__float_as_uint(vv[4 * i]), __float_as_uint(vv[4 * i + 1]),
                                            __float_as_uint(vv[4 * i + 2]), __float_as_uint(vv[4 * i + 3]));
                    warp_store_segment<64>(stage, drow, 64 * g, seg, lane);
                }
                tc_fence_before();
                mbar_arrive(bar(C::bOFree + ob));
            } else {
                // exact causal leaf part merged with the level parts of this row (log space): level l holds the row
                // when it lies in the lower half of its node
                const int64_t orow = x.leaf_start + static_cast<int64_t>(x.gt) * 128 + r;
                const int64_t bhi = x.bhi, qrow = orow - bhi * a.n;
                const int64_t half_n = a.n / 2;
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
                const bool bf16 = a.out_dtype == 0;
                unsigned char *drow = static_cast<unsigned char *>(a.O) + orow * D * (bf16 ? 2 : 4);
#pragma unroll 1
                for (int g = 0; g < D / 16; ++g) {
                    float vv[16];
                    merged16(g, cb, vv);
                    for (int lvl = 1; lvl <= a.levels; ++lvl) {
                        int64_t dense;
                        if (!part_index(lvl, dense)) continue;
                        const float Lp = a.Lpart_r[dense];
                        if (Lp == -INFINITY) continue;
                        const float wi = __expf(Lp - Lmax) * inv_tot;
                        const float4 *src = reinterpret_cast<const float4 *>(a.Opart_r + dense * D + g * 16);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 p = src[e];
                            vv[4 * e] += wi * p.x; vv[4 * e + 1] += wi * p.y;
                            vv[4 * e + 2] += wi * p.z; vv[4 * e + 3] += wi * p.w;
                        }
                    }
                    if (bf16) {
                        uint4 seg[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            seg[i] = make_uint4(pack_bf16x2(vv[8 * i], vv[8 * i + 1]), pack_bf16x2(vv[8 * i + 2], vv[8 * i + 3]),
                                                pack_bf16x2(vv[8 * i + 4], vv[8 * i + 5]),
                                                pack_bf16x2(vv[8 * i + 6], vv[8 * i + 7]));
                        warp_store_segment<32>(stage, drow, 32 * g, seg, lane);
                    } else {
                        uint4 seg[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            seg[i] = make_uint4(__float_as_uint(vv[4 * i]), __float_as_uint(vv[4 * i + 1]),
                                                __float_as_uint(vv[4 * i + 2]), __float_as_uint(vv[4 * i + 3]));
                        warp_store_segment<64>(stage, drow, 64 * g, seg, lane);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(C::bOFree + ob));
            }
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

template <int D, int MODE>
int launch_st_t(TcArgs args, int sms, cudaStream_t st) {
    const size_t smem = STCfg<D>::kBytes + 1024;
    auto kern = attn_st_kernel<D, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return -1;
    // one item per query tile, chunks of kCK keys
    if (is_level(MODE)) {
        const int64_t blocks = args.lv.seg_len / args.lv.bp;
        args.per_outer = static_cast<uint32_t>(blocks * args.tiles_per_block);
        args.items = args.lv.bh * args.lv.nodes * blocks * args.tiles_per_block;
        args.nb = args.lv.bp / kCK;
        args.ns = (args.m + kCK - 1) / kCK;
        if (args.nb + args.ns > kMaxItemChunks) return -2;
    } else {
        args.per_outer = static_cast<uint32_t>(args.bh * args.nleaves);
        args.items = static_cast<int64_t>(args.tiles_per_leaf) * args.bh * args.nleaves;
    }
    if (args.items >= (int64_t(1) << 31)) return -2;
    const int64_t grid = args.items < sms ? args.items : sms;
    if (grid <= 0) return 0;
    kern<<<static_cast<unsigned>(grid), kSTThreads, smem, st>>>(args);
    return cudaPeekAtLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

// The kernel of this file for the modes and head dims it covers; -2 for the others (the caller then uses the kernel
// of ha_attn_tc.cu).
int launch_attn_pp(int d, const attn::TcArgs &args, int sms, cudaStream_t st) {
    if (args.stall_ns > 0) return -2;   // the timeout test hook lives in the kernel of ha_attn_tc.cu
    // Level mode only: for the exact causal leaves and dense attention one query tile per item loads every key
    // chunk once per tile, and the two-tile items of ha_attn_tc.cu measured faster (2.08 against 2.58 ms for the
    // leaves of the causal prefill workload).
    if (args.mode != attn::MODE_LEVEL) return -2;
    if (d == 64) return launch_st_t<64, attn::MODE_LEVEL>(args, sms, st);
    if (d == 128) return launch_st_t<128, attn::MODE_LEVEL>(args, sms, st);
    return -2;
}

}  // namespace ha
