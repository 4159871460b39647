// ha_attn_items.cuh -- work items and output staging shared by the tensor-core attention kernels
// (ha_attn_tc.cu, ha_attn_pp.cu): the kernel arguments, the decode of a work item (a pair of 128-row query
// tiles of one sorted block, or of one exact causal leaf), and the warp-wide staged stores of output rows.
#pragma once

#include <math.h>

#include "ha_common.cuh"
#include "ha_internal.h"
#include "ha_sm100.cuh"

namespace ha {
namespace attn {

using namespace sm100;

constexpr int kKC = 128;                // keys per chunk
constexpr int kMaxLevels = 16;
constexpr int kMaxSampleList = 1024;    // sampled columns per problem handled by the tensor-core path
constexpr int kMaxSampleListRn = 256;   // the same with row-norm sampling (m uniform samples + m draws)
constexpr int kMaxBlock = 1024;         // rows per sorted block handled by the tensor-core path
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the running max grows by more than this

// MODE_DENSE: exact (non-causal) softmax attention of every query tile against every key chunk of its
// sequence, with the CAUSAL mode's work layout (a "leaf" is the whole sequence) and no mask.
enum { MODE_LEVEL = 0, MODE_CAUSAL = 1, MODE_DENSE = 2, MODE_LEVEL_RN = 3 };
__host__ __device__ constexpr bool is_level(int mode) { return mode == MODE_LEVEL || mode == MODE_LEVEL_RN; }

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
    const int32_t *Srn;    // LEVEL_RN: row-norm draws [bh][nodes_total][m] (local key row, -1: none)
    const float *lwrn;     // LEVEL_RN: their natural-log weights log(1 / (m p_j))
    int nr;                // LEVEL_RN: row-norm chunks (0 otherwise)
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
    int64_t stall_ns;      // test hook: > 0 makes the first softmax wait give up after this long (see bNever)
    int64_t items;
    uint32_t per_outer;    // LEVEL: items per problem; CAUSAL: items per query-tile pair index
};

struct Item {
    bool v0, v1;          // tile validity
    int nc0, nc1;         // key chunks of each tile (0 when invalid)
    int nc_max, npairs;
    // LEVEL
    int64_t prob, blk, bhi, node;
    int pair;
    // CAUSAL
    int64_t leaf_start;   // global row of the leaf's first row (bhi * n + leaf offset)
    int gt0, gt1;         // query tile index within the leaf
};

// Item index -> item. Item counts, problem counts and their factors are below 2^31 (checked on the host), so the
// divisions are 32-bit.
template <int MODE>
__device__ __forceinline__ Item decode(const TcArgs &a, int64_t it64) {
    Item x{};
    const uint32_t it = static_cast<uint32_t>(it64);
    if (is_level(MODE)) {
        const uint32_t prob = it / a.per_outer;
        const uint32_t rem = it - prob * a.per_outer;
        const uint32_t ppb = static_cast<uint32_t>(a.pairs_per_block);
        const uint32_t blk = rem / ppb;
        x.prob = prob;
        x.blk = blk;
        x.pair = static_cast<int>(rem - blk * ppb);
        const uint32_t nodes = static_cast<uint32_t>(a.lv.nodes);
        const uint32_t bhi = prob / nodes;
        x.bhi = bhi;
        x.node = prob - bhi * nodes;
        x.v0 = x.pair * 2 < a.tiles_per_block;
        x.v1 = x.pair * 2 + 1 < a.tiles_per_block;
        x.nc0 = x.v0 ? a.nb + a.ns + a.nr : 0;
        x.nc1 = x.v1 ? a.nb + a.ns + a.nr : 0;
    } else {
        const uint32_t po = it / a.per_outer;
        const int pair = a.pairs_per_leaf - 1 - static_cast<int>(po);   // heaviest first
        const uint32_t rem = it - po * a.per_outer;
        const uint32_t nl = static_cast<uint32_t>(a.nleaves);
        const uint32_t bhi = rem / nl;
        x.bhi = bhi;
        x.leaf_start = static_cast<int64_t>(bhi) * a.n + static_cast<int64_t>(rem - bhi * nl) * a.leaf;
        x.pair = pair;
        x.gt0 = pair * 2;
        x.gt1 = pair * 2 + 1;
        x.v0 = x.gt0 < a.tiles_per_leaf;
        x.v1 = x.gt1 < a.tiles_per_leaf;
        x.nc0 = x.v0 ? (MODE == MODE_DENSE ? a.tiles_per_leaf : x.gt0 + 1) : 0;
        x.nc1 = x.v1 ? (MODE == MODE_DENSE ? a.tiles_per_leaf : x.gt1 + 1) : 0;
    }
    x.nc_max = max(x.nc0, x.nc1);
    x.npairs = x.nc0 + x.nc1;
    return x;
}

// Position of pair (t, c) in the item's pair order (c-major, t-minor, skipping finished tiles).
__device__ __forceinline__ int pair_index(const Item &x, int t, int c) {
    const int mn = min(x.nc0, x.nc1);
    if (mn == 0) return c;
    if (c < mn) return 2 * c + t;
    return 2 * mn + (c - mn);
}

// Inverse of pair_index.
__device__ __forceinline__ void pair_tc(const Item &x, int k, int &t, int &c) {
    const int mn = min(x.nc0, x.nc1);
    if (mn == 0) { t = x.v0 ? 0 : 1; c = k; return; }
    if (k < 2 * mn) { t = k & 1; c = k >> 1; return; }
    t = x.nc0 > x.nc1 ? 0 : 1;
    c = mn + (k - 2 * mn);
}

__device__ __forceinline__ void flag_status(int *status) {
    if (status) atomicOr(status, kStatusTimeout);
}

// HA_DEBUG builds: a row index read from data (a permutation, a sample list) outside [0, limit) sets
// kStatusBounds in the status word and is replaced by 0, so that the kernel reads a valid row instead of
// faulting. Regular builds compile the check away.
__device__ __forceinline__ int32_t checked_index(int32_t i, int64_t limit, int *status) {
#ifdef HA_DEBUG
    if (i < 0 || i >= limit) {
        if (status) atomicOr(status, kStatusBounds);
        return 0;
    }
#endif
    (void)limit;
    (void)status;
    return i;
}

// The same check, in place, on `count` entries of an index array in shared memory (the warp's lanes strided).
__device__ __forceinline__ void check_indices(int32_t *idx, int count, int64_t limit, int *status, int lane) {
#ifdef HA_DEBUG
    __syncwarp();
    for (int i = lane; i < count; i += 32) idx[i] = checked_index(idx[i], limit, status);
    __syncwarp();
#endif
    (void)idx;
    (void)count;
    (void)limit;
    (void)status;
    (void)lane;
}

// One SEG-byte segment, at byte offset `off`, of each of the warp's 32 output rows: lane l holds the segment of
// its own row (16-byte pieces pc[0..SEG/16)) and `drow` points at the start of that row. The segments pass
// through the warp's shared-memory stage (32 x SEG bytes, pieces XOR-swizzled so that neither the row-wise
// writes nor the column-wise reads conflict on banks), so that SEG/16 consecutive lanes store one row's SEG
// contiguous bytes: an instruction touches 32 / (SEG/16) rows instead of 32.
template <int SEG>
__device__ __forceinline__ void warp_store_segment(unsigned char *stage, unsigned char *drow, int off,
                                                   const uint4 (&pc)[SEG / 16], int lane) {
    constexpr int P = SEG / 16, SH = SEG == 64 ? 1 : 0;
    __syncwarp();   // the previous segment's reads of the stage are done
#pragma unroll
    for (int j = 0; j < P; ++j)
        *reinterpret_cast<uint4 *>(stage + lane * SEG + ((j ^ ((lane >> SH) & (P - 1))) << 4)) = pc[j];
    __syncwarp();
    const int sub = lane / P, piece = lane % P;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const int row = i * (32 / P) + sub;
        const uint4 v = *reinterpret_cast<const uint4 *>(stage + row * SEG + ((piece ^ ((row >> SH) & (P - 1))) << 4));
        unsigned char *rb = reinterpret_cast<unsigned char *>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(drow), row));
        *reinterpret_cast<uint4 *>(rb + off + piece * 16) = v;
    }
}

// Write the warp's 32 rows of D output values (bf16 or fp32; lane l owns row l at `drow`). vals(j, v) yields
// the row's columns [32 j, 32 j + 32) as floats.
template <int D, int SEG, typename F>
__device__ __forceinline__ void warp_write_rows(unsigned char *stage, unsigned char *drow, bool bf16, int lane,
                                                F &&vals) {
    constexpr int PS = SEG / 16;
    uint4 seg[PS];
    if (bf16) {
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
            float v[32];
            vals(j, v);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pi = j * 4 + q;
                seg[pi % PS] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                          pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                if (pi % PS == PS - 1) warp_store_segment<SEG>(stage, drow, (pi / PS) * SEG, seg, lane);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
            float v[32];
            vals(j, v);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int pi = j * 8 + q;
                seg[pi % PS] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                          __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
                if (pi % PS == PS - 1) warp_store_segment<SEG>(stage, drow, (pi / PS) * SEG, seg, lane);
            }
        }
    }
}

// byte offset of 16-byte piece j of row `row` inside a 128-row, 128-byte-swizzled tile (slab s = 64 columns)
__device__ __forceinline__ uint32_t swz(int slab, int row, int j) {
    return static_cast<uint32_t>(slab * (128 * 128) + row * 128 + ((j ^ (row & 7)) << 4));
}

// MODE (MODE_LEVEL, MODE_LEVEL_RN, MODE_CAUSAL or MODE_DENSE) is a compile-time parameter: each instance holds
// only its own mode's loads,
// masks and epilogue, which keeps the instruction footprint of the concurrently running roles small (measured:

// Copy ROWS rows of a [*, D] bf16 matrix into a ROWS-row, 128-byte-swizzled tile at shared address `dst` with 16-byte
// cp.async (lane l copies piece l mod D/8 of every (32 / (D/8))-th row). Row i is global row add + list[i] (LIST,
// list in shared memory) or add + i. A batch of row indices is read into registers before its copies, so that the
// copies issue back to back (each copy is an asm statement with a memory clobber, which would otherwise order every
// index read behind the previous copy).
template <int D, bool LIST, int ROWS = 128>
__device__ __forceinline__ void gather_rows(uint32_t dst, const uint16_t *src, int64_t add, const int32_t *list,
                                            int lane) {
    constexpr int PPR = D / 8, RPI = 32 / PPR, IT = ROWS / RPI, BATCH = IT < 32 ? IT : 32;
    const int rsub = lane / PPR, piece = lane % PPR, slab = piece >> 3, jp = piece & 7;
    const uint16_t *col = src + piece * 8;
#pragma unroll
    for (int i0 = 0; i0 < IT; i0 += BATCH) {
        int32_t idx[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) idx[i] = LIST ? list[(i0 + i) * RPI + rsub] : (i0 + i) * RPI + rsub;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int row = (i0 + i) * RPI + rsub;
            cp_async16(dst + static_cast<uint32_t>(slab * (ROWS * 128) + row * 128 + ((jp ^ (row & 7)) << 4)),
                       col + (add + idx[i]) * D);
        }
    }
}

}  // namespace attn

// The per-tile score-buffer kernel of ha_attn_pp.cu for the modes and head dims it covers (returns -2 for the
// others, the number of kernels launched, or -1 on a launch error).
int launch_attn_pp(int d, const attn::TcArgs &args, int sms, cudaStream_t st);

}  // namespace ha
