// ha_internal.h -- declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ha {

constexpr int kMaxR = 16;            // hash bits
constexpr int kMaxPassBits = 10;     // radix digit of one counting-sort pass (<= 1024 buckets)
constexpr int kSortChunk = 2048;     // rows per counting-sort chunk (one CTA)
constexpr int kSortWarps = 8;

// Device status word bits (written by kernels that wait with a bound, read by hyper_attn_status).
constexpr int kStatusTimeout = 1;
constexpr int kStatusBounds = 2;     // HA_DEBUG builds: a row index read from data was out of range

// One level of the computation. Level 0 is the non-causal problem (one node covering all n rows);
// causal level l >= 1 has nodes of node_len = n >> (l-1) rows whose off-diagonal problem pairs the
// query rows [q_off, node_len) with the key rows [0, seg_len) of the node (q_off = seg_len = node_len/2).
struct Level {
    int64_t n;          // rows per (batch, head)
    int64_t bh;         // batch * heads
    int64_t nodes;      // nodes at this level
    int64_t node_len;   // rows per node
    int64_t seg_len;    // N: query rows = key rows of one problem
    int64_t q_off;      // first query row of a node, relative to the node start
    int64_t heap0;      // heap id of node 0 of this level
    int level;          // 0 = non-causal, >= 1 causal level
    int bp;             // block size b' = min(block, N)
};

// Sort pass description: digit = (rank >> shift) & (radix - 1).
struct SortPass {
    int shift;
    int radix;          // power of two <= 1 << kMaxPassBits
};

// ---- kernels (launch wrappers return the number of kernels launched, or -1 on launch error) ----

// sortLSH hash of 2*bh*n rows (Q rows then K rows of each problem): rank[bh][2][n], near[bh][2][n].
// P is the [d][r] projection matrix in host memory (it travels in the launch's parameters).
int launch_hash(const void *Q, const void *K, int dtype, int64_t bh, int64_t n, int d, const float *P, int r,
                uint16_t *rank, uint8_t *near, cudaStream_t st);

// Stable counting sort of all segments of a level by one digit.
//   in_idx: nullptr (rows in natural order) or the previous pass's permutation (same layout as perm).
//   perm[s*N + pos] = local row; inv[s*N + row] = pos (inv may be nullptr).
int launch_sort_pass(const Level &lv, const uint16_t *rank, SortPass ps, const int32_t *in_idx,
                     int32_t *hist, int32_t *perm, int32_t *inv, cudaStream_t st);

// SIMT attention of one level: for level 0 writes O (out dtype); for causal levels writes the parts
// Opart[bh][n/2][d] (fp32, normalised) and Lpart[bh][n/2] (log normaliser) of this level.
// Srn/lwrn (nullptr for uniform sampling): row-norm draws and their log weights, [bh][nodes_total][m]; when
// given, the uniform samples S feed only the normaliser and the row-norm draws only the product with V.
int launch_attn_simt(const Level &lv, const void *Q, const void *K, const void *V, int dtype, int d,
                     const int32_t *perm, const int32_t *inv, const int32_t *S, int m, int64_t nodes_total,
                     void *O, int out_dtype, float *lse, float *Opart, float *Lpart, cudaStream_t st,
                     const int32_t *Srn = nullptr, const float *lwrn = nullptr);

// SIMT exact causal attention on leaves of `leaf` rows, merged with the parts of levels 1..L.
// Lout (optional): the final log normaliser of every row [bh][n].
int launch_causal_base_simt(const void *Q, const void *K, const void *V, int dtype, int64_t bh, int64_t n,
                            int d, int64_t leaf, int levels, const float *Opart, const float *Lpart,
                            void *O, int out_dtype, cudaStream_t st, float *Lout = nullptr);

// Tensor-core (tcgen05) kernels; return -2 when a shape is not supported by the tensor-core path.
int launch_attn_tc(const Level &lv, const void *Q, const void *K, const void *V, int d,
                   const int32_t *perm, const int32_t *inv, const int32_t *S, int m, int64_t nodes_total,
                   void *O, int out_dtype, float *lse, float *Opart, float *Lpart, int *status, cudaStream_t st,
                   int64_t stall_ns = 0, const int32_t *Srn = nullptr, const float *lwrn = nullptr);
// Srn/lwrn (row-norm sampling, m <= 256; larger m returns -2): as for launch_attn_simt.
int launch_causal_base_tc(const void *Q, const void *K, const void *V, int64_t bh, int64_t n, int d,
                          int64_t leaf, int levels, const float *Opart, const float *Lpart,
                          void *O, int out_dtype, int *status, cudaStream_t st, int64_t stall_ns = 0);
// stall_ns > 0 (test hook): the first softmax wait gives up after stall_ns on a barrier nothing completes.
// Exact softmax attention (causal: keys up to the query) of bh problems of n rows on the tensor cores.
int launch_exact_tc(const void *Q, const void *K, const void *V, int64_t bh, int64_t n, int d, int causal, void *O,
                    int out_dtype, int *status, cudaStream_t st);

// Hardness diagnostics (ha_diag.cu) of bh non-causal problems of n rows: out[2b] = alpha, out[2b+1] = kappa.
// inv: level-0 inverse permutations [bh][2][n]; scratch: 4 * bh * n floats.
int launch_diagnostics(const void *Q, const void *K, int dtype, int64_t bh, int64_t n, int d, const int32_t *inv,
                       int64_t bp, int64_t first_col, float *scratch, double *out, cudaStream_t st);

// Row-norm samples (ha_rownorm.cu): geometry of the sample sets of one call. Set (problem b, heap node k) has
// m draws; its cumulative distribution lives at cdf[b * per_prob + offset of the set].
struct RowNormGeom {
    int64_t n;
    int causal;
    int depths;             // 1 (non-causal) or the causal levels L
    int m;
    int64_t nodes_total;    // sample sets per problem
    int64_t slot0[33];      // first 2048-row chunk slot of each depth; slot0[depths] = slots
    int64_t slots;          // chunk slots per problem
    int64_t per_prob;       // cdf doubles per problem: n (non-causal) or L * n / 2
};
RowNormGeom rownorm_geometry(int64_t n, int causal, int levels, int m, int64_t nodes_total);
// Squared norms nrm[bh][n] (fp32), chunk sums csum[bh][slots], cdf[bh][per_prob] (double), then the draws
// S[bh][nodes_total][m] (row index local to the set's key rows, -1 when all its rows are zero) and their log
// weights logw[bh][nodes_total][m] = log(total / (m ||v_j||^2)). Returns the kernels launched, -1 on error,
// -2 if bh exceeds the grid's second dimension.
int launch_rownorm_draws(const RowNormGeom &g, const void *V, int dtype, int d, int64_t bh, uint64_t seed,
                         int64_t bh_offset, float *nrm, double *csum, double *cdf, int32_t *S, float *logw,
                         cudaStream_t st);

// Backward pass (ha_backward.cu): g[rows] = dO . O (O fp32); the key terms of one level and of the exact causal
// leaves, adding into fp32 dQ, dK, dV [bh][n][d] (zeroed by the caller). L: final log normaliser [bh][n].
int launch_bwd_rowdot(const void *dO, int dtype, const float *O, int64_t rows, int d, float *g, cudaStream_t st);
int launch_bwd_level(const Level &lv, const void *Q, const void *K, const void *V, const void *dO, int dtype, int d,
                     const int32_t *perm, const int32_t *inv, const int32_t *S, int m, int64_t nodes_total,
                     const int32_t *Srn, const float *lwrn, const float *L, const float *g, float *dQ, float *dK,
                     float *dV, cudaStream_t st);
int launch_bwd_leaf(const void *Q, const void *K, const void *V, const void *dO, int dtype, int64_t bh, int64_t n,
                    int d, int64_t leaf, const float *L, const float *g, float *dQ, float *dK, float *dV,
                    cudaStream_t st);

// ---- host-side draws (ha_draws.cpp) ----
void draw_projection(uint64_t seed, int d, int r, float *P);
int draw_samples(uint64_t seed, uint64_t bh, uint64_t node, int64_t N, int m, int32_t *S, uint8_t *scratch);

}  // namespace ha
