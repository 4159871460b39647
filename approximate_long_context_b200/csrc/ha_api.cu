// ha_api.cu -- the C ABI (include/hyper_attn.h): argument checks, the handle's workspace, the host-side
// draws and the launch sequence of the forward pass. No step of the method is computed here; every step
// runs in the kernels of ha_hash.cu, ha_sort.cu, ha_attn_simt.cu and ha_attn_tc.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/hyper_attn.h"
#include "ha_internal.h"

struct hyper_attn_s {
    int device = 0;
    ha_options opt{};
    std::string err;
    // device workspace (grow-only)
    unsigned char *ws = nullptr;
    size_t ws_bytes = 0;
    // page-locked staging of the draws, and the event that guards its reuse
    unsigned char *pin = nullptr;
    size_t pin_bytes = 0;
    cudaEvent_t pin_free = nullptr;
    // device copies for hyper_attn_forward_host (grow-only), and its copy streams and chunk events
    unsigned char *io = nullptr;
    size_t io_bytes = 0;
    cudaStream_t cs_in = nullptr, cs_out = nullptr;
    std::vector<cudaEvent_t> pipe_ev;
    // test hook: the number of upcoming allocations to fail (hyper_attn_test_fail_alloc)
    int fail_alloc = 0;
    // draws currently resident in the workspace, and a host copy of their projection matrix ([d][r]), which the
    // hash kernel takes as launch parameters
    bool draws_valid = false;
    std::vector<float> hostP;
    uint64_t dk_seed = 0;
    int dk_d = 0, dk_r = 0, dk_m = 0, dk_causal = 0;
    int64_t dk_bh = 0, dk_n = 0, dk_base = 0, dk_off = 0;
    // layout of the last forward (for debug copies)
    struct Layout {
        size_t status, P, S, rank, near, lse, perm_tmp, hist, Opart, Lpart, end;
        std::vector<size_t> perm, inv;
        std::vector<size_t> perm_bytes;
        size_t rank_bytes, near_bytes, lse_bytes;
        // row-norm sampling (0 bytes when off): squared norms, chunk sums, cumulative sums, draws, log weights
        size_t rn_nrm, rn_csum, rn_cdf, rn_S, rn_lw, rn_bytes;
    } lay{};
    bool have_last = false;
    // the forward pass runs for a backward pass: fp32 O, per-row log normalisers captured (causal: final ones)
    bool bwd = false;
    int last_launches = 0;
    int last_kernel = 0;
    // profiling: event pairs recorded around kernel-class launches
    bool profiling = false;
    std::vector<cudaEvent_t> ev_pool;
    struct Rec { int cls, launches; size_t e0, e1; };
    std::vector<Rec> recs;
    size_t ev_used = 0;
};

namespace {

constexpr int kVersion = 100;   // 0.1.0
constexpr int kDiagMaxN = 16384;   // the diagnostics visit every entry of A

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

int fail(hyper_attn_t h, int code, const char *fmt, ...) __attribute__((format(printf, 3, 4)));
int fail(hyper_attn_t h, int code, const char *fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        h->err = buf;
    }
    return code;
}

#define HA_CUDA(h, call)                                                                                \
    do {                                                                                                \
        cudaError_t e_ = (call);                                                                        \
        if (e_ != cudaSuccess) return fail((h), HA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));  \
    } while (0)

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Causal recursion depth: n <= base -> 0 levels (one exact causal problem); else n = base * 2^L.
int causal_levels(int64_t n, int64_t base, int *L) {
    if (base <= 0 || n <= 0) return -1;
    int l = 0;
    int64_t x = n;
    while (x > base) {
        if (x & 1) return -1;
        x >>= 1;
        ++l;
    }
    if (l > 0 && x != base) return -1;
    *L = l;
    return 0;
}

struct Shape {
    int64_t n, bh;
    int d, block, m, r, causal;
    int levels;          // causal levels L (0 for non-causal)
    int64_t nodes_total; // sample sets per problem
    int64_t leaf;        // exact causal leaf rows
    int nlev;            // sort levels: 1 (non-causal, level 0) or L (causal, levels 1..L)
};

int check_shape(hyper_attn_t h, int64_t n, int d, int64_t bh, int block, int m, int r, int causal, Shape *s) {
    if (n <= 0) return fail(h, HA_ERR_INVALID_ARG, "n must be positive (got %lld)", (long long)n);
    if (n > (int64_t(1) << 30)) return fail(h, HA_ERR_INVALID_ARG, "n too large (%lld)", (long long)n);
    if (d != 64 && d != 128) return fail(h, HA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
    if (bh <= 0) return fail(h, HA_ERR_INVALID_ARG, "batch*heads must be positive");
    if (block <= 0) return fail(h, HA_ERR_INVALID_ARG, "block must be positive (got %d)", block);
    if (m < 0) return fail(h, HA_ERR_INVALID_ARG, "m must be >= 0 (got %d)", m);
    if (r < 0 || r > ha::kMaxR) return fail(h, HA_ERR_INVALID_ARG, "r must be in [0, 16] (got %d)", r);
    if (causal != 0 && causal != 1) return fail(h, HA_ERR_INVALID_ARG, "causal must be 0 or 1");
    s->n = n; s->bh = bh; s->d = d; s->block = block; s->m = m; s->r = r; s->causal = causal;
    if (!causal) {
        const int64_t bp = block < n ? block : n;
        if (n % bp) return fail(h, HA_ERR_INVALID_ARG, "n (%lld) must be a multiple of min(block, n) (%lld)",
                                (long long)n, (long long)bp);
        if (m > n) return fail(h, HA_ERR_INVALID_ARG, "m (%d) must be <= n (%lld)", m, (long long)n);
        s->levels = 0; s->nodes_total = 1; s->leaf = 0; s->nlev = 1;
        return HA_OK;
    }
    const int64_t base = h ? h->opt.causal_base : 0;
    int L = 0;
    if (causal_levels(n, base, &L))
        return fail(h, HA_ERR_INVALID_ARG, "causal needs n <= base or n = base * 2^L (n=%lld, base=%lld)",
                    (long long)n, (long long)base);
    for (int l = 1; l <= L; ++l) {
        const int64_t N = n >> l;
        const int64_t bp = block < N ? block : N;
        if (N % bp) return fail(h, HA_ERR_INVALID_ARG, "level %d: N=%lld not a multiple of block", l, (long long)N);
        if (m > N) return fail(h, HA_ERR_INVALID_ARG, "level %d: m=%d > N=%lld", l, m, (long long)N);
    }
    s->levels = L;
    s->nodes_total = (int64_t(1) << L) - 1;
    s->leaf = n < base ? n : base;
    s->nlev = L;
    return HA_OK;
}

ha::Level make_level(const Shape &s, int l) {
    ha::Level lv{};
    lv.n = s.n;
    lv.bh = s.bh;
    lv.level = l;
    if (l == 0) {
        lv.nodes = 1; lv.node_len = s.n; lv.seg_len = s.n; lv.q_off = 0; lv.heap0 = 1;
    } else {
        lv.nodes = int64_t(1) << (l - 1);
        lv.node_len = s.n >> (l - 1);
        lv.seg_len = lv.node_len / 2;
        lv.q_off = lv.seg_len;
        lv.heap0 = lv.nodes;
    }
    lv.bp = static_cast<int>(s.block < lv.seg_len ? s.block : lv.seg_len);
    return lv;
}

void sort_passes(int r, ha::SortPass *p, int *np) {
    if (r <= ha::kMaxPassBits) {
        p[0] = {0, 1 << r};
        *np = 1;
    } else {
        const int lo = (r + 1) / 2, hi = r - lo;
        p[0] = {0, 1 << lo};
        p[1] = {lo, 1 << hi};
        *np = 2;
    }
}

// Lay out the workspace for shape s; returns total bytes.
size_t plan_layout(const Shape &s, int esz_in, int capture, bool rownorm, hyper_attn_s::Layout *L) {
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += align_up(bytes ? bytes : 1); return o; };
    L->status = take(256);
    L->P = take(sizeof(float) * ha::kMaxR * 128);
    L->S = take(sizeof(int32_t) * s.bh * s.nodes_total * (s.m > 0 ? s.m : 1));
    L->rank_bytes = sizeof(uint16_t) * s.bh * 2 * s.n;
    L->rank = take(L->rank_bytes);
    L->near_bytes = s.bh * 2 * s.n;
    L->near = take(L->near_bytes);
    L->lse_bytes = capture ? sizeof(float) * s.bh * s.n : 0;
    L->lse = take(L->lse_bytes);
    L->perm.clear(); L->inv.clear(); L->perm_bytes.clear();
    size_t hist_max = 0, perm_max = 0;
    for (int i = 0; i < s.nlev; ++i) {
        const ha::Level lv = make_level(s, s.causal ? i + 1 : 0);
        const size_t pb = sizeof(int32_t) * lv.bh * lv.nodes * 2 * lv.seg_len;
        L->perm_bytes.push_back(pb);
        L->perm.push_back(take(pb));
        L->inv.push_back(take(pb));
        perm_max = pb > perm_max ? pb : perm_max;
        const int64_t cps = (lv.seg_len + ha::kSortChunk - 1) / ha::kSortChunk;
        const size_t hb = sizeof(int32_t) * lv.bh * lv.nodes * 2 * cps * (1 << ha::kMaxPassBits);
        hist_max = hb > hist_max ? hb : hist_max;
    }
    L->perm_tmp = take(s.r > ha::kMaxPassBits ? perm_max : 0);
    L->hist = take(hist_max);
    const size_t half_rows = static_cast<size_t>(s.bh) * (s.n / 2);
    L->Opart = take(s.causal ? sizeof(float) * s.levels * half_rows * s.d : 0);
    L->Lpart = take(s.causal ? sizeof(float) * s.levels * half_rows : 0);
    const ha::RowNormGeom g = ha::rownorm_geometry(s.n, s.causal, s.levels, s.m, s.nodes_total);
    const size_t draws = rownorm ? static_cast<size_t>(s.bh) * s.nodes_total * s.m : 0;
    L->rn_nrm = take(rownorm ? sizeof(float) * s.bh * s.n : 0);
    L->rn_csum = take(rownorm ? sizeof(double) * s.bh * g.slots : 0);
    L->rn_cdf = take(rownorm ? sizeof(double) * s.bh * g.per_prob : 0);
    L->rn_bytes = draws * 4;
    L->rn_S = take(L->rn_bytes);
    L->rn_lw = take(L->rn_bytes);
    L->end = off;
    (void)esz_in;
    return off;
}

// Every allocation of a handle goes through these, so that the allocation-failure test hook can fail one.
cudaError_t device_alloc(hyper_attn_t h, unsigned char **p, size_t bytes) {
    if (h->fail_alloc > 0) {
        --h->fail_alloc;
        return cudaErrorMemoryAllocation;
    }
    return cudaMalloc(p, bytes);
}

cudaError_t host_alloc(hyper_attn_t h, unsigned char **p, size_t bytes) {
    if (h->fail_alloc > 0) {
        --h->fail_alloc;
        return cudaErrorMemoryAllocation;
    }
    return cudaMallocHost(p, bytes);
}

int ensure_workspace(hyper_attn_t h, size_t bytes) {
    if (bytes <= h->ws_bytes) return HA_OK;
    if (h->ws) {
        cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
        HA_CUDA(h, cudaStreamSynchronize(st));
        HA_CUDA(h, cudaFree(h->ws));
        h->ws = nullptr;
        h->ws_bytes = 0;
    }
    h->draws_valid = false;
    const size_t want = align_up(bytes + bytes / 8, 1 << 20);
    if (device_alloc(h, &h->ws, want) != cudaSuccess) {
        cudaGetLastError();
        h->ws = nullptr;
        return fail(h, HA_ERR_OOM, "workspace allocation of %zu bytes failed", want);
    }
    h->ws_bytes = want;
    HA_CUDA(h, cudaMemset(h->ws, 0, 256));   // status word
    return HA_OK;
}

int ensure_pinned(hyper_attn_t h, size_t bytes) {
    if (bytes <= h->pin_bytes) return HA_OK;
    if (h->pin) {
        HA_CUDA(h, cudaEventSynchronize(h->pin_free));
        HA_CUDA(h, cudaFreeHost(h->pin));
        h->pin = nullptr;
        h->pin_bytes = 0;
    }
    const size_t want = align_up(bytes, 1 << 16);
    if (host_alloc(h, &h->pin, want) != cudaSuccess) {
        cudaGetLastError();
        h->pin = nullptr;
        return fail(h, HA_ERR_OOM, "page-locked staging of %zu bytes failed", want);
    }
    h->pin_bytes = want;
    return HA_OK;
}

// Fill host buffers with the draws of shape s (P: [d][r]; S: [bh][nodes_total][m]).
int host_draws(uint64_t seed, const Shape &s, int64_t bh_offset, float *P, int32_t *S) {
    if (P) ha::draw_projection(seed, s.d, s.r, P);
    if (!S || s.m == 0) return 0;
    std::vector<uint8_t> scratch(static_cast<size_t>(s.n), 0);
    for (int64_t b = 0; b < s.bh; ++b) {
        for (int64_t k = 0; k < s.nodes_total; ++k) {
            const int64_t node = k + 1;
            int64_t N = s.n;
            if (s.causal) {
                int depth = 0;
                for (int64_t x = node; x > 1; x >>= 1) ++depth;
                N = s.n >> (depth + 1);
            }
            if (ha::draw_samples(seed, static_cast<uint64_t>(bh_offset + b), static_cast<uint64_t>(node), N, s.m,
                                 S + (b * s.nodes_total + k) * s.m, scratch.data()))
                return -1;
        }
    }
    return 0;
}

int upload_draws(hyper_attn_t h, uint64_t seed, const Shape &s, int64_t bh_offset, cudaStream_t st) {
    if (h->draws_valid && h->dk_seed == seed && h->dk_d == s.d && h->dk_r == s.r && h->dk_m == s.m &&
        h->dk_causal == s.causal && h->dk_bh == s.bh && h->dk_n == s.n && h->dk_off == bh_offset &&
        (!s.causal || h->dk_base == h->opt.causal_base))
        return HA_OK;
    const size_t pbytes = sizeof(float) * ha::kMaxR * 128;
    const size_t sbytes = sizeof(int32_t) * s.bh * s.nodes_total * s.m;
    int rc = ensure_pinned(h, pbytes + sbytes + 16);
    if (rc) return rc;
    HA_CUDA(h, cudaEventSynchronize(h->pin_free));   // the previous upload has left the staging buffer
    float *P = reinterpret_cast<float *>(h->pin);
    int32_t *S = reinterpret_cast<int32_t *>(h->pin + pbytes);
    if (host_draws(seed, s, bh_offset, P, S)) return fail(h, HA_ERR_INVALID_ARG, "sample draw failed");
    h->hostP.assign(P, P + static_cast<size_t>(s.d) * s.r);
    HA_CUDA(h, cudaMemcpyAsync(h->ws + h->lay.P, P, sizeof(float) * s.d * (s.r ? s.r : 1), cudaMemcpyHostToDevice, st));
    if (sbytes) HA_CUDA(h, cudaMemcpyAsync(h->ws + h->lay.S, S, sbytes, cudaMemcpyHostToDevice, st));
    HA_CUDA(h, cudaEventRecord(h->pin_free, st));
    h->draws_valid = true;
    h->dk_seed = seed; h->dk_d = s.d; h->dk_r = s.r; h->dk_m = s.m; h->dk_causal = s.causal;
    h->dk_bh = s.bh; h->dk_n = s.n; h->dk_base = h->opt.causal_base; h->dk_off = bh_offset;
    return HA_OK;
}

// The forward pass of shape s on device buffers; the problems' draws are keyed from global index bh_offset.
// sort_only: stop after the hash and the sort (their outputs stay in the workspace; V and O are not used).
int run_forward(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O, const Shape &s,
                uint64_t seed, int64_t bh_offset, bool sort_only = false) {
    cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
    const int dtype = h->opt.dtype;
    const int out_dtype = h->bwd ? HA_DTYPE_FP32 : (h->opt.out_dtype < 0 ? dtype : h->opt.out_dtype);
    const int esz = dtype == HA_DTYPE_BF16 ? 2 : 4;
    const int capture = h->opt.debug_captures || h->bwd;
    bool use_tc = false;
    if (h->opt.kernel == HA_KERNEL_TC) {
        if (dtype != HA_DTYPE_BF16) return fail(h, HA_ERR_UNSUPPORTED, "tensor-core kernels need bf16 inputs");
        use_tc = true;
    } else if (h->opt.kernel == HA_KERNEL_AUTO) {
        use_tc = dtype == HA_DTYPE_BF16;
    }

    const bool rownorm = h->opt.sampling == HA_SAMPLING_ROWNORM && s.m > 0 && !sort_only;
    hyper_attn_s::Layout lay;
    const size_t bytes = plan_layout(s, esz, capture, rownorm, &lay);
    int rc = ensure_workspace(h, bytes);
    if (rc) return rc;
    // a layout change invalidates resident draws only if their offsets moved
    if (h->have_last && (lay.P != h->lay.P || lay.S != h->lay.S)) h->draws_valid = false;
    h->lay = lay;
    h->have_last = true;
    rc = upload_draws(h, seed, s, bh_offset, st);
    if (rc) return rc;

    unsigned char *ws = h->ws;
    const int32_t *S = reinterpret_cast<const int32_t *>(ws + lay.S);
    uint16_t *rank = reinterpret_cast<uint16_t *>(ws + lay.rank);
    uint8_t *near = ws + lay.near;
    int32_t *hist = reinterpret_cast<int32_t *>(ws + lay.hist);
    int32_t *perm_tmp = reinterpret_cast<int32_t *>(ws + lay.perm_tmp);
    float *lse = capture ? reinterpret_cast<float *>(ws + lay.lse) : nullptr;
    float *Opart = reinterpret_cast<float *>(ws + lay.Opart);
    float *Lpart = reinterpret_cast<float *>(ws + lay.Lpart);
    int *status = reinterpret_cast<int *>(ws + lay.status);
    const int64_t stall_ns = static_cast<int64_t>(h->opt.test_stall_ms) * 1000000;   // test hook, 0 = off
    const size_t half_rows = static_cast<size_t>(s.bh) * (s.n / 2);

    int launches = 0;
    int family = 0;
    // every kernel class's enqueue sits in an NVTX range (a no-op unless a tracing tool is attached); with
    // profiling on, two events from the pool (grown on demand) bracket it on the stream
    static const char *const kRangeName[HA_KC_COUNT] = {"ha:hash", "ha:sort", "ha:attn", "ha:causal_base",
                                                        "ha:draws"};
    auto prof_begin = [&](int cls) -> long {
        nvtxRangePushA(kRangeName[cls]);
        if (!h->profiling) return -1;
        while (h->ev_pool.size() < h->ev_used + 2) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return -1;
            h->ev_pool.push_back(e);
        }
        const size_t i = h->ev_used;
        h->ev_used += 2;
        cudaEventRecord(h->ev_pool[i], st);
        return static_cast<long>(i);
    };
    auto prof_end = [&](long i, int cls, int k) {
        nvtxRangePop();
        if (i < 0) return;
        cudaEventRecord(h->ev_pool[i + 1], st);
        h->recs.push_back({cls, k > 0 ? k : 0, static_cast<size_t>(i), static_cast<size_t>(i + 1)});
    };
    auto count = [&](int k, const char *what) -> int {
        if (k < 0) {
            cudaError_t e = cudaGetLastError();
            return fail(h, k == -2 ? HA_ERR_UNSUPPORTED : HA_ERR_CUDA, "%s launch failed: %s", what,
                        k == -2 ? "shape not supported by this kernel" : cudaGetErrorString(e));
        }
        launches += k;
        return HA_OK;
    };

    const int32_t *Srn = nullptr;
    const float *lwrn = nullptr;
    long ev;
    int kl;
    if (rownorm) {
        const ha::RowNormGeom g = ha::rownorm_geometry(s.n, s.causal, s.levels, s.m, s.nodes_total);
        int32_t *rS = reinterpret_cast<int32_t *>(ws + lay.rn_S);
        float *rlw = reinterpret_cast<float *>(ws + lay.rn_lw);
        ev = prof_begin(HA_KC_DRAWS);
        kl = ha::launch_rownorm_draws(g, V, dtype, s.d, s.bh, seed, bh_offset, reinterpret_cast<float *>(ws + lay.rn_nrm),
                                      reinterpret_cast<double *>(ws + lay.rn_csum),
                                      reinterpret_cast<double *>(ws + lay.rn_cdf), rS, rlw, st);
        prof_end(ev, HA_KC_DRAWS, kl);
        if (kl == -2) return fail(h, HA_ERR_UNSUPPORTED, "row-norm sampling supports at most 65535 problems per call");
        if ((rc = count(kl, "row-norm draws"))) return rc;
        Srn = rS;
        lwrn = rlw;
    }
    ev = prof_begin(HA_KC_HASH);
    kl = ha::launch_hash(Q, K, dtype, s.bh, s.n, s.d, h->hostP.data(), s.r, rank, near, st);
    prof_end(ev, HA_KC_HASH, kl);
    if ((rc = count(kl, "hash"))) return rc;

    ha::SortPass passes[2];
    int npass = 0;
    sort_passes(s.r, passes, &npass);
    const bool any_level = !s.causal || s.levels > 0;
    for (int i = 0; any_level && i < s.nlev; ++i) {
        const int l = s.causal ? i + 1 : 0;
        const ha::Level lv = make_level(s, l);
        int32_t *perm = reinterpret_cast<int32_t *>(ws + lay.perm[i]);
        int32_t *inv = reinterpret_cast<int32_t *>(ws + lay.inv[i]);
        ev = prof_begin(HA_KC_SORT);
        if (npass == 1) {
            kl = ha::launch_sort_pass(lv, rank, passes[0], nullptr, hist, perm, inv, st);
        } else {
            kl = ha::launch_sort_pass(lv, rank, passes[0], nullptr, hist, perm_tmp, nullptr, st);
            if (kl > 0) {
                const int k2 = ha::launch_sort_pass(lv, rank, passes[1], perm_tmp, hist, perm, inv, st);
                kl = k2 < 0 ? k2 : kl + k2;
            }
        }
        prof_end(ev, HA_KC_SORT, kl);
        if ((rc = count(kl, "sort"))) return rc;
        if (sort_only) continue;
        float *Op = s.causal ? Opart + static_cast<size_t>(l - 1) * half_rows * s.d : nullptr;
        float *Lp = s.causal ? Lpart + static_cast<size_t>(l - 1) * half_rows : nullptr;
        int k = -2;
        ev = prof_begin(HA_KC_ATTN);
        if (use_tc) family = HA_KERNEL_TC;
        if (use_tc)
            k = ha::launch_attn_tc(lv, Q, K, V, s.d, perm, inv, S, s.m, s.nodes_total, O, out_dtype, lse, Op, Lp,
                                   status, st, stall_ns, Srn, lwrn);
        if (k == -2 && h->opt.kernel != HA_KERNEL_TC) family = HA_KERNEL_SIMT;
        if (k == -2 && h->opt.kernel != HA_KERNEL_TC)
            k = ha::launch_attn_simt(lv, Q, K, V, dtype, s.d, perm, inv, S, s.m, s.nodes_total, O, out_dtype, lse, Op,
                                     Lp, st, Srn, lwrn);
        prof_end(ev, HA_KC_ATTN, k);
        if ((rc = count(k, "attention"))) return rc;
    }
    if (s.causal && !sort_only) {
        int k = -2;
        ev = prof_begin(HA_KC_CAUSAL_BASE);
        if (use_tc && family != HA_KERNEL_SIMT) family = HA_KERNEL_TC;
        // a backward pass needs each row's final log normaliser, which the SIMT kernel writes
        if (use_tc && !h->bwd)
            k = ha::launch_causal_base_tc(Q, K, V, s.bh, s.n, s.d, s.leaf, s.levels, Opart, Lpart, O, out_dtype, status,
                                          st, stall_ns);
        const bool simt_ok = h->opt.kernel != HA_KERNEL_TC || h->bwd;
        if (k == -2 && simt_ok) family = HA_KERNEL_SIMT;
        if (k == -2 && simt_ok)
            k = ha::launch_causal_base_simt(Q, K, V, dtype, s.bh, s.n, s.d, s.leaf, s.levels, Opart, Lpart, O,
                                            out_dtype, st, h->bwd ? lse : nullptr);
        prof_end(ev, HA_KC_CAUSAL_BASE, k);
        if ((rc = count(k, "causal base"))) return rc;
    }
    h->last_launches = launches;
    h->last_kernel = family;
    return HA_OK;
}

int validate_options(hyper_attn_t h, const ha_options *o) {
    if (o->dtype != HA_DTYPE_BF16 && o->dtype != HA_DTYPE_FP32) return fail(h, HA_ERR_INVALID_ARG, "bad dtype");
    if (o->out_dtype != -1 && o->out_dtype != HA_DTYPE_BF16 && o->out_dtype != HA_DTYPE_FP32)
        return fail(h, HA_ERR_INVALID_ARG, "bad out_dtype");
    if (o->batch < 1) return fail(h, HA_ERR_INVALID_ARG, "batch must be >= 1");
    if (o->causal_base < 1) return fail(h, HA_ERR_INVALID_ARG, "causal_base must be >= 1");
    if (o->kernel < HA_KERNEL_AUTO || o->kernel > HA_KERNEL_TC) return fail(h, HA_ERR_INVALID_ARG, "bad kernel");
    if (o->debug_captures != 0 && o->debug_captures != 1) return fail(h, HA_ERR_INVALID_ARG, "bad debug_captures");
    if (o->bh_offset < 0 || o->bh_offset > (int64_t(1) << 40))
        return fail(h, HA_ERR_INVALID_ARG, "bh_offset out of range");
    if (o->test_stall_ms < 0 || o->test_stall_ms > 1000) return fail(h, HA_ERR_INVALID_ARG, "test_stall_ms out of range");
    if (o->sampling != HA_SAMPLING_UNIFORM && o->sampling != HA_SAMPLING_ROWNORM)
        return fail(h, HA_ERR_INVALID_ARG, "bad sampling");
    return HA_OK;
}

int check_ptrs(hyper_attn_t h, const void *Q, const void *K, const void *V, const void *O) {
    if (!Q || !K || !V || !O) return fail(h, HA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(h, HA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (O == Q || O == K || O == V) return fail(h, HA_ERR_INVALID_ARG, "O must not alias Q, K or V");
    return HA_OK;
}

}  // namespace

extern "C" {

void hyper_attn_default_options(ha_options *o) {
    if (!o) return;
    o->dtype = HA_DTYPE_BF16;
    o->out_dtype = -1;
    o->batch = 1;
    o->causal_base = 4096;
    o->stream = nullptr;
    o->kernel = HA_KERNEL_AUTO;
    o->debug_captures = 0;
    o->bh_offset = 0;
    o->test_stall_ms = 0;
    o->sampling = HA_SAMPLING_UNIFORM;
}

int hyper_attn_version(void) { return kVersion; }

int hyper_attn_create(hyper_attn_t *out, int device) {
    if (!out) return HA_ERR_INVALID_ARG;
    *out = nullptr;
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0) {
        cudaGetLastError();
        return HA_ERR_CUDA;
    }
    if (device < 0 || device >= count) return HA_ERR_INVALID_ARG;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return HA_ERR_CUDA;
    if (prop.major != 10) return HA_ERR_UNSUPPORTED;   // built for sm_100a only
    auto *h = new (std::nothrow) hyper_attn_s;
    if (!h) return HA_ERR_OOM;
    h->device = device;
    hyper_attn_default_options(&h->opt);
    DeviceGuard g(device);
    if (cudaEventCreateWithFlags(&h->pin_free, cudaEventDisableTiming) != cudaSuccess) {
        delete h;
        return HA_ERR_CUDA;
    }
    *out = h;
    return HA_OK;
}

int hyper_attn_set_options(hyper_attn_t h, const ha_options *o) {
    if (!h || !o) return HA_ERR_INVALID_ARG;
    int rc = validate_options(h, o);
    if (rc) return rc;
    if (h->opt.stream != o->stream && h->ws) {
        // keep stream order for the workspace: finish work on the old stream first
        DeviceGuard g(h->device);
        HA_CUDA(h, cudaStreamSynchronize(static_cast<cudaStream_t>(h->opt.stream)));
    }
    h->opt = *o;
    return HA_OK;
}

int hyper_attn_forward(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O, int64_t n, int d,
                       int heads, int block, int m, int r, int causal, uint64_t seed) {
    if (!h) return HA_ERR_INVALID_ARG;
    h->err.clear();
    int rc = check_ptrs(h, Q, K, V, O);
    if (rc) return rc;
    if (heads <= 0) return fail(h, HA_ERR_INVALID_ARG, "heads must be positive");
    Shape s{};
    rc = check_shape(h, n, d, h->opt.batch * heads, block, m, r, causal, &s);
    if (rc) return rc;
    DeviceGuard g(h->device);
    return run_forward(h, Q, K, V, O, s, seed, h->opt.bh_offset);
}

int hyper_attn_backward(hyper_attn_t h, const void *Q, const void *K, const void *V, const void *dO, float *dQ,
                        float *dK, float *dV, int64_t n, int d, int heads, int block, int m, int r, int causal,
                        uint64_t seed) {
    if (!h) return HA_ERR_INVALID_ARG;
    h->err.clear();
    if (!Q || !K || !V || !dO || !dQ || !dK || !dV) return fail(h, HA_ERR_INVALID_ARG, "null tensor pointer");
    const void *all[7] = {Q, K, V, dO, dQ, dK, dV};
    for (const void *p : all)
        if (!aligned16(p)) return fail(h, HA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    for (int i = 4; i < 7; ++i)
        for (int j = 0; j < 7; ++j)
            if (i != j && all[i] == all[j]) return fail(h, HA_ERR_INVALID_ARG, "gradients must not alias any tensor");
    if (heads <= 0) return fail(h, HA_ERR_INVALID_ARG, "heads must be positive");
    Shape s{};
    int rc = check_shape(h, n, d, h->opt.batch * heads, block, m, r, causal, &s);
    if (rc) return rc;
    DeviceGuard g(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
    const int dtype = h->opt.dtype;
    const int esz = dtype == HA_DTYPE_BF16 ? 2 : 4;
    const bool rownorm = h->opt.sampling == HA_SAMPLING_ROWNORM && s.m > 0;
    // workspace: the forward's layout (with the captured log normalisers), then O (fp32) and g = dO . O
    hyper_attn_s::Layout lay;
    const size_t fwd = align_up(plan_layout(s, esz, 1, rownorm, &lay));
    const size_t rows = static_cast<size_t>(s.bh) * static_cast<size_t>(s.n);
    const size_t obytes = align_up(sizeof(float) * rows * s.d);
    rc = ensure_workspace(h, fwd + obytes + align_up(sizeof(float) * rows));
    if (rc) return rc;
    float *Of = reinterpret_cast<float *>(h->ws + fwd);
    float *gq = reinterpret_cast<float *>(h->ws + fwd + obytes);
    h->bwd = true;
    rc = run_forward(h, Q, K, V, Of, s, seed, h->opt.bh_offset);
    h->bwd = false;
    if (rc) return rc;
    int launches = h->last_launches;
    auto count = [&](int k, const char *what) -> int {
        if (k < 0) return fail(h, HA_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(cudaGetLastError()));
        launches += k;
        return HA_OK;
    };
    const size_t gbytes = sizeof(float) * rows * s.d;
    HA_CUDA(h, cudaMemsetAsync(dQ, 0, gbytes, st));
    HA_CUDA(h, cudaMemsetAsync(dK, 0, gbytes, st));
    HA_CUDA(h, cudaMemsetAsync(dV, 0, gbytes, st));
    unsigned char *ws = h->ws;
    const float *L = reinterpret_cast<const float *>(ws + h->lay.lse);
    if ((rc = count(ha::launch_bwd_rowdot(dO, dtype, Of, static_cast<int64_t>(rows), s.d, gq, st), "backward dot")))
        return rc;
    const int32_t *S = reinterpret_cast<const int32_t *>(ws + h->lay.S);
    const int32_t *Srn = rownorm ? reinterpret_cast<const int32_t *>(ws + h->lay.rn_S) : nullptr;
    const float *lwrn = rownorm ? reinterpret_cast<const float *>(ws + h->lay.rn_lw) : nullptr;
    for (int i = 0; (!s.causal || s.levels > 0) && i < s.nlev; ++i) {
        const ha::Level lv = make_level(s, s.causal ? i + 1 : 0);
        const int32_t *perm = reinterpret_cast<const int32_t *>(ws + h->lay.perm[i]);
        const int32_t *inv = reinterpret_cast<const int32_t *>(ws + h->lay.inv[i]);
        rc = count(ha::launch_bwd_level(lv, Q, K, V, dO, dtype, s.d, perm, inv, S, s.m, s.nodes_total, Srn, lwrn, L,
                                        gq, dQ, dK, dV, st),
                   "backward level");
        if (rc) return rc;
    }
    if (s.causal &&
        (rc = count(ha::launch_bwd_leaf(Q, K, V, dO, dtype, s.bh, s.n, s.d, s.leaf, L, gq, dQ, dK, dV, st),
                    "backward leaves")))
        return rc;
    h->last_launches = launches;
    return HA_OK;
}

int hyper_attn_diagnostics(hyper_attn_t h, const void *Q, const void *K, int64_t n, int d, int heads, int block,
                           int r, uint64_t seed, int64_t first_col, double *alpha, double *kappa) {
    if (!h) return HA_ERR_INVALID_ARG;
    h->err.clear();
    if (!Q || !K || !alpha || !kappa) return fail(h, HA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(Q) || !aligned16(K)) return fail(h, HA_ERR_INVALID_ARG, "Q and K must be 16-byte aligned");
    if (heads <= 0) return fail(h, HA_ERR_INVALID_ARG, "heads must be positive");
    if (n > kDiagMaxN) return fail(h, HA_ERR_INVALID_ARG, "diagnostics take n <= %d (every entry of A)", kDiagMaxN);
    if (first_col < 0 || first_col >= n) return fail(h, HA_ERR_INVALID_ARG, "first_col must lie in [0, n)");
    Shape s{};
    int rc = check_shape(h, n, d, h->opt.batch * heads, block, 0, r, 0, &s);
    if (rc) return rc;
    DeviceGuard g(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
    const int esz = h->opt.dtype == HA_DTYPE_BF16 ? 2 : 4;
    hyper_attn_s::Layout lay;
    const size_t fwd_bytes = align_up(plan_layout(s, esz, h->opt.debug_captures, false, &lay));
    const size_t diag_scratch = align_up(sizeof(float) * 4 * static_cast<size_t>(s.bh) * n);
    const size_t diag_out = sizeof(double) * 2 * static_cast<size_t>(s.bh);
    rc = ensure_workspace(h, fwd_bytes + diag_scratch + diag_out);   // the forward below reuses it as is
    if (rc) return rc;
    rc = run_forward(h, Q, K, nullptr, nullptr, s, seed, h->opt.bh_offset, true);
    if (rc) return rc;
    float *scratch = reinterpret_cast<float *>(h->ws + fwd_bytes);
    double *out = reinterpret_cast<double *>(h->ws + fwd_bytes + diag_scratch);
    const int32_t *inv = reinterpret_cast<const int32_t *>(h->ws + h->lay.inv[0]);
    const int64_t bp = s.block < n ? s.block : n;
    const int k = ha::launch_diagnostics(Q, K, h->opt.dtype == HA_DTYPE_BF16 ? 0 : 1, s.bh, n, d, inv, bp, first_col,
                                         scratch, out, st);
    if (k < 0) return fail(h, HA_ERR_CUDA, "diagnostics launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    std::vector<double> host(2 * static_cast<size_t>(s.bh));
    HA_CUDA(h, cudaMemcpyAsync(host.data(), out, diag_out, cudaMemcpyDeviceToHost, st));
    HA_CUDA(h, cudaStreamSynchronize(st));
    for (int64_t b = 0; b < s.bh; ++b) {
        alpha[b] = host[2 * b];
        kappa[b] = host[2 * b + 1];
    }
    return HA_OK;
}

int hyper_attn_exact(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O, int64_t n, int d,
                     int heads, int causal) {
    if (!h) return HA_ERR_INVALID_ARG;
    h->err.clear();
    int rc = check_ptrs(h, Q, K, V, O);
    if (rc) return rc;
    if (heads <= 0 || n <= 0) return fail(h, HA_ERR_INVALID_ARG, "heads and n must be positive");
    if (causal != 0 && causal != 1) return fail(h, HA_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (d != 64 && d != 128) return fail(h, HA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (h->opt.dtype != HA_DTYPE_BF16) return fail(h, HA_ERR_UNSUPPORTED, "exact attention needs bf16 inputs");
    if (n % 128 != 0) return fail(h, HA_ERR_UNSUPPORTED, "exact attention needs n to be a multiple of 128");
    DeviceGuard g(h->device);
    rc = ensure_workspace(h, 256);   // the status word (first 256 bytes of every layout)
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
    const int out_dtype = h->opt.out_dtype < 0 ? h->opt.dtype : h->opt.out_dtype;
    const int k = ha::launch_exact_tc(Q, K, V, h->opt.batch * heads, n, d, causal, O, out_dtype,
                                      reinterpret_cast<int *>(h->ws + h->lay.status), st);
    if (k == -2) return fail(h, HA_ERR_UNSUPPORTED, "shape not supported by the exact kernel");
    if (k < 0) return fail(h, HA_ERR_CUDA, "exact attention launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    h->last_launches = k;
    h->last_kernel = HA_KERNEL_TC;
    return HA_OK;
}

int hyper_attn_forward_host(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O, int64_t n, int d,
                            int heads, int block, int m, int r, int causal, uint64_t seed) {
    if (!h) return HA_ERR_INVALID_ARG;
    h->err.clear();
    if (!Q || !K || !V || !O) return fail(h, HA_ERR_INVALID_ARG, "null host pointer");
    if (heads <= 0) return fail(h, HA_ERR_INVALID_ARG, "heads must be positive");
    Shape s{};
    int rc = check_shape(h, n, d, h->opt.batch * heads, block, m, r, causal, &s);
    if (rc) return rc;
    DeviceGuard g(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(h->opt.stream);
    const int out_dtype = h->opt.out_dtype < 0 ? h->opt.dtype : h->opt.out_dtype;
    const size_t in_bytes = static_cast<size_t>(s.bh) * n * d * (h->opt.dtype == HA_DTYPE_BF16 ? 2 : 4);
    const size_t out_bytes = static_cast<size_t>(s.bh) * n * d * (out_dtype == HA_DTYPE_BF16 ? 2 : 4);
    const size_t need = 3 * align_up(in_bytes) + align_up(out_bytes);
    if (need > h->io_bytes) {
        if (h->io) {
            HA_CUDA(h, cudaStreamSynchronize(st));
            HA_CUDA(h, cudaFree(h->io));
            h->io = nullptr;
            h->io_bytes = 0;
        }
        if (device_alloc(h, &h->io, need) != cudaSuccess) {
            cudaGetLastError();
            h->io = nullptr;
            return fail(h, HA_ERR_OOM, "device buffers of %zu bytes failed", need);
        }
        h->io_bytes = need;
    }
    unsigned char *dQ = h->io, *dK = dQ + align_up(in_bytes), *dV = dK + align_up(in_bytes);
    unsigned char *dO = dV + align_up(in_bytes);
    // The problems are independent: they go through in up to kChunks contiguous groups, so that the copy of
    // group i+1 to the device, the forward pass of group i (on the handle's stream) and the copy of group i-1's
    // output back overlap (two copy streams; page-locked host buffers are needed for the overlap). Each group's
    // draws are keyed from its global problem index, so the output equals one pass over all problems. With
    // debug captures on, one group (the captures then describe the whole call).
    constexpr int64_t kChunks = 8;
    const int64_t nchunk = h->opt.debug_captures ? 1 : (s.bh < kChunks ? s.bh : kChunks);
    if (!h->cs_in) {
        HA_CUDA(h, cudaStreamCreateWithFlags(&h->cs_in, cudaStreamNonBlocking));
        HA_CUDA(h, cudaStreamCreateWithFlags(&h->cs_out, cudaStreamNonBlocking));
    }
    while (h->pipe_ev.size() < static_cast<size_t>(2 * kChunks + 1)) {
        cudaEvent_t e;
        HA_CUDA(h, cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        h->pipe_ev.push_back(e);
    }
    cudaEvent_t ev_start = h->pipe_ev[2 * kChunks];
    HA_CUDA(h, cudaEventRecord(ev_start, st));   // earlier work on the handle's stream comes first
    HA_CUDA(h, cudaStreamWaitEvent(h->cs_in, ev_start, 0));
    HA_CUDA(h, cudaStreamWaitEvent(h->cs_out, ev_start, 0));
    const size_t in_row = in_bytes / s.bh, out_row = out_bytes / s.bh;   // bytes per problem
    const unsigned char *hQ = static_cast<const unsigned char *>(Q), *hK = static_cast<const unsigned char *>(K),
                        *hV = static_cast<const unsigned char *>(V);
    unsigned char *hO = static_cast<unsigned char *>(O);
    for (int64_t ci = 0; ci < nchunk; ++ci) {
        const int64_t p0 = s.bh * ci / nchunk, p1 = s.bh * (ci + 1) / nchunk;
        const size_t off = in_row * p0, len = in_row * (p1 - p0);
        HA_CUDA(h, cudaMemcpyAsync(dQ + off, hQ + off, len, cudaMemcpyHostToDevice, h->cs_in));
        HA_CUDA(h, cudaMemcpyAsync(dK + off, hK + off, len, cudaMemcpyHostToDevice, h->cs_in));
        HA_CUDA(h, cudaMemcpyAsync(dV + off, hV + off, len, cudaMemcpyHostToDevice, h->cs_in));
        HA_CUDA(h, cudaEventRecord(h->pipe_ev[ci], h->cs_in));
    }
    for (int64_t ci = 0; ci < nchunk && rc == HA_OK; ++ci) {
        const int64_t p0 = s.bh * ci / nchunk, p1 = s.bh * (ci + 1) / nchunk;
        Shape sc = s;
        sc.bh = p1 - p0;
        HA_CUDA(h, cudaStreamWaitEvent(st, h->pipe_ev[ci], 0));
        rc = run_forward(h, dQ + in_row * p0, dK + in_row * p0, dV + in_row * p0, dO + out_row * p0, sc, seed,
                         h->opt.bh_offset + p0);
        if (rc) break;
        HA_CUDA(h, cudaEventRecord(h->pipe_ev[kChunks + ci], st));
        HA_CUDA(h, cudaStreamWaitEvent(h->cs_out, h->pipe_ev[kChunks + ci], 0));
        HA_CUDA(h, cudaMemcpyAsync(hO + out_row * p0, dO + out_row * p0, out_row * (p1 - p0),
                                   cudaMemcpyDeviceToHost, h->cs_out));
    }
    if (rc) {
        cudaStreamSynchronize(st);
        cudaStreamSynchronize(h->cs_in);
        cudaStreamSynchronize(h->cs_out);
        return rc;
    }
    HA_CUDA(h, cudaStreamSynchronize(h->cs_out));
    HA_CUDA(h, cudaStreamSynchronize(st));
    return HA_OK;
}

int hyper_attn_draw(uint64_t seed, int d, int r, int64_t bh, int64_t n, int m, int causal, int64_t base,
                    float *P_out, int32_t *S_out) {
    Shape s{};
    hyper_attn_s tmp;
    tmp.opt.causal_base = base;
    if (d <= 0 || d > 128) return HA_ERR_INVALID_ARG;
    int rc = check_shape(&tmp, n, d == 64 || d == 128 ? d : 64, bh, 1, m, r, causal, &s);
    if (rc) return rc;
    s.d = d;
    return host_draws(seed, s, 0, P_out, S_out) ? HA_ERR_INVALID_ARG : HA_OK;
}

int hyper_attn_levels(int64_t n, int causal, int64_t base, int *levels_out, int64_t *nodes_out) {
    int L = 0;
    if (causal && causal_levels(n, base, &L)) return HA_ERR_INVALID_ARG;
    if (levels_out) *levels_out = causal ? L : 0;
    if (nodes_out) *nodes_out = causal ? (int64_t(1) << L) - 1 : 1;
    return HA_OK;
}

int hyper_attn_debug_copy(hyper_attn_t h, int what, int level, void *dst, size_t bytes) {
    if (!h || !dst) return HA_ERR_INVALID_ARG;
    if (!h->have_last || !h->ws) return fail(h, HA_ERR_INVALID_ARG, "no forward call yet");
    DeviceGuard g(h->device);
    const auto &L = h->lay;
    size_t off = 0, avail = 0;
    switch (what) {
        case HA_DBG_RANK: off = L.rank; avail = L.rank_bytes; break;
        case HA_DBG_NEAR: off = L.near; avail = L.near_bytes; break;
        case HA_DBG_LSE: off = L.lse; avail = L.lse_bytes; break;
        case HA_DBG_RN_S: off = L.rn_S; avail = L.rn_bytes; break;
        case HA_DBG_RN_LOGW: off = L.rn_lw; avail = L.rn_bytes; break;
        case HA_DBG_PERM:
        case HA_DBG_INV: {
            const int idx = h->dk_causal ? level - 1 : level;
            if (idx < 0 || idx >= static_cast<int>(L.perm.size())) return fail(h, HA_ERR_INVALID_ARG, "bad level");
            off = what == HA_DBG_PERM ? L.perm[idx] : L.inv[idx];
            avail = L.perm_bytes[idx];
            break;
        }
        default: return fail(h, HA_ERR_INVALID_ARG, "bad capture id");
    }
    if (bytes > avail) return fail(h, HA_ERR_INVALID_ARG, "capture holds %zu bytes, %zu requested", avail, bytes);
    HA_CUDA(h, cudaStreamSynchronize(static_cast<cudaStream_t>(h->opt.stream)));
    HA_CUDA(h, cudaMemcpy(dst, h->ws + off, bytes, cudaMemcpyDeviceToHost));
    return HA_OK;
}

int hyper_attn_status(hyper_attn_t h) {
    if (!h) return HA_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    HA_CUDA(h, cudaStreamSynchronize(static_cast<cudaStream_t>(h->opt.stream)));
    if (!h->ws) return HA_OK;
    int word = 0;
    HA_CUDA(h, cudaMemcpy(&word, h->ws + h->lay.status, sizeof word, cudaMemcpyDeviceToHost));
    if (word) {
        HA_CUDA(h, cudaMemset(h->ws + h->lay.status, 0, sizeof word));
        if (word & ha::kStatusTimeout) return fail(h, HA_ERR_TIMEOUT, "a device-side wait gave up (status %d)", word);
        if (word & ha::kStatusBounds)
            return fail(h, HA_ERR_CUDA, "a row index read from a permutation or a sample list was out of range, "
                                        "HA_DEBUG build (status %d)", word);
        return fail(h, HA_ERR_CUDA, "device status word %d", word);
    }
    return HA_OK;
}

int hyper_attn_profile(hyper_attn_t h, int enable) {
    if (!h || (enable != 0 && enable != 1)) return HA_ERR_INVALID_ARG;
    h->profiling = enable == 1;
    return HA_OK;
}

int hyper_attn_profile_read(hyper_attn_t h, double *ms, int *launches, int n) {
    if (!h || n < 0) return HA_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    HA_CUDA(h, cudaStreamSynchronize(static_cast<cudaStream_t>(h->opt.stream)));
    for (int i = 0; i < n; ++i) {
        if (ms) ms[i] = 0.0;
        if (launches) launches[i] = 0;
    }
    for (const auto &r : h->recs) {
        float t = 0.0f;
        HA_CUDA(h, cudaEventElapsedTime(&t, h->ev_pool[r.e0], h->ev_pool[r.e1]));
        if (r.cls < n) {
            if (ms) ms[r.cls] += t;
            if (launches) launches[r.cls] += r.launches;
        }
    }
    h->recs.clear();
    h->ev_used = 0;
    return HA_OK;
}

int hyper_attn_last_kernel(hyper_attn_t h) { return h ? h->last_kernel : 0; }

int hyper_attn_last_launch_count(hyper_attn_t h) { return h ? h->last_launches : 0; }

const char *hyper_attn_last_error(hyper_attn_t h) { return h ? h->err.c_str() : "null handle"; }

int hyper_attn_test_fail_alloc(hyper_attn_t h, int count) {
    if (!h || count < 0) return HA_ERR_INVALID_ARG;
    h->fail_alloc = count;
    return HA_OK;
}

int hyper_attn_destroy(hyper_attn_t h) {
    if (!h) return HA_OK;
    {
        DeviceGuard g(h->device);
        cudaStreamSynchronize(static_cast<cudaStream_t>(h->opt.stream));
        if (h->ws) cudaFree(h->ws);
        if (h->io) cudaFree(h->io);
        if (h->pin_free) cudaEventSynchronize(h->pin_free);
        if (h->pin) cudaFreeHost(h->pin);
        if (h->pin_free) cudaEventDestroy(h->pin_free);
        for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
        if (h->cs_in) cudaStreamSynchronize(h->cs_in);
        if (h->cs_out) cudaStreamSynchronize(h->cs_out);
        for (cudaEvent_t e : h->pipe_ev) cudaEventDestroy(e);
        if (h->cs_in) cudaStreamDestroy(h->cs_in);
        if (h->cs_out) cudaStreamDestroy(h->cs_out);
    }
    delete h;
    return HA_OK;
}

}  // extern "C"
