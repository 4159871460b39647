// ha_noalloc.cu -- a non-causal forward entry point that allocates nothing.
//
// Some callers cannot call cudaMalloc: a plugin running inside an engine that reserves all device memory
// up front and forbids allocation while it enqueues work, or a latency-critical loop that cannot afford
// the device-wide synchronisation an allocation may cause. hyper_attn_forward_noalloc serves them: the
// caller passes Q, K, V and O, and every scratch buffer of the pass (draws, ranks, flags, permutations,
// sort histograms) lives in one file-scope __device__ array of kNoAllocScratchBytes that each GPU loading
// this library holds until the process exits. Calls share that array, so calls that overlap on the GPU (on
// different streams, or from different host threads on different streams) race; callers must order them.
// Host-side draws use file-scope host arrays under a mutex, so concurrent host calls are serialised. The
// draws reach the device through copies from those pageable host arrays, which only hold outside stream
// capture (a captured copy would read the arrays when the graph is replayed, after later calls changed
// them), so a call made while its stream is capturing is refused. No kernel on this path waits on anything
// on the device, so the path has no status word to report.
#include <mutex>

#include "../../include/hyper_attn.h"
#include "ha_internal.h"

namespace {

constexpr int64_t kMaxRows = 65536;     // batch*heads*n
constexpr int64_t kMaxProblems = 64;    // batch*heads
constexpr int kMaxM = 512;
constexpr int kMaxRBits = ha::kMaxPassBits;   // one counting-sort pass
constexpr int kMaxDevices = 64;

constexpr size_t al(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kPOff = 0;
constexpr size_t kSOff = kPOff + al(sizeof(float) * ha::kMaxR * 128);
constexpr size_t kRankOff = kSOff + al(sizeof(int32_t) * kMaxProblems * kMaxM);
constexpr size_t kNearOff = kRankOff + al(sizeof(uint16_t) * 2 * kMaxRows);
constexpr size_t kPermOff = kNearOff + al(2 * kMaxRows);
constexpr size_t kInvOff = kPermOff + al(sizeof(int32_t) * 2 * kMaxRows);
constexpr size_t kHistOff = kInvOff + al(sizeof(int32_t) * 2 * kMaxRows);
// segments x chunks <= 2 * (rows / chunk + problems)
constexpr size_t kHistBytes =
    sizeof(int32_t) * 2 * (kMaxRows / ha::kSortChunk + kMaxProblems) * (size_t(1) << kMaxRBits);
constexpr size_t kNoAllocScratchBytes = kHistOff + al(kHistBytes);
static_assert(kNoAllocScratchBytes <= (size_t(5) << 19), "scratch stays within 2.5 MiB");

static __device__ __align__(256) unsigned char g_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void *g_scratch_dev[kMaxDevices] = {};                  // device address of g_scratch, per device
float g_P[ha::kMaxR * 128];
int32_t g_S[kMaxProblems * kMaxM];
uint8_t g_floyd[kMaxRows];                               // zero on entry and exit of draw_samples

}  // namespace

extern "C" int hyper_attn_forward_noalloc(const void *Q, const void *K, const void *V, void *O, int64_t n, int d,
                                          int heads, int block, int m, int r, uint64_t seed, int dtype,
                                          void *stream) {
    if (!Q || !K || !V || !O) return HA_ERR_INVALID_ARG;
    // the hash and attention kernels read rows with 16-byte copies
    for (const void *p : {static_cast<const void *>(Q), K, V, static_cast<const void *>(O)})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return HA_ERR_INVALID_ARG;
    if (O == Q || O == K || O == V) return HA_ERR_INVALID_ARG;
    if (dtype != HA_DTYPE_BF16 && dtype != HA_DTYPE_FP32) return HA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return HA_ERR_UNSUPPORTED;
    if (heads <= 0 || heads > kMaxProblems || n <= 0 || n * heads > kMaxRows) return HA_ERR_INVALID_ARG;
    if (block <= 0 || m < 0 || m > kMaxM || m > n || r < 0 || r > kMaxRBits) return HA_ERR_INVALID_ARG;
    const int64_t bp = block < n ? block : n;
    if (n % bp) return HA_ERR_INVALID_ARG;

    std::lock_guard<std::mutex> lock(g_mutex);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HA_ERR_CUDA;
    if (!g_scratch_dev[dev]) {
        // first call on this device: resolve the array's device address with the device current
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return HA_ERR_CUDA;
        }
        g_scratch_dev[dev] = p;
    }
    unsigned char *base = static_cast<unsigned char *>(g_scratch_dev[dev]);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
        cudaGetLastError();
        return HA_ERR_CUDA;
    }
    if (cap != cudaStreamCaptureStatusNone) return HA_ERR_UNSUPPORTED;

    // host draws (same definitions as every other entry point)
    ha::draw_projection(seed, d, r, g_P);
    for (int h = 0; h < heads; ++h)
        if (ha::draw_samples(seed, static_cast<uint64_t>(h), 1, n, m, g_S + static_cast<int64_t>(h) * m, g_floyd))
            return HA_ERR_INVALID_ARG;
    // pageable-host copies return once the source has been staged, so the host arrays are free again
    if (cudaMemcpyAsync(base + kPOff, g_P, sizeof(float) * d * (r ? r : 1), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        (m > 0 && cudaMemcpyAsync(base + kSOff, g_S, sizeof(int32_t) * heads * m, cudaMemcpyHostToDevice, st) !=
                      cudaSuccess)) {
        cudaGetLastError();
        return HA_ERR_CUDA;
    }

    ha::Level lv{};
    lv.n = n; lv.bh = heads; lv.level = 0; lv.nodes = 1; lv.node_len = n; lv.seg_len = n; lv.q_off = 0;
    lv.heap0 = 1; lv.bp = static_cast<int>(bp);
    const int32_t *S = reinterpret_cast<const int32_t *>(base + kSOff);
    uint16_t *rank = reinterpret_cast<uint16_t *>(base + kRankOff);
    uint8_t *near = base + kNearOff;
    int32_t *perm = reinterpret_cast<int32_t *>(base + kPermOff);
    int32_t *inv = reinterpret_cast<int32_t *>(base + kInvOff);
    int32_t *hist = reinterpret_cast<int32_t *>(base + kHistOff);

    // a failed launch leaves its error behind: take it, so that the caller's next check starts clean
    const ha::SortPass pass{0, 1 << r};
    if (ha::launch_hash(Q, K, dtype, heads, n, d, g_P, r, rank, near, st) < 0 ||
        ha::launch_sort_pass(lv, rank, pass, nullptr, hist, perm, inv, st) < 0 ||
        ha::launch_attn_simt(lv, Q, K, V, dtype, d, perm, inv, S, m, 1, O, dtype, nullptr, nullptr, nullptr, st) < 0) {
        cudaGetLastError();
        return HA_ERR_CUDA;
    }
    return HA_OK;
}
