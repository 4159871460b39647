// ha_draws.cpp -- host-side random draws of the forward pass: the Gaussian projection matrix of sortLSH
// and the uniform column samples of the normaliser estimate ("HyperAttention: Long-context Attention in
// Near-Linear Time", research-map summary, "Approach").
//
// Generator: Philox4x64 with 10 rounds (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11). Key word 0 is the seed, key word 1 a stream tag (1: projection, 2: samples).
//   projection entry e = k*r + j (P is [d][r]): counter (e, 0, 0, 0); output words 0 and 1 give
//     u1 = (w0 >> 11 + 1) * 2^-53 in (0,1], u2 = (w1 >> 11) * 2^-53 in [0,1); the entry is the cosine
//     branch of Box-Muller, sqrt(-2 ln u1) cos(2 pi u2), evaluated in double and rounded to float.
//   samples of problem (bh, node): word t of the stream is output word t mod 4 of counter
//     (t / 4, node, bh, 0); bounded integers by Lemire's multiply-shift with rejection; the m-subset of
//     [0, N) by Floyd's algorithm; returned in ascending order.
#include <cmath>
#include <cstring>

#include "ha_internal.h"

namespace ha {
namespace {

struct Philox4x64 {
    static constexpr uint64_t kMulA = 0xD2E7470EE14C6C93ULL;
    static constexpr uint64_t kMulB = 0xCA5A826395121157ULL;
    static constexpr uint64_t kBumpA = 0x9E3779B97F4A7C15ULL;
    static constexpr uint64_t kBumpB = 0xBB67AE8584CAA73BULL;

    static void mulhilo(uint64_t a, uint64_t b, uint64_t &hi, uint64_t &lo) {
        const unsigned __int128 p = static_cast<unsigned __int128>(a) * b;
        hi = static_cast<uint64_t>(p >> 64);
        lo = static_cast<uint64_t>(p);
    }

    // 10 rounds; the key is bumped by the Weyl constants before every round after the first.
    static void block(const uint64_t in[4], uint64_t k0, uint64_t k1, uint64_t out[4]) {
        uint64_t c[4] = {in[0], in[1], in[2], in[3]};
        for (int i = 0; i < 10; ++i) {
            if (i) { k0 += kBumpA; k1 += kBumpB; }
            uint64_t hA, lA, hB, lB;
            mulhilo(kMulA, c[0], hA, lA);
            mulhilo(kMulB, c[2], hB, lB);
            const uint64_t n0 = hB ^ c[1] ^ k0, n2 = hA ^ c[3] ^ k1;
            c[0] = n0; c[1] = lB; c[2] = n2; c[3] = lA;
        }
        std::memcpy(out, c, sizeof c);
    }
};

constexpr uint64_t kTagProjection = 1;
constexpr uint64_t kTagSamples = 2;

class SampleStream {
  public:
    SampleStream(uint64_t seed, uint64_t bh, uint64_t node) : seed_(seed), bh_(bh), node_(node) {}
    uint64_t next() {
        const uint64_t slot = t_ & 3u;
        if (slot == 0) {
            const uint64_t ctr[4] = {t_ >> 2, node_, bh_, 0};
            Philox4x64::block(ctr, seed_, kTagSamples, buf_);
        }
        ++t_;
        return buf_[slot];
    }
    // uniform in [0, range), range >= 1 (Lemire 2019)
    uint64_t below(uint64_t range) {
        unsigned __int128 prod = static_cast<unsigned __int128>(next()) * range;
        uint64_t low = static_cast<uint64_t>(prod);
        if (low < range) {
            const uint64_t reject_below = (0 - range) % range;
            while (low < reject_below) {
                prod = static_cast<unsigned __int128>(next()) * range;
                low = static_cast<uint64_t>(prod);
            }
        }
        return static_cast<uint64_t>(prod >> 64);
    }

  private:
    uint64_t seed_, bh_, node_;
    uint64_t t_ = 0;
    uint64_t buf_[4] = {0, 0, 0, 0};
};

}  // namespace

void draw_projection(uint64_t seed, int d, int r, float *P) {
    const double kTwoPi = 6.283185307179586476925286766559;
    const double kScale53 = 1.0 / 9007199254740992.0;
    const int64_t total = static_cast<int64_t>(d) * r;
    for (int64_t e = 0; e < total; ++e) {
        const uint64_t ctr[4] = {static_cast<uint64_t>(e), 0, 0, 0};
        uint64_t w[4];
        Philox4x64::block(ctr, seed, kTagProjection, w);
        const double u1 = static_cast<double>((w[0] >> 11) + 1) * kScale53;
        const double u2 = static_cast<double>(w[1] >> 11) * kScale53;
        P[e] = static_cast<float>(std::sqrt(-2.0 * std::log(u1)) * std::cos(kTwoPi * u2));
    }
}

// scratch: N bytes, zeroed on entry and left zeroed on return.
int draw_samples(uint64_t seed, uint64_t bh, uint64_t node, int64_t N, int m, int32_t *S, uint8_t *scratch) {
    if (m < 0 || m > N) return -1;
    SampleStream rng(seed, bh, node);
    for (int64_t top = N - m; top < N; ++top) {
        const int64_t pick = static_cast<int64_t>(rng.below(static_cast<uint64_t>(top) + 1));
        scratch[scratch[pick] ? top : pick] = 1;
    }
    int64_t out = 0;
    for (int64_t i = 0; i < N && out < m; ++i)
        if (scratch[i]) { S[out++] = static_cast<int32_t>(i); }
    // clear only what was set
    for (int u = 0; u < m; ++u) scratch[S[u]] = 0;
    return out == m ? 0 : -1;
}

}  // namespace ha
