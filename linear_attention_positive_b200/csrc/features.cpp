// Host-side draw of the block-orthogonal random feature matrix W (favor_draw_features).
//
// Positive orthogonal random features ("Rethinking Attention with Performers", abstract; the
// summary page's limitations: orthogonality within blocks of at most d rows). The generator is
// Philox4x64-10 (Salmon et al., SC'11), the Gaussians come from Box-Muller, the blocks are
// orthonormalised by modified Gram-Schmidt with one re-orthogonalisation pass and the rows get
// independent chi(d) norms. Every floating-point step is a single IEEE double operation in a
// fixed order: this file is compiled without FMA contraction or fast-math, so the result does
// not depend on the compiler's scheduling.

#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/favor.h"

namespace {

constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull;
constexpr uint64_t kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kPhiloxW1 = 0xBB67AE8584CAA73Bull;

struct Block4 {
    uint64_t v[4];
};

// Philox4x64 with 10 rounds: per round, 64x64->128 products of counter words 0 and 2 with the
// two multipliers, then the word permutation (hi1^c1^k0, lo1, hi0^c3^k1, lo0) and a Weyl bump
// of the key.
Block4 philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3, uint64_t k0, uint64_t k1) {
    for (int r = 0; r < 10; ++r) {
        const unsigned __int128 p0 = (unsigned __int128)kPhiloxM0 * c0;
        const unsigned __int128 p1 = (unsigned __int128)kPhiloxM1 * c2;
        const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        const uint64_t n0 = hi1 ^ c1 ^ k0;
        const uint64_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
        k0 += kPhiloxW0;
        k1 += kPhiloxW1;
    }
    return Block4{{c0, c1, c2, c3}};
}

// Top 53 bits plus half an ulp: a double strictly inside (0, 1).
double uniform_open01(uint64_t x) { return ((double)(x >> 11) + 0.5) * 0x1.0p-53; }

// Gaussians 0..count-1 of the stream (seed, block, purpose): counter (n/4, block, purpose, 0);
// outputs (x0, x1) give Gaussians 4k, 4k+1 and (x2, x3) give 4k+2, 4k+3.
void gaussians(uint64_t seed, uint64_t block, uint64_t purpose, size_t count, double *out) {
    const double two_pi = 2.0 * M_PI;
    const size_t calls = (count + 3) / 4;
    for (size_t k = 0; k < calls; ++k) {
        const Block4 x = philox4x64_10((uint64_t)k, block, purpose, 0, seed, 0);
        for (int pair = 0; pair < 2; ++pair) {
            const double ua = uniform_open01(x.v[2 * pair]);
            const double ub = uniform_open01(x.v[2 * pair + 1]);
            const double r = std::sqrt(-2.0 * std::log(ua));
            const double theta = two_pi * ub;
            const double g[2] = {r * std::cos(theta), r * std::sin(theta)};
            for (int j = 0; j < 2; ++j) {
                const size_t idx = 4 * k + 2 * pair + j;
                if (idx < count) out[idx] = g[j];
            }
        }
    }
}

// Left-to-right sum of products: s = 0; s = s + a[k]*b[k].
double seq_dot(const double *a, const double *b, int n) {
    double s = 0.0;
    for (int k = 0; k < n; ++k) {
        const double p = a[k] * b[k];
        s = s + p;
    }
    return s;
}

}  // namespace

extern "C" favor_status favor_draw_features(uint64_t seed, int m, int d, double *W_host) {
    if (W_host == nullptr || m <= 0 || d <= 0 || d > 1024) return FAVOR_ERR_INVALID_ARG;
    const int n_blocks = (m + d - 1) / d;
    std::vector<double> G((size_t)d * d), U((size_t)d * d), C((size_t)d * d), v(d);
    int row_out = 0;
    for (int b = 0; b < n_blocks; ++b) {
        gaussians(seed, (uint64_t)b, 0, (size_t)d * d, G.data());
        // Modified Gram-Schmidt over the rows, twice per row.
        for (int i = 0; i < d; ++i) {
            for (int k = 0; k < d; ++k) v[k] = G[(size_t)i * d + k];
            for (int pass = 0; pass < 2; ++pass) {
                for (int j = 0; j < i; ++j) {
                    const double *u = &U[(size_t)j * d];
                    const double p = seq_dot(u, v.data(), d);
                    for (int k = 0; k < d; ++k) {
                        const double t = p * u[k];
                        v[k] = v[k] - t;
                    }
                }
            }
            const double nrm = std::sqrt(seq_dot(v.data(), v.data(), d));
            for (int k = 0; k < d; ++k) U[(size_t)i * d + k] = v[k] / nrm;
        }
        // Independent chi(d) row norms.
        gaussians(seed, (uint64_t)b, 1, (size_t)d * d, C.data());
        for (int i = 0; i < d && row_out < m; ++i, ++row_out) {
            const double *c = &C[(size_t)i * d];
            const double n = std::sqrt(seq_dot(c, c, d));
            for (int k = 0; k < d; ++k) W_host[(size_t)row_out * d + k] = n * U[(size_t)i * d + k];
        }
    }
    return FAVOR_OK;
}
