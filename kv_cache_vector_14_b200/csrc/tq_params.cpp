// Host-side constants of the method: sign diagonal D, JL matrix S, codebook.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装", K-Cache section: step 2 rotates with a fast Walsh-Hadamard
// transform (here preceded by a fixed random sign diagonal D), step 3 uses a
// 3-bit Lloyd-Max codebook, step 5 a Johnson-Lindenstrauss matrix (here iid
// N(0,1), m = d rows).  The random draws come from one counter-based
// SplitMix64 stream (Steele, Lea & Flood 2014), written here from its
// published definition; Gaussians by the Box-Muller transform.
#include <cmath>
#include <cstring>

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

// SplitMix64 output number i of the stream whose state starts at `seed`.
inline uint64_t splitmix_draw(uint64_t seed, uint64_t i) {
    uint64_t x = seed + kGamma * (i + 1);
    x ^= x >> 30;
    x *= 0xBF58476D1CE4E5B9ull;
    x ^= x >> 27;
    x *= 0x94D049BB133111EBull;
    x ^= x >> 31;
    return x;
}

// Conditional mean of N(0,1) on (lo, hi), hi may be +inf.
double gauss_cell_mean(double lo, double hi) {
    const double inv_sqrt2pi = 0.3989422804014327;
    double dens_lo = inv_sqrt2pi * std::exp(-0.5 * lo * lo);
    double dens_hi = std::isinf(hi) ? 0.0 : inv_sqrt2pi * std::exp(-0.5 * hi * hi);
    double mass = 0.5 * (std::erfc(lo / std::sqrt(2.0)) - (std::isinf(hi) ? 0.0 : std::erfc(hi / std::sqrt(2.0))));
    return (dens_lo - dens_hi) / mass;
}

// Positive half of the symmetric 8-level Lloyd-Max quantiser of N(0,1):
// levels a0 < a1 < a2 < a3 on [0, inf), cells [0, e1], [e1, e2], [e2, e3],
// [e3, inf) with e_k the midpoints; iterate the two Lloyd conditions.
void lloyd_positive_half(double a[4]) {
    a[0] = 0.25; a[1] = 0.75; a[2] = 1.25; a[3] = 1.75;
    for (int iter = 0; iter < 1000000; ++iter) {
        double e1 = 0.5 * (a[0] + a[1]), e2 = 0.5 * (a[1] + a[2]), e3 = 0.5 * (a[2] + a[3]);
        double n0 = gauss_cell_mean(0.0, e1), n1 = gauss_cell_mean(e1, e2);
        double n2 = gauss_cell_mean(e2, e3), n3 = gauss_cell_mean(e3, INFINITY);
        double delta = std::fmax(std::fmax(std::fabs(n0 - a[0]), std::fabs(n1 - a[1])),
                                 std::fmax(std::fabs(n2 - a[2]), std::fabs(n3 - a[3])));
        a[0] = n0; a[1] = n1; a[2] = n2; a[3] = n3;
        if (delta < 1e-13) break;
    }
}

}  // namespace

// IEEE binary16 bits of a double, round to nearest even, from the double's bits.
uint16_t double_to_half_bits(double x) {
    uint64_t u;
    std::memcpy(&u, &x, 8);
    const uint16_t sgn = (uint16_t)((u >> 48) & 0x8000u);
    const uint64_t mag = u & 0x7FFFFFFFFFFFFFFFull;
    if (mag >= 0x7FF0000000000000ull) return sgn | (mag > 0x7FF0000000000000ull ? 0x7E00 : 0x7C00);
    const int bexp = (int)(mag >> 52);
    if (bexp == 0) return sgn;                       // double subnormal: far below half range
    const int e = bexp - 1023;
    if (e > 15) return sgn | 0x7C00;
    const uint64_t sig = (mag & ((1ull << 52) - 1)) | (1ull << 52);
    const int drop = (e >= -14) ? 42 : 42 + (-14 - e);  // bits removed from the 53-bit significand
    if (drop > 62) return sgn;
    uint64_t q = sig >> drop;
    const uint64_t rem = sig & ((1ull << drop) - 1), halfway = 1ull << (drop - 1);
    if (rem > halfway || (rem == halfway && (q & 1))) ++q;
    if (e >= -14) {
        int ee = e;
        if (q == 2048) { q = 1024; ++ee; }
        if (ee > 15) return sgn | 0x7C00;
        return (uint16_t)(sgn | ((ee + 15) << 10) | (q - 1024));
    }
    return (uint16_t)(sgn | q);                      // q == 1024 is the smallest normal
}

double half_bits_to_double(uint16_t h) {
    int e = (h >> 10) & 31, f = h & 1023;
    double v = (e == 0) ? std::ldexp((double)f, -24) : std::ldexp((double)(1024 + f), e - 25);
    return (h & 0x8000) ? -v : v;
}

bool make_params(int d, uint64_t seed, int8_t* D, float* S, float* c8, float* b7) {
    if (!head_dim_ok(d)) return false;
    if (D)
        for (int j = 0; j < d; ++j) D[j] = (splitmix_draw(seed, (uint64_t)j) & (1ull << 63)) ? -1 : 1;
    if (S) {
        const uint64_t pairs = (uint64_t)d * (uint64_t)d / 2;  // m = d rows
        const double two_pow_m53 = 1.0 / 9007199254740992.0;
        for (uint64_t p = 0; p < pairs; ++p) {
            const uint64_t a = splitmix_draw(seed, (uint64_t)d + 2 * p);
            const uint64_t b = splitmix_draw(seed, (uint64_t)d + 2 * p + 1);
            const double u1 = (double)((a >> 11) + 1) * two_pow_m53;   // (0, 1]
            const double u2 = (double)(b >> 11) * two_pow_m53;         // [0, 1)
            const double radius = std::sqrt(-2.0 * std::log(u1));
            const double theta = 2.0 * M_PI * u2;
            S[2 * p] = (float)(radius * std::cos(theta));
            S[2 * p + 1] = (float)(radius * std::sin(theta));
        }
    }
    double a[4];
    lloyd_positive_half(a);
    double cent[8];
    for (int k = 0; k < 4; ++k) {
        const double v = half_bits_to_double(double_to_half_bits(a[k] / std::sqrt((double)d)));
        cent[4 + k] = v;
        cent[3 - k] = -v;
    }
    if (c8)
        for (int k = 0; k < 8; ++k) c8[k] = (float)cent[k];
    if (b7)
        for (int k = 0; k < 7; ++k) b7[k] = (float)(0.5 * (cent[k] + cent[k + 1]));
    return true;
}

}  // namespace tqi
