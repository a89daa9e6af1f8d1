/*
 * tq_oracle.c -- plain, slow, float64 CPU oracle for TurboQuant KV-cache
 * compression and compressed-cache decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library: every step below is written out again from
 * the method's description.
 *
 * Sources (pages on the subject):
 *   [P4] "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
 *        Streamingを実装" (ai-heartland.com), section "K-Cache圧縮：3-bit
 *        PolarQuant + 1-bit QJL = 4.25 bits/dim" (the five-step K flow) and
 *        section "V-Cache圧縮：3-bit PolarQuant = 3.125 bits/dim".
 *   [P1] techfi24.com article, section "Contexte Technique" (polar
 *        quantisation plus QJL residual correction).
 * Readings where the pages are silent are stated beside each function (the
 * random-sign rotation, the Gaussian JL matrix with m = d rows, the
 * sqrt(pi/2)/m estimator constant, fp16 norms, fp16 centroids).
 *
 * Parity status: every function below is pinned by a CPU test against a
 * closed form, a textbook table, a library routine or brute force.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BLOCK_T 64

/* ------------------------------------------------------------------------
 * Counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; the public splitmix64.c
 * finaliser).  Output number i of stream `seed` is the finaliser applied to
 * seed + (i + 1) * golden-gamma, so any element can be drawn directly.
 * ---------------------------------------------------------------------- */
static uint64_t orc_splitmix64_at(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t orc_rng(uint64_t seed, uint64_t i) { return orc_splitmix64_at(seed, i); }

/* ------------------------------------------------------------------------
 * IEEE binary16 round-to-nearest-even from a double, and back.  Used for the
 * stored norms (n, gamma) and for the centroids.
 * ---------------------------------------------------------------------- */
uint16_t orc_to_fp16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(x)) return (uint16_t)(sign | 0x7C00u);
    if (a < ldexp(1.0, -14)) {                 /* subnormal range: units of 2^-24 */
        double r = nearbyint(ldexp(a, 24));    /* exact scaling, RNE */
        return (uint16_t)(sign | (uint16_t)r); /* r == 1024 gives the smallest normal */
    }
    int e2;
    frexp(a, &e2);                             /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                            /* a in [2^e, 2^(e+1)) */
    double r = nearbyint(ldexp(a, 10 - e));    /* significand in [1024, 2048] */
    if (r >= 2048.0) { r = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(r - 1024.0));
}

double orc_from_fp16(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp(1024.0 + f, e - 25);
    return s ? -v : v;
}

/* ------------------------------------------------------------------------
 * Lloyd-Max quantiser for the standard normal [P4, K-Cache section, step 3: the
 * 3-bit non-linear Lloyd-Max codebook; the hybrid V2+V3 section: the codebook
 * taken from V3].  Lloyd's two optimality
 * conditions are applied alternately: decision edges at midpoints of adjacent
 * levels; each level at the conditional mean of N(0,1) on its cell,
 * (phi(a) - phi(b)) / (Phi(b) - Phi(a)).  Iterates until the largest level
 * change is below 1e-12.
 * ---------------------------------------------------------------------- */
static double orc_phi(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }
/* P(a < Z < b) written with erfc so that tail cells keep full precision */
static double orc_cell_mass(double a, double b) {
    return 0.5 * (erfc(a / sqrt(2.0)) - erfc(b / sqrt(2.0)));
}

int orc_lloyd_max_std(int levels, double* c) {
    for (int k = 0; k < levels; ++k) c[k] = -1.75 + 3.5 * k / (levels - 1);
    int it;
    for (it = 0; it < 1000000; ++it) {
        double edge[65];
        edge[0] = -INFINITY;
        edge[levels] = INFINITY;
        for (int k = 1; k < levels; ++k) edge[k] = 0.5 * (c[k - 1] + c[k]);
        double maxd = 0.0;
        for (int k = 0; k < levels; ++k) {
            double pa = isinf(edge[k]) ? 0.0 : orc_phi(edge[k]);
            double pb = isinf(edge[k + 1]) ? 0.0 : orc_phi(edge[k + 1]);
            double nc = (pa - pb) / orc_cell_mass(edge[k], edge[k + 1]);
            double dlt = fabs(nc - c[k]);
            if (dlt > maxd) maxd = dlt;
            c[k] = nc;
        }
        if (maxd < 1e-12) break;
    }
    return it + 1;
}

/* ------------------------------------------------------------------------
 * The method's constants for head dimension d and seed [P4, K flow steps 2,
 * 3 and 5].  Readings:
 *  - rotation sign diagonal D: D_j = -1 if the top bit of draw j is set;
 *  - JL matrix S (m x d, m = d, row-major), iid N(0,1): Box-Muller on draws
 *    d + 2p (u1 = ((x >> 11) + 1) * 2^-53, in (0,1]) and d + 2p + 1
 *    (u2 = (x >> 11) * 2^-53), radius sqrt(-2 ln u1), angle 2*pi*u2; element
 *    2p takes the cosine output and element 2p + 1 the sine output; each
 *    rounded to fp32;
 *  - codebook: the 8 standard-normal Lloyd-Max levels, made exactly
 *    antisymmetric, scaled by 1/sqrt(d) (a rotated unit vector has
 *    N(0, 1/d) coordinates) and rounded to fp16;
 *  - boundaries: midpoints of adjacent rounded levels (exact).
 * ---------------------------------------------------------------------- */
void orc_params(int d, uint64_t seed, int8_t* D, double* S, double* c8, double* b7) {
    for (int j = 0; j < d; ++j) D[j] = (orc_splitmix64_at(seed, (uint64_t)j) >> 63) ? -1 : 1;
    const int m = d;
    const uint64_t npair = (uint64_t)m * (uint64_t)d / 2;
    for (uint64_t p = 0; p < npair; ++p) {
        uint64_t x1 = orc_splitmix64_at(seed, (uint64_t)d + 2 * p);
        uint64_t x2 = orc_splitmix64_at(seed, (uint64_t)d + 2 * p + 1);
        double u1 = ((double)(x1 >> 11) + 1.0) * ldexp(1.0, -53);
        double u2 = (double)(x2 >> 11) * ldexp(1.0, -53);
        double rad = sqrt(-2.0 * log(u1));
        double ang = 2.0 * M_PI * u2;
        S[2 * p] = (double)(float)(rad * cos(ang));
        S[2 * p + 1] = (double)(float)(rad * sin(ang));
    }
    double lv[8];
    orc_lloyd_max_std(8, lv);
    for (int k = 0; k < 4; ++k) {           /* exact antisymmetry */
        double a = 0.5 * (lv[7 - k] - lv[k]);
        lv[k] = -a;
        lv[7 - k] = a;
    }
    for (int k = 0; k < 8; ++k) c8[k] = orc_from_fp16(orc_to_fp16(lv[k] / sqrt((double)d)));
    for (int k = 0; k < 7; ++k) b7[k] = 0.5 * (c8[k] + c8[k + 1]);
}

/* ------------------------------------------------------------------------
 * Orthonormal Walsh-Hadamard transform in natural (Sylvester) order,
 * (H v)_i = sum_j (-1)^popcount(i & j) v_j / sqrt(d), by the textbook
 * in-place butterfly [P4, K flow step 2, "Fast Walsh-Hadamard Transform"].
 * ---------------------------------------------------------------------- */
void orc_fwht(double* v, int d) {
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) v[i] *= s;
}

/* ------------------------------------------------------------------------
 * Encode N vectors [P4, K flow steps 1-5; V section: steps 1-3 only].
 *   1. n = ||x||, x_hat = x / n                         (step 1)
 *   2. y = H D x_hat                                    (step 2)
 *   3. idx_j = #{ i : b_i <= y_j }  (ties go up)        (step 3)
 *   4. r = y - c[idx], gamma = ||r||                    (step 4)
 *   5. z = S r, sigma_i = [z_i >= 0]                    (step 5)
 * A zero vector encodes as idx 4, gamma 0 and all signs 1.
 * Outputs are unrounded n, gamma (the caller rounds them to fp16 as stored);
 * y and z are returned for the boundary-window accounting of the tests.
 * with_qjl = 0 gives the V path (sig, gam and z untouched).
 * ---------------------------------------------------------------------- */
/* Steps 4-5 for one vector whose codes are given: r = y - c[idx] (r = 0 for a
 * zero input), gamma = ||r||, z = S r, sigma_i = [z_i >= 0]. */
static void orc_residual_sketch(int d, const double* S, const double* c8, const double* y,
                                const uint8_t* idx, int nonzero, uint8_t* sig, double* gam,
                                double* z_out) {
    const int m = d;
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    double g2 = 0.0;
    for (int j = 0; j < d; ++j) {
        r[j] = nonzero ? y[j] - c8[idx[j]] : 0.0;
        g2 += r[j] * r[j];
    }
    *gam = sqrt(g2);
    for (int i = 0; i < m; ++i) {
        double z = 0.0;
        for (int j = 0; j < d; ++j) z += S[(size_t)i * d + j] * r[j];
        sig[i] = (z >= 0.0) ? 1 : 0;
        if (z_out) z_out[i] = z;
    }
    free(r);
}

void orc_encode(int d, const int8_t* D, const double* S, const double* c8, const double* b7,
                const double* x, int64_t N, int with_qjl,
                uint8_t* idx, uint8_t* sig, double* nrm, double* gam,
                double* y_out, double* z_out) {
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < N; ++v) {
        const double* xv = x + v * d;
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += xv[j] * xv[j];
        double n = sqrt(ss);                                   /* step 1 */
        nrm[v] = n;
        for (int j = 0; j < d; ++j) y[j] = (n > 0.0) ? D[j] * (xv[j] / n) : 0.0;
        orc_fwht(y, d);                                        /* step 2 */
        for (int j = 0; j < d; ++j) {                          /* step 3 */
            int k = 0;
            for (int i = 0; i < 7; ++i) k += (b7[i] <= y[j]) ? 1 : 0;
            idx[v * d + j] = (uint8_t)k;
            if (y_out) y_out[v * d + j] = y[j];
        }
        if (with_qjl)                                          /* steps 4-5 */
            orc_residual_sketch(d, S, c8, y, idx + v * d, n > 0.0, sig + v * d, &gam[v],
                                z_out ? z_out + v * d : NULL);
        free(y);
    }
}

/* Steps 4-5 for N vectors with y and the codes supplied (y [N][d], idx [N][d],
 * nonzero [N]): lets a test compare sign bits where the two sides took a
 * different code decision inside the boundary window. */
void orc_sketch_given_codes(int d, const double* S, const double* c8, const double* y,
                            const uint8_t* idx, const uint8_t* nonzero, int64_t N,
                            uint8_t* sig, double* gam, double* z_out) {
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < N; ++v)
        orc_residual_sketch(d, S, c8, y + v * d, idx + v * d, nonzero[v], sig + v * d, &gam[v],
                            z_out ? z_out + v * d : NULL);
}

/* ------------------------------------------------------------------------
 * Packed cache layout (this library's own contract; the pages give none
 * beyond the bit budget of 4.25 b/dim for K and 3.125 b/dim for V).
 *
 * A cache is [B][Hkv][Tcap/64 blocks]; one block holds 64 tokens:
 *   K block: codes 64 x 3d/8 B | signs 64 x d/8 B | n fp16 x 64 | gamma fp16 x 64
 *   V block: codes 64 x 3d/8 B | n fp16 x 64
 * Per token, codes are 3d/32 little-endian uint32 words: for slice s (128
 * coordinates) and slot t (0..3) words 12s+3t+{0,1,2} = Wa, Wb, Wc hold slot
 * codes i = 0..31, slot code i meaning coordinate
 *     j = 128 s + 16 (i >> 2) + 2 t + (i & 1) + 8 ((i >> 1) & 1).
 * Nibble k (bits 4k..4k+3) of Wa holds code(i=k) in bits 0-2 and bit 0 of
 * code(24+k) in bit 3; Wb: code(8+k) and bit 1 of code(24+k); Wc: code(16+k)
 * and bit 2 of code(24+k).
 * Signs are d/32 words per token: word 4s+t has sign(i = 2q) at bit q and
 * sign(i = 2q+1) at bit 16+q (q = 0..15), i mapping to a JL row as above.
 * d = 64 has one 64-coordinate slice of 16 codes per slot (i = 0..15, same
 * coordinate formula with s = 0).  Per token, word t (t = 0..3) holds code(k)
 * in bits 0-2 of nibble k (k = 0..7); halfword t of bytes 16..23 (bits
 * 16 (t & 1) .. of word 4 + t / 2) holds code(8 + k) in bits 0-2 of nibble k
 * (k = 0..3); the three bits of code(12 + k) are bit 3 of nibble k of word t,
 * bit 3 of nibble 4 + k of word t and bit 3 of nibble k of halfword t.  Its
 * signs are 4 halfwords per token: bit i of halfword t (bits 16 (t & 1) + i
 * of word t / 2) is the sign of the JL row of slot position i.
 * These functions pack/unpack one (b, kv-head) sequence of Tcap slots.
 * ---------------------------------------------------------------------- */
int64_t orc_block_bytes(int d, int is_k) {
    int64_t codes = (int64_t)ORC_BLOCK_T * 3 * d / 8;
    if (is_k) return codes + (int64_t)ORC_BLOCK_T * d / 8 + 4 * ORC_BLOCK_T;
    return codes + 2 * ORC_BLOCK_T;
}

static int orc_slot_coord(int s, int t, int i) {
    return 128 * s + 16 * (i >> 2) + 2 * t + (i & 1) + 8 * ((i >> 1) & 1);
}

static void orc_put_bit(uint32_t* w, int pos, int bit) {
    if (bit) *w |= (1u << pos);
    else *w &= ~(1u << pos);
}
static int orc_get_bit(uint32_t w, int pos) { return (int)((w >> pos) & 1u); }

/* d = 64: bit `bit` of halfword t of the code record (words 4, 5) */
static int orc_h64_pos(int t, int bit) { return 16 * (t & 1) + bit; }

static void orc_pack_codes64(const uint8_t* code, uint32_t* words) {
    for (int w = 0; w < 6; ++w) words[w] = 0;
    for (int t = 0; t < 4; ++t) {
        uint32_t* H = &words[4 + t / 2];
        for (int k = 0; k < 8; ++k) {
            int c = code[orc_slot_coord(0, t, k)];
            for (int b = 0; b < 3; ++b) orc_put_bit(&words[t], 4 * k + b, (c >> b) & 1);
        }
        for (int k = 0; k < 4; ++k) {
            int c = code[orc_slot_coord(0, t, 8 + k)];
            for (int b = 0; b < 3; ++b) orc_put_bit(H, orc_h64_pos(t, 4 * k + b), (c >> b) & 1);
            int c4 = code[orc_slot_coord(0, t, 12 + k)];
            orc_put_bit(&words[t], 4 * k + 3, c4 & 1);
            orc_put_bit(&words[t], 4 * (4 + k) + 3, (c4 >> 1) & 1);
            orc_put_bit(H, orc_h64_pos(t, 4 * k + 3), (c4 >> 2) & 1);
        }
    }
}

static void orc_unpack_codes64(const uint32_t* words, uint8_t* code) {
    for (int t = 0; t < 4; ++t) {
        const uint32_t H = words[4 + t / 2];
        for (int k = 0; k < 8; ++k) {
            int c = 0;
            for (int b = 0; b < 3; ++b) c |= orc_get_bit(words[t], 4 * k + b) << b;
            code[orc_slot_coord(0, t, k)] = (uint8_t)c;
        }
        for (int k = 0; k < 4; ++k) {
            int c = 0;
            for (int b = 0; b < 3; ++b) c |= orc_get_bit(H, orc_h64_pos(t, 4 * k + b)) << b;
            code[orc_slot_coord(0, t, 8 + k)] = (uint8_t)c;
            int c4 = orc_get_bit(words[t], 4 * k + 3) | (orc_get_bit(words[t], 4 * (4 + k) + 3) << 1) |
                     (orc_get_bit(H, orc_h64_pos(t, 4 * k + 3)) << 2);
            code[orc_slot_coord(0, t, 12 + k)] = (uint8_t)c4;
        }
    }
}

static void orc_pack_codes(int d, const uint8_t* code, uint32_t* words) {
    if (d == 64) {
        orc_pack_codes64(code, words);
        return;
    }
    for (int s = 0; s < d / 128; ++s)
        for (int t = 0; t < 4; ++t) {
            uint32_t* W = words + 12 * s + 3 * t;
            W[0] = W[1] = W[2] = 0;
            for (int k = 0; k < 8; ++k) {
                for (int g = 0; g < 3; ++g) {        /* Wa, Wb, Wc: codes k, 8+k, 16+k */
                    int c = code[orc_slot_coord(s, t, 8 * g + k)];
                    for (int b = 0; b < 3; ++b) orc_put_bit(&W[g], 4 * k + b, (c >> b) & 1);
                }
                int c4 = code[orc_slot_coord(s, t, 24 + k)];
                for (int g = 0; g < 3; ++g) orc_put_bit(&W[g], 4 * k + 3, (c4 >> g) & 1);
            }
        }
}

static void orc_unpack_codes(int d, const uint32_t* words, uint8_t* code) {
    if (d == 64) {
        orc_unpack_codes64(words, code);
        return;
    }
    for (int s = 0; s < d / 128; ++s)
        for (int t = 0; t < 4; ++t) {
            const uint32_t* W = words + 12 * s + 3 * t;
            for (int k = 0; k < 8; ++k) {
                for (int g = 0; g < 3; ++g) {
                    int c = 0;
                    for (int b = 0; b < 3; ++b) c |= orc_get_bit(W[g], 4 * k + b) << b;
                    code[orc_slot_coord(s, t, 8 * g + k)] = (uint8_t)c;
                }
                int c4 = 0;
                for (int g = 0; g < 3; ++g) c4 |= orc_get_bit(W[g], 4 * k + 3) << g;
                code[orc_slot_coord(s, t, 24 + k)] = (uint8_t)c4;
            }
        }
}

static void orc_pack_signs(int d, const uint8_t* sg, uint32_t* words) {
    if (d == 64) {
        words[0] = words[1] = 0;
        for (int t = 0; t < 4; ++t)
            for (int i = 0; i < 16; ++i) orc_put_bit(&words[t / 2], 16 * (t & 1) + i, sg[orc_slot_coord(0, t, i)]);
        return;
    }
    for (int s = 0; s < d / 128; ++s)
        for (int t = 0; t < 4; ++t) {
            uint32_t w = 0;
            for (int q = 0; q < 16; ++q) {
                orc_put_bit(&w, q, sg[orc_slot_coord(s, t, 2 * q)]);
                orc_put_bit(&w, 16 + q, sg[orc_slot_coord(s, t, 2 * q + 1)]);
            }
            words[4 * s + t] = w;
        }
}

static void orc_unpack_signs(int d, const uint32_t* words, uint8_t* sg) {
    if (d == 64) {
        for (int t = 0; t < 4; ++t)
            for (int i = 0; i < 16; ++i)
                sg[orc_slot_coord(0, t, i)] = (uint8_t)orc_get_bit(words[t / 2], 16 * (t & 1) + i);
        return;
    }
    for (int s = 0; s < d / 128; ++s)
        for (int t = 0; t < 4; ++t)
            for (int q = 0; q < 16; ++q) {
                sg[orc_slot_coord(s, t, 2 * q)] = (uint8_t)orc_get_bit(words[4 * s + t], q);
                sg[orc_slot_coord(s, t, 2 * q + 1)] = (uint8_t)orc_get_bit(words[4 * s + t], 16 + q);
            }
}

/* byte offsets of the fields of token tau inside its block */
static int64_t orc_off_codes(int d, int tau) { return (int64_t)tau * 3 * d / 8; }
static int64_t orc_off_signs(int d, int tau) {
    return (int64_t)ORC_BLOCK_T * 3 * d / 8 + (int64_t)tau * d / 8;
}
static int64_t orc_off_norm(int d, int is_k, int tau) {
    int64_t base = (int64_t)ORC_BLOCK_T * 3 * d / 8 + (is_k ? (int64_t)ORC_BLOCK_T * d / 8 : 0);
    return base + 2 * tau;
}
static int64_t orc_off_gamma(int d, int tau) {
    return (int64_t)ORC_BLOCK_T * 3 * d / 8 + (int64_t)ORC_BLOCK_T * d / 8 + 2 * ORC_BLOCK_T + 2 * tau;
}

/* tokens [t0, t0 + T) of one sequence; blocks points at the sequence's first block */
void orc_pack(int d, int is_k, int64_t t0, int64_t T, const uint8_t* idx, const uint8_t* sig,
              const uint16_t* nh, const uint16_t* gh, uint8_t* blocks) {
    const int64_t bb = orc_block_bytes(d, is_k);
    for (int64_t tt = 0; tt < T; ++tt) {
        int64_t t = t0 + tt;
        uint8_t* blk = blocks + (t / ORC_BLOCK_T) * bb;
        int tau = (int)(t % ORC_BLOCK_T);
        uint32_t cw[24], sw[8];
        orc_pack_codes(d, idx + tt * d, cw);
        memcpy(blk + orc_off_codes(d, tau), cw, (size_t)3 * d / 8);
        memcpy(blk + orc_off_norm(d, is_k, tau), &nh[tt], 2);
        if (is_k) {
            orc_pack_signs(d, sig + tt * d, sw);
            memcpy(blk + orc_off_signs(d, tau), sw, (size_t)d / 8);
            memcpy(blk + orc_off_gamma(d, tau), &gh[tt], 2);
        }
    }
}

void orc_unpack(int d, int is_k, int64_t t0, int64_t T, const uint8_t* blocks,
                uint8_t* idx, uint8_t* sig, uint16_t* nh, uint16_t* gh) {
    const int64_t bb = orc_block_bytes(d, is_k);
#pragma omp parallel for schedule(static)
    for (int64_t tt = 0; tt < T; ++tt) {
        int64_t t = t0 + tt;
        const uint8_t* blk = blocks + (t / ORC_BLOCK_T) * bb;
        int tau = (int)(t % ORC_BLOCK_T);
        uint32_t cw[24], sw[8];
        memcpy(cw, blk + orc_off_codes(d, tau), (size_t)3 * d / 8);
        orc_unpack_codes(d, cw, idx + tt * d);
        memcpy(&nh[tt], blk + orc_off_norm(d, is_k, tau), 2);
        if (is_k) {
            memcpy(sw, blk + orc_off_signs(d, tau), (size_t)d / 8);
            orc_unpack_signs(d, sw, sig + tt * d);
            memcpy(&gh[tt], blk + orc_off_gamma(d, tau), 2);
        }
    }
}

/* ------------------------------------------------------------------------
 * Decode attention of G query heads that share one compressed KV head
 * [P4 hybrid section: dequantisation fused into the attention shader; K
 * section: the QJL bit acts on inner-product attention scores; V section: V is
 * not scored, so it carries no QJL bit].  With q' = H D q and u = S q':
 *   s_t = scale * n_t * ( <q', c[idx_t]> + gamma_t * sqrt(pi/2)/m * <u, 2 sigma_t - 1> )
 *   p   = softmax(s)    (max-subtracted)
 *   o   = D H sum_t p_t * nv_t * c[idxv_t]
 * n_t, gamma_t and nv_t are the stored fp16 values, decoded.  T == 0 gives a
 * zero output.  Layouts: q [G][d]; idx/sig [T][d]; out [G][d].
 * ---------------------------------------------------------------------- */
/* scores s_t of one query head (q [d]) against tokens [0, T); s [T] */
void orc_scores(int d, const int8_t* D, const double* S, const double* c8, const double* q,
                int64_t T, const uint8_t* idxk, const uint8_t* sig, const double* nk,
                const double* gk, double scale, double* s) {
    const int m = d;
    const double cq = sqrt(M_PI / 2.0) / m;
    double* qp = (double*)malloc(sizeof(double) * (size_t)d);
    double* u = (double*)malloc(sizeof(double) * (size_t)m);
    for (int j = 0; j < d; ++j) qp[j] = D[j] * q[j];
    orc_fwht(qp, d);                                   /* q' = H D q */
    for (int i = 0; i < m; ++i) {                      /* u = S q' */
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += S[(size_t)i * d + j] * qp[j];
        u[i] = a;
    }
    /* tokens are independent: split over threads, each score summed as written */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double a = 0.0, b = 0.0;
        for (int j = 0; j < d; ++j) a += qp[j] * c8[idxk[t * d + j]];
        for (int i = 0; i < m; ++i) b += u[i] * (2.0 * sig[t * m + i] - 1.0);
        s[t] = scale * nk[t] * (a + gk[t] * cq * b);
    }
    free(qp);
    free(u);
}

/* Threads split the work without changing any sum: the scores by token (each
 * score summed over its coordinates as written), the value sum by coordinate
 * (each acc[j] summed over the tokens in order t = 0, 1, ...). */
void orc_attend(int d, int G, const int8_t* D, const double* S, const double* c8,
                const double* q, int64_t T,
                const uint8_t* idxk, const uint8_t* sig, const double* nk, const double* gk,
                const uint8_t* idxv, const double* nv, double scale, double* out) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    for (int g = 0; g < G; ++g) {
        orc_scores(d, D, S, c8, q + (size_t)g * d, T, idxk, sig, nk, gk, scale, s);
        double smax = -INFINITY;
        for (int64_t t = 0; t < T; ++t)
            if (s[t] > smax) smax = s[t];
        double l = 0.0;
        for (int64_t t = 0; t < T; ++t) {              /* softmax weights */
            p[t] = exp(s[t] - smax);
            l += p[t];
        }
#pragma omp parallel for schedule(static)
        for (int j = 0; j < d; ++j) {                  /* V summed in the rotated domain */
            double a = 0.0;
            for (int64_t t = 0; t < T; ++t) a += p[t] * nv[t] * c8[idxv[t * d + j]];
            acc[j] = a;
        }
        for (int j = 0; j < d; ++j) acc[j] = (T > 0) ? acc[j] / l : 0.0;
        orc_fwht(acc, d);                              /* single inverse transform: D H */
        for (int j = 0; j < d; ++j) out[(size_t)g * d + j] = D[j] * acc[j];
    }
    free(acc);
    free(p);
    free(s);
}

/* Threads used by the parallel loops from now on (n <= 0: all the host's cores). */
void orc_set_threads(int n) {
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
#else
    (void)n;
#endif
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_to_fp16_array(const double* x, int64_t n, uint16_t* h) {
    for (int64_t i = 0; i < n; ++i) h[i] = orc_to_fp16(x[i]);
}
