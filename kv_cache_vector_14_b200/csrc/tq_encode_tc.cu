// TurboQuant K/V encode for head_dim 128 on sm_100a, with the QJL projection
// of the K path on the 5th-generation tensor cores (tcgen05, accumulators in
// tensor memory).
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com), section "K-Cache圧縮：3-bit PolarQuant +
// 1-bit QJL = 4.25 bits/dim" (steps 1-5) and section "V-Cache圧縮：3-bit
// PolarQuant = 3.125 bits/dim" (steps 1-3, no QJL).
//
// Per vector, 8 lanes of a warp (lane l holds coordinates 16 l .. 16 l + 15,
// four vectors per warp at a time): ||x|| by three shuffle steps, the random
// sign flip, the Walsh-Hadamard butterflies (4 register stages over coordinate
// bits 0..3, 3 shuffle stages over bits 4..6), the scale 1 / (||x|| sqrt(d)),
// the bucket index and centroid by saturating compares on the FMA pipe, and for
// K the residual r = y - c[idx] and gamma = ||r||.
//
// K, step 5 (z = S r, sign bits): the tile's residuals (up to 128 vectors) are
// written to shared memory as two fp16 limbs of r * 2^12 (hi = fp16(r 2^12),
// lo = fp16 of the remainder), in the 128-byte-swizzled K-major layout the
// tensor core reads.  The JL matrix is held the same way (hi, lo limbs of the
// fp32 S), its rows permuted so that column n of the product is bit n % 32 of
// stored sign word n / 32.  The tensor core accumulates in fp32 in tensor
// memory
//     Z = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T
// with 24 tcgen05.mma (M = 128 vectors, N = 128 JL rows, K = 16).  The limbs
// carry ~22 significant bits and the dropped lo*lo term is ~2^-22 relative,
// so |dz| stays near 1e-7 for a unit-norm direction, below the 1e-6 exclusion
// window of the parity rule.  Each thread then loads one 32-column row
// segment of Z (one sign word of one vector) and sets bit b when z >= 0.
//
// One tile of tile_rows vectors per CTA iteration; the CTA (16 warps, one per
// SM) stages the JL limbs once (one bulk copy) and loops over tiles.  The
// residual operand and the accumulator are double-buffered: the mma of tile i
// runs while the warps compute steps 1-4 of tile i + 1, and its sign words are
// read out after that.  Small
// encodes (one new token per head) use short tiles so that they spread over
// many SMs; every vector goes through the same instructions whatever its row,
// so bulk encodes and one-token appends store identical bytes.
#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kD = 128;
constexpr int kWarps = 16;                      // K kernel: 512 threads, one CTA per SM
constexpr int kOpBytes = kTcRows * kD * 2;      // one fp16 limb of a 128 x 128 operand (32 KB)
constexpr float kRScale = 4096.f;               // residual scale before the fp16 split
constexpr int kWaitLimit = 1 << 20;

constexpr int kOffA = 0;                        // two residual buffers, each hi then lo limb
constexpr int kABytes = 2 * kOpBytes;
constexpr int kOffBhi = 2 * kABytes;            // B image (hi then lo), one bulk copy
constexpr int kOffCode = kOffBhi + 2 * kOpBytes; // [16 warps][4 vectors][128] code bytes in slot order
constexpr int kOffBar = kOffCode + kWarps * 4 * 128;
constexpr int kSmemK = kOffBar + 64 + 1024;     // + slack to align the base to 1024 bytes
static_assert(kSmemK <= 227 * 1024, "shared memory per CTA");

// instruction descriptor: D fp32, A and B fp16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// give up after kWaitLimit polls or about one second, whichever comes first
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (int i = 1; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0 && global_ns() - t0 > kWaitNs) return false;
    }
    return false;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16, issued by one thread
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}
// the mbarrier completes once every mma issued so far by this thread is done
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane; the wait is
// in the same statement so no use of the registers can move above it
__device__ __forceinline__ void tc_load32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
// shared-memory operand descriptor: 128-byte swizzle, K-major, 8-row groups
// 1024 bytes apart (leading offset unused for this layout), descriptor version 1
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// ---------------------------------------------------------------- phase 1
template <int DT>
__device__ __forceinline__ void load16(const void* x, int64_t off, bool vec, float (&v)[16]) {
    if constexpr (DT == TQ_F32) {
        const float* p = static_cast<const float*>(x) + off;
        if (vec) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 f = __ldg(reinterpret_cast<const float4*>(p) + k);
                v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __ldg(p + i);
        }
    } else {
        const uint16_t* p = static_cast<const uint16_t*>(x) + off;
        uint32_t w[8];
        if (vec) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = (uint32_t)__ldg(p + 2 * k) | ((uint32_t)__ldg(p + 2 * k + 1) << 16);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if constexpr (DT == TQ_BF16) {
                v[2 * k] = __uint_as_float(w[k] << 16);
                v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            } else {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
                v[2 * k] = f.x;
                v[2 * k + 1] = f.y;
            }
        }
    }
}

struct GroupOut {
    uint32_t cw[4];    // slot t: codes of positions 4l .. 4l+3 as bytes
    uint32_t rh[8];    // K: fp16 hi limbs of r * 2^12, coordinates 16 l + 2k, +1
    uint32_t rl[8];    // K: fp16 lo limbs
    float n;           // ||x||
    float g2;          // ||r||^2 (K)
};

// Steps 1-4 for the vector of this lane's group of 8 lanes (lane l = lane & 7).
template <int DT, bool IS_K>
__device__ __forceinline__ void encode_group(const void* x, int64_t off, bool valid, bool vec, int l,
                                             const float (&dsg)[16], const Codebook& cb, GroupOut& o) {
    float v[16];
    if (valid) {
        load16<DT>(x, off + 16 * l, vec, v);
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) ss = fmaf(v[i], v[i], ss);
    ss += __shfl_xor_sync(kFull, ss, 1);
    ss += __shfl_xor_sync(kFull, ss, 2);
    ss += __shfl_xor_sync(kFull, ss, 4);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] *= dsg[i];
    // butterflies over coordinate bits 0..3 (registers)
#pragma unroll
    for (int hb = 1; hb < 16; hb <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & hb) == 0) {
                const float u = v[i], w = v[i | hb];
                v[i] = u + w;
                v[i | hb] = u - w;
            }
    // butterflies over coordinate bits 4..6 (lanes of the group)
#pragma unroll
    for (int hb = 1; hb < 8; hb <<= 1) {
        const float sg = (l & hb) ? -1.f : 1.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float p = __shfl_xor_sync(kFull, v[i], hb);
            v[i] = fmaf(v[i], sg, p);            // own + partner, or partner - own
        }
    }
    const float n = sqrtf(ss);
    const bool nz = n > 0.f;
    const float rcp = nz ? __frcp_rn(n * 11.3137084989847604f) : 0.f;   // 1 / (||x|| sqrt(128))
    // Bucket index and centroid on the FMA pipe.  The codebook is antisymmetric
    // (b3 = 0, b[6-k] = -b[k], c[7-k] = -c[k]), so with a = |y| and
    // t_k = sat((b_k - a) 2^60) = [a < b_k] for k = 4, 5, 6 (the product is exact,
    // its sign decides, and any nonzero difference of two such floats
    // saturates), T = t4 + t5 + t6 boundaries lie above a: the code is 7 - T for
    // y >= 0 and T below (a tie at a positive boundary goes up; at a negative
    // one it goes down, which is inside the 1e-6 window), and
    // |c| = c7 - t6 (c7 - c6) - t5 (c6 - c5) - t4 (c5 - c4), every partial sum an
    // exact centroid.
    constexpr float kBig = 1152921504606846976.f;        // 2^60
    const float bb4 = cb.b[4] * kBig, bb5 = cb.b[5] * kBig, bb6 = cb.b[6] * kBig;
    [[maybe_unused]] const float d3 = cb.c[7] - cb.c[6], d2 = cb.c[6] - cb.c[5], d1 = cb.c[5] - cb.c[4];
    float codef[16];
    float g2 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float rr[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float y = v[i + e] * rcp;
            const float a = fabsf(y);
            const float t4 = __saturatef(fmaf(a, -kBig, bb4));
            const float t5 = __saturatef(fmaf(a, -kBig, bb5));
            const float t6 = __saturatef(fmaf(a, -kBig, bb6));
            const float T = (t4 + t5) + t6;
            const float pos = (y >= 0.f) ? 1.f : 0.f;
            codef[i + e] = fmaf(pos, fmaf(T, -2.f, 7.f), T);
            if constexpr (IS_K) {
                float m = fmaf(-t6, d3, cb.c[7]);
                m = fmaf(-t5, d2, m);
                m = fmaf(-t4, d1, m);
                const float r = nz ? y - m * fmaf(pos, 2.f, -1.f) : 0.f;
                g2 = fmaf(r, r, g2);
                rr[e] = r * kRScale;
            }
        }
        if constexpr (IS_K) {
            const __half2 h = __floats2half2_rn(rr[0], rr[1]);
            const float2 hf = __half22float2(h);
            const __half2 lo = __floats2half2_rn(rr[0] - hf.x, rr[1] - hf.y);
            o.rh[i >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            o.rl[i >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
        }
    }
    if constexpr (IS_K) {
        g2 += __shfl_xor_sync(kFull, g2, 1);
        g2 += __shfl_xor_sync(kFull, g2, 2);
        g2 += __shfl_xor_sync(kFull, g2, 4);
    }
    // slot t holds positions 4l + {0,1,2,3} = coordinates 16l + {2t, 2t+1, 2t+8, 2t+9}; the
    // byte pairs are formed as exact float sums and read out of the mantissa (x + 2^23)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float lo = fmaf(codef[2 * t + 1], 256.f, codef[2 * t]) + 8388608.f;
        const float hi = fmaf(codef[2 * t + 9], 256.f, codef[2 * t + 8]) + 8388608.f;
        o.cw[t] = __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x5410);
    }
    o.n = n;
    o.g2 = g2;
}

// Pack 8 byte-sized values (< 16) held in two words into 8 nibbles.
__device__ __forceinline__ uint32_t nibbles8(uint32_t lo4, uint32_t hi4) {
    uint32_t a = (lo4 | (lo4 >> 4)) & 0x00FF00FFu;
    a = (a | (a >> 8)) & 0x0000FFFFu;
    uint32_t b = (hi4 | (hi4 >> 4)) & 0x00FF00FFu;
    b = (b | (b >> 8)) & 0x0000FFFFu;
    return a | (b << 16);
}

// Code word w (0..11) of a token record from its 128 staged code bytes.
__device__ __forceinline__ uint32_t pack_code_word(const uint8_t* rec, int w) {
    const int t = w / 3, g = w % 3;
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(rec + t * 32);
    const uint32_t main = nibbles8(sw[2 * g], sw[2 * g + 1]);
    const uint32_t tail = nibbles8(sw[6], sw[7]);
    return main | (((tail >> g) & 0x11111111u) << 3);
}

// The 12 code words of each of the warp's four vectors (group g holds vector
// g; my_rec is the code record of this lane's vector, null to skip) from the
// staged bytes.
__device__ __forceinline__ void store_code_words(const uint8_t* stage, uint8_t* my_rec, int nvalid, int lane) {
    const unsigned long long mine = reinterpret_cast<unsigned long long>(my_rec);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int idx = lane + 32 * k;                 // 4 vectors x 12 words
        const int vv = idx / 12, w = idx % 12;
        const unsigned long long rec = __shfl_sync(kFull, mine, 8 * (vv < 4 ? vv : 3));
        if (idx < 48 && vv < nvalid && rec != 0ull)
            reinterpret_cast<uint32_t*>(rec)[w] = pack_code_word(stage + vv * 128, w);
    }
}

// ---------------------------------------------------------------- K kernel
template <int DT>
__global__ void __launch_bounds__(kWarps * 32, 1) tq_encode_k128_tc_kernel(const EncArgs a, int tile_rows) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);     // [0] JL image copy, [1..2] mma done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + 32);
    uint8_t* scode = sm + kOffCode;
    pdl_trigger();                 // a chained kernel may start (it waits for this one's writes)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 3, l = lane & 7;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + tile_rows - 1) / tile_rows;
    const int64_t bb = block_bytes(kD, true);
    const uint32_t bar_b = smem_u32(&bars[0]);

    if (threadIdx.x == 0) {
        mbar_init(bar_b, 1);
        mbar_init(smem_u32(&bars[1]), 1);
        mbar_init(smem_u32(&bars[2]), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), 2 * kTcRows);    // two 128-column fp32 accumulators
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        mbar_expect_tx(bar_b, 2 * kOpBytes);
        bulk_g2s(sbase + kOffBhi, a.bimg, 2 * kOpBytes, bar_b);
    }
    float dsg[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) dsg[i] = __ldg(a.dsign + 16 * l + i);
    const bool vec = a.vec16 != 0;

    bool failed = __syncthreads_or(!mbar_wait_bounded(bar_b, 0)) != 0;
    if (failed) {
        if (threadIdx.x == 0) atomicExch(a.err, 1);
        mbar_wait_bounded(bar_b, 0);
    }
    uint32_t phases = 0;                 // bit j: parity of the next completion of buffer j
    int64_t prev_row0 = -1;
    int prev_nrows = 0, buf = 0;

    // sign words of the tile held in accumulator pb: warp w reads lanes
    // 32 (w & 3) .. + 31 and columns 32 (w >> 2) .. + 31 (one word per thread)
    auto finish = [&](int pb, int64_t r0, int nr) -> bool {
        const uint32_t bar = smem_u32(&bars[1 + pb]);
        const bool ok = mbar_wait_bounded(bar, (phases >> pb) & 1u);
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) atomicExch(a.err, 1);
            mbar_wait_bounded(bar, (phases >> pb) & 1u);
            return false;
        }
        phases ^= 1u << pb;
        tc_fence_after();
        uint32_t z[32];
        tc_load32(tmem + (uint32_t)(pb * kTcRows) + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(32 * (warp >> 2)),
                  z);
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 32; ++b) word |= (__uint_as_float(z[b]) >= 0.f ? 1u : 0u) << b;
        const int v = 32 * (warp & 3) + lane;
        if (v < nr) {
            int64_t xoff;
            uint8_t* blk;
            int tau;
            encode_locate(a, (uint32_t)(r0 + v), bb, xoff, blk, tau);
            if (blk)
                reinterpret_cast<uint32_t*>(blk + kBlockT * code_bytes(kD) + tau * sign_bytes(kD))[warp >> 2] = word;
        }
        tc_fence_before();
        return true;
    };

    for (int64_t tile = blockIdx.x; tile < ntiles && !failed; tile += gridDim.x) {
        const int64_t row0 = tile * tile_rows;
        const int nrows = (int)((N - row0) < tile_rows ? (N - row0) : tile_rows);
        uint8_t* A = sm + kOffA + buf * kABytes;
        // ---- steps 1-4: pass p, warp w: tile rows 64 p + 4 w + g; code words stored per pass
        uint8_t* stage = scode + warp * 4 * 128;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int r0 = 64 * p + 4 * warp;
            if (r0 >= nrows) break;                        // warp-uniform
            const int v = r0 + g;
            const bool valid = v < nrows;
            int64_t xoff;
            uint8_t* blk;
            int tau;
            encode_locate(a, (uint32_t)(row0 + (valid ? v : r0)), bb, xoff, blk, tau);
            GroupOut o;
            encode_group<DT, true>(a.x, xoff, valid, vec, l, dsg, a.cb, o);
            *reinterpret_cast<uint4*>(A + sw128_k_offset(v, 16 * l)) = make_uint4(o.rh[0], o.rh[1], o.rh[2], o.rh[3]);
            *reinterpret_cast<uint4*>(A + sw128_k_offset(v, 16 * l + 8)) =
                make_uint4(o.rh[4], o.rh[5], o.rh[6], o.rh[7]);
            *reinterpret_cast<uint4*>(A + kOpBytes + sw128_k_offset(v, 16 * l)) =
                make_uint4(o.rl[0], o.rl[1], o.rl[2], o.rl[3]);
            *reinterpret_cast<uint4*>(A + kOpBytes + sw128_k_offset(v, 16 * l + 8)) =
                make_uint4(o.rl[4], o.rl[5], o.rl[6], o.rl[7]);
#pragma unroll
            for (int t = 0; t < 4; ++t) *reinterpret_cast<uint32_t*>(stage + g * 128 + t * 32 + 4 * l) = o.cw[t];
            if (valid && l == 0 && blk) {
                __half* nf = reinterpret_cast<__half*>(blk + kBlockT * (code_bytes(kD) + sign_bytes(kD)));
                nf[tau] = __float2half_rn(o.n);
                nf[kBlockT + tau] = __float2half_rn(sqrtf(o.g2));
            }
            __syncwarp();
            store_code_words(stage, blk ? blk + tau * code_bytes(kD) : nullptr, nrows - r0, lane);
            __syncwarp();
        }
        // ---- step 5 on the tensor core: Z = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t abase = sbase + kOffA + buf * kABytes, d_tmem = tmem + (uint32_t)(buf * kTcRows);
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t koff = (uint32_t)((ks >> 2) * (kTcRows * 128) + (ks & 3) * 32);
                const uint64_t ah = sw128_desc(abase + koff), al = sw128_desc(abase + kOpBytes + koff);
                const uint64_t bh = sw128_desc(sbase + kOffBhi + koff);
                const uint64_t bl = sw128_desc(sbase + kOffBhi + kOpBytes + koff);
                tc_mma(d_tmem, ah, bh, ks > 0 ? 1u : 0u);
                tc_mma(d_tmem, ah, bl, 1u);
                tc_mma(d_tmem, al, bh, 1u);
            }
            tc_commit(smem_u32(&bars[1 + buf]));
        }
        // ---- sign words of the previous tile (its mma ran under steps 1-4 above)
        if (prev_row0 >= 0 && !finish(buf ^ 1, prev_row0, prev_nrows)) {
            failed = true;
            break;
        }
        prev_row0 = row0;
        prev_nrows = nrows;
        buf ^= 1;
    }
    if (failed) {
        // a timed-out wait: let any mma still in flight finish before releasing tensor memory
        for (int pb = 0; pb < 2; ++pb) mbar_wait_bounded(smem_u32(&bars[1 + pb]), (phases >> pb) & 1u);
    } else if (prev_row0 >= 0) {
        failed = !finish(buf ^ 1, prev_row0, prev_nrows);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, 2 * kTcRows);
    }
    pdl_wait();                    // when chained: complete only after the previous kernel
}

// ---------------------------------------------------------------- V kernel
constexpr int kVWarps = 8;

template <int DT>
__global__ void __launch_bounds__(kVWarps * 32, 3) tq_encode_v128_kernel(const EncArgs a) {
    __shared__ __align__(16) uint8_t scode[kVWarps][4][128];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 3, l = lane & 7;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t nquads = (N + 3) / 4;
    const int64_t bb = block_bytes(kD, false);
    float dsg[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) dsg[i] = __ldg(a.dsign + 16 * l + i);
    const bool vec = a.vec16 != 0;
    for (int64_t q = (int64_t)blockIdx.x * kVWarps + warp; q < nquads; q += (int64_t)gridDim.x * kVWarps) {
        const int64_t gv0 = 4 * q;
        const bool valid = gv0 + g < N;
        int64_t xoff;
        uint8_t* blk;
        int tau;
        encode_locate(a, (uint32_t)(valid ? gv0 + g : gv0), bb, xoff, blk, tau);
        GroupOut o;
        encode_group<DT, false>(a.x, xoff, valid, vec, l, dsg, a.cb, o);
#pragma unroll
        for (int t = 0; t < 4; ++t) *reinterpret_cast<uint32_t*>(&scode[warp][g][t * 32 + 4 * l]) = o.cw[t];
        if (valid && l == 0 && blk) reinterpret_cast<__half*>(blk + kBlockT * code_bytes(kD))[tau] = __float2half_rn(o.n);
        __syncwarp();
        store_code_words(&scode[warp][0][0], blk ? blk + tau * code_bytes(kD) : nullptr, (int)(N - gv0 < 4 ? N - gv0 : 4),
                         lane);
        __syncwarp();
    }
    pdl_wait();
}

template <int DT>
cudaError_t launch_t(bool is_k, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    const int64_t N = a.B * a.Hkv * a.Tnew;
    if (N <= 0) return cudaSuccess;
    if (is_k) {
        // rows per tile: enough tiles to cover the SMs, multiples of 4, at most 128
        int64_t rows = (N + num_sms - 1) / num_sms;
        rows = ((rows + 3) / 4) * 4;
        if (rows > kTcRows) rows = kTcRows;
        const int64_t ntiles = (N + rows - 1) / rows;
        const int grid = (int)(ntiles < num_sms ? ntiles : num_sms);
        auto kern = tq_encode_k128_tc_kernel<DT>;
        cudaError_t e = set_smem_once<tq_encode_k128_tc_kernel<DT>>(kSmemK);
        if (e != cudaSuccess) return e;
        if (pdl) return launch_pdl(kern, dim3(grid), dim3(kWarps * 32), kSmemK, s, a, (int)rows);
        kern<<<grid, kWarps * 32, kSmemK, s>>>(a, (int)rows);
        return cudaGetLastError();
    }
    const int64_t nquads = (N + 3) / 4;
    const int64_t ctas = (nquads + kVWarps - 1) / kVWarps;
    const int64_t cap = (int64_t)num_sms * 8;
    const unsigned grid = (unsigned)(ctas < cap ? ctas : cap);
    const cudaError_t e = set_carveout_once<tq_encode_v128_kernel<DT>>();
    if (e != cudaSuccess) return e;
    if (pdl) return launch_pdl(tq_encode_v128_kernel<DT>, dim3(grid), dim3(kVWarps * 32), 0, s, a);
    tq_encode_v128_kernel<DT><<<grid, kVWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode128(bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    switch (dt) {
        case TQ_F32: return launch_t<TQ_F32>(is_k, a, num_sms, pdl, s);
        case TQ_BF16: return launch_t<TQ_BF16>(is_k, a, num_sms, pdl, s);
        case TQ_F16: return launch_t<TQ_F16>(is_k, a, num_sms, pdl, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tqi
