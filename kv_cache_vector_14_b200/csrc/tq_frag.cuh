// Shared pieces of the tensor-core attention kernels (split-K decode and
// chunked prefill): the per-head-dim shape of a staged chunk of the packed
// cache, bulk-copy and mbarrier helpers, mma.sync wrappers, and the
// dequantisation of the packed codes into fp16 fragments (see the cache
// layout in tq.h: a lane's 32 codes of one slot are three words whose nibbles
// index byte look-up tables of the fp16 centroids).
#pragma once

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kStages = 3;             // ring depth per warp
constexpr int kWaitLimit = kDefaultWaitLimit;

// Per-head-dim shape of a ring stage (bytes).  QJL = false: the K cache is a
// PolarQuant-only cache in the V layout (codes and norms, no signs, no gamma).
template <int D, bool QJL = true>
struct Cfg {
    static constexpr int kS = D >= 128 ? D / 128 : 1;         // 128-coordinate slices (d = 64: one half slice)
    static constexpr int kKC = D / 16;                        // coordinate chunks (mma k-steps)
    static constexpr int kCodeB = 3 * D / 8;                  // code bytes per token
    static constexpr int kSignB = D / 8;                      // sign bytes per token (QJL)
    static constexpr int kChunk = D <= 128 ? 32 : 16;         // tokens per stage
    static constexpr int kTiles = kChunk / 16;
    static constexpr int kOffKc = 0;
    static constexpr int kOffKs = kOffKc + kChunk * kCodeB;
    static constexpr int kOffKn = kOffKs + (QJL ? kChunk * kSignB : 0);
    static constexpr int kOffKg = kOffKn + 2 * kChunk;
    static constexpr int kOffVc = kOffKg + (QJL ? 2 * kChunk : 0);
    static constexpr int kOffVn = kOffVc + kChunk * kCodeB;
    static constexpr int kStageB = kOffVn + 2 * kChunk;
    static constexpr bool kBRegs = D <= 128;                   // q'/u' fragments in registers
    static_assert(kStageB % 16 == 0 && kOffKn % 16 == 0 && kOffKg % 16 == 0 && kOffVc % 16 == 0 &&
                      kOffVn % 16 == 0,
                  "stage fields must keep 16-byte alignment");
};


// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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
// Wait for the phase of parity `parity` to complete; give up after `limit`
// polls or about one second, whichever comes first (a poll may suspend the
// thread for an unspecified time, so the count alone bounds nothing in time).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int limit = kWaitLimit) {
    if (limit <= 0) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (int i = 1; i < limit; ++i) {
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
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D += A B with signed 8-bit operands and exact 32-bit integer accumulation
__device__ __forceinline__ void imma16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// 2^x on the special-function unit (relative error ~2^-22); -inf gives 0
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// fp32 pair -> (hi, lo) fp16 pairs with hi + lo carrying ~22 significant bits
__device__ __forceinline__ void split_hilo(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 hf = __half22float2(h);
    hi = h2_bits(h);
    lo = h2_bits(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}

// Left shifts as integer multiplies, x << k = x * 2^k (IMAD): the powers of two
// come from the kernel parameters, so the compiler cannot turn them back into
// shifts; they run on the FMA pipe and leave the ALU pipe (prmt, lop3) to the
// dequantisation.  Right shifts stay shifts (the multiply-high form is a
// quarter-rate instruction).
__device__ __forceinline__ uint32_t shl_m(uint32_t x, const uint32_t* pw, int k) { return x * pw[k]; }
__device__ __forceinline__ uint32_t shr_m(uint32_t x, const uint32_t* pw, int k) { (void)pw; return x >> k; }

// Selector words for the 32 slot codes of one token: sel[w] holds, in its
// nibbles, the codes of slot positions 8w .. 8w+7.
__device__ __forceinline__ void code_selectors(const uint8_t* rec, const uint32_t* pw, uint32_t (&sel)[4]) {
    const uint32_t wa = *reinterpret_cast<const uint32_t*>(rec);
    const uint32_t wb = *reinterpret_cast<const uint32_t*>(rec + 4);
    const uint32_t wc = *reinterpret_cast<const uint32_t*>(rec + 8);
    sel[0] = wa & 0x77777777u;
    sel[1] = wb & 0x77777777u;
    sel[2] = wc & 0x77777777u;
    // bit 3 of each nibble of wa, wb, wc holds bits 0, 1, 2 of codes 24..31
    sel[3] = (shr_m(wa, pw, 3) & 0x11111111u) | (shr_m(wb, pw, 2) & 0x22222222u) |
             (shr_m(wc, pw, 1) & 0x44444444u);
}

// fp16 centroid pairs for slot positions 4kc .. 4kc+3: e=0,1 -> x0, e=2,3 -> x1
__device__ __forceinline__ void dequant4(uint32_t sel16, const uint32_t (&lut)[4], uint32_t& x0, uint32_t& x1) {
    const uint32_t lo4 = __byte_perm(lut[0], lut[1], sel16);
    const uint32_t hi4 = __byte_perm(lut[2], lut[3], sel16);
    x0 = __byte_perm(lo4, hi4, 0x5140);
    x1 = __byte_perm(lo4, hi4, 0x7362);
}

__device__ __forceinline__ uint32_t sel_for(const uint32_t (&sel)[4], const uint32_t* pw, int kc) {
    return (kc & 1) ? shr_m(sel[kc >> 1], pw, 16) : sel[kc >> 1];
}

// Selector words of slot t of slice sl of one token record (tok), in the
// sel_for order.  d = 64 (16 codes per slot): word t gives positions 0..7
// (sel[0]); halfword t gives positions 8..11 and, with the bit-3 planes of
// both, positions 12..15 (sel[1]).
template <int D>
__device__ __forceinline__ void token_selectors(const uint8_t* tok, int sl, int t, const uint32_t* pw,
                                                uint32_t (&sel)[4]) {
    if constexpr (D == 64) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(tok + 4 * t);
        const uint32_t h = *reinterpret_cast<const uint16_t*>(tok + 16 + 2 * t);
        sel[0] = w & 0x77777777u;
        const uint32_t plane = (shr_m(w, pw, 3) & 0x1111u) | (shr_m(w, pw, 18) & 0x2222u) | (shr_m(h, pw, 1) & 0x4444u);
        sel[1] = (h & 0x7777u) | shl_m(plane, pw, 16);
        sel[2] = sel[3] = 0u;
    } else {
        code_selectors(tok + sl * 48 + t * 12, pw, sel);
    }
}

// Sign word of slot t of slice sl of one token's sign record.  d = 64: the
// 16-bit halfword h of slot t as h | h << 20 (m64 = 2^20 + 1), so that byte e
// of the word has h's bits 4e' .. 4e'+3 in its bits 4..7 (e' = 1, 3, 0, 2 for
// e = 0..3) and the shifts of the d >= 128 extraction pick every bit once.
template <int D>
__device__ __forceinline__ uint32_t token_signs(const uint8_t* tok, int sl, int t, uint32_t m64) {
    if constexpr (D == 64) return (uint32_t)*reinterpret_cast<const uint16_t*>(tok + 2 * t) * m64;
    else return *reinterpret_cast<const uint32_t*>(tok + sl * 16 + t * 4);
}

}  // namespace
}  // namespace tqi
