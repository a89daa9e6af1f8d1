// Tensor-core split-K decode attention over the packed TurboQuant cache
// (head_dim 128, up to 8 query heads per kv head), for sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com), hybrid V2+V3 section: dequantisation is
// fused into the attention kernel.  Per token t and query head g:
//   s = scale * n_t * (<q', c[idx_t]> + gamma_t * <u', 2 sigma_t - 1>),  u' = sqrt(pi/2)/m * S q'
//   acc += softmax weight * nv_t * c[idxv_t]   (rotated domain)
//
// Why tensor cores: per token and kv head the kernel reads 118 bytes but does
// 3 * 128 * G multiply-adds; at G = 4 an fp32 FMA design needs ~12 SM clocks
// per token, about twice the HBM time.  The contraction maps onto
// mma.sync.m16n8k16 (f16 inputs, f32 accumulation) with every operand exact:
//   * dequantised keys/values c[idx] are fp16 numbers (the codebook is fp16);
//   * sign terms are +-gamma_t with gamma_t the stored fp16 value;
//   * q', u' and the softmax weights p * nv are fp32, split into fp16 hi + lo
//     rows (rows 0..7 hi, 8..15 lo of the 16-row A operand), so the products
//     carry ~22 significant bits and the sums are fp32.
// Score tile:  D[16 rows = (head, hi|lo)][8 tokens] = sum over 8 coordinate
//   chunks (B = c[idx]) and 8 sign chunks (B = +-gamma) of A(q'|u') B.
// Value tile:  O[16 rows][8 coords] += P[16 rows][16 tokens] * V[16 tokens][8 coords],
//   P taken straight from the score accumulators' register layout.
// The packed layout is built for these fragments: a lane's codes for one
// token come as three words whose nibbles are prmt selectors into byte
// look-up tables of the fp16 centroids (lo bytes, hi bytes), and its sign
// bits come as one word shifted into the fp16 sign positions.  Value
// fragments are produced key-style and transposed in registers (movmatrix).
//
// Data movement: each warp owns a ring of STAGES shared-memory buffers of 32
// tokens (K codes, signs, norms, gammas, V codes, norms: six bulk copies,
// cp.async.bulk with an mbarrier transaction count, no multicast).  Waits are
// bounded: on timeout the kernel sets the handle's check word, waits (bounded)
// for its own copies, and contributes an empty partial.
#include <type_traits>

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kD = 128;
constexpr int kStages = 3;             // ring depth per warp
constexpr int kChunk = 32;             // tokens per stage
constexpr int kCodeB = 48;             // code bytes per token (d = 128)
constexpr int kSignB = 16;             // sign bytes per token
// stage layout (bytes)
constexpr int kOffKc = 0;
constexpr int kOffKs = kOffKc + kChunk * kCodeB;      // 1536
constexpr int kOffKn = kOffKs + kChunk * kSignB;      // 2048
constexpr int kOffKg = kOffKn + 2 * kChunk;           // 2112
constexpr int kOffVc = kOffKg + 2 * kChunk;           // 2176
constexpr int kOffVn = kOffVc + kChunk * kCodeB;      // 3712
constexpr int kStageB = kOffVn + 2 * kChunk;          // 3776
constexpr int kWaitLimit = 1 << 20;

static_assert(kStageB % 16 == 0, "stage must keep 16-byte alignment");

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
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    for (int i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
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

// ---------------------------------------------------------------- kernel
// Token-row orientation: each mma tile has 16 tokens on M and the (head,
// hi|lo) columns on N (NT n-tiles of 4 heads), so no M rows are wasted:
//   scores  S[16 tok][8] += Kdeq[16 tok][16 coords] * Q'[16 coords][8]   (8 coordinate chunks)
//                         + Sgn[16 tok][16 signs] * U'[16 signs][8]       (8 sign chunks)
//   values  O^T[16 coords][8] += Vdeq^T[16 coords][16 tok] * P[16 tok][8] (8 coordinate tiles)
// Lane (g, t) = (lane / 4, lane % 4) dequantises tokens g and g + 8 of each
// 16-token tile; its score columns are head t (hi, lo), so its softmax state
// and output rows belong to head t (and head 4 + t when NT = 2).
template <int NT, int NW>
__global__ void __launch_bounds__(NW * 32, 1) tq_decode_mma128_kernel(const DecArgs a, int G) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NW * kStages * kStageB);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, tq4 = lane & 3;
    uint8_t* ring = smem + (size_t)warp * kStages * kStageB;
    const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;

    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[b] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    const int64_t s0 = (int64_t)split * a.split_tokens;
    const int64_t s1 = (s0 + a.split_tokens < Tb) ? s0 + a.split_tokens : Tb;
    const int nchunk = s1 > s0 ? (int)((s1 - s0 + kChunk - 1) / kChunk) : 0;
    const int nmine = nchunk > warp ? (nchunk - warp + NW - 1) / NW : 0;
    const int64_t seq = (int64_t)b * a.Hkv + hkv;
    const int64_t kbb = block_bytes(kD, true), vbb = block_bytes(kD, false);

    if (lane == 0)
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[warp * kStages + s]), 1);
    fence_mbar_init();
    __syncwarp();

    auto issue = [&](int i) {
        const int64_t t0 = s0 + (int64_t)(warp + i * NW) * kChunk;     // multiple of 32
        const int64_t blk = seq * a.NB + (t0 >> 6);
        const int half = (int)((t0 >> 5) & 1);
        const uint8_t* kb = a.kc + blk * kbb;
        const uint8_t* vb = a.vc + blk * vbb;
        uint8_t* st = ring + (i % kStages) * kStageB;
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        mbar_expect_tx(bar, kStageB);
        bulk_g2s(smem_u32(st + kOffKc), kb + half * kChunk * kCodeB, kChunk * kCodeB, bar);
        bulk_g2s(smem_u32(st + kOffKs), kb + 64 * kCodeB + half * kChunk * kSignB, kChunk * kSignB, bar);
        bulk_g2s(smem_u32(st + kOffKn), kb + 64 * (kCodeB + kSignB) + half * 2 * kChunk, 2 * kChunk, bar);
        bulk_g2s(smem_u32(st + kOffKg), kb + 64 * (kCodeB + kSignB) + 128 + half * 2 * kChunk, 2 * kChunk, bar);
        bulk_g2s(smem_u32(st + kOffVc), vb + half * kChunk * kCodeB, kChunk * kCodeB, bar);
        bulk_g2s(smem_u32(st + kOffVn), vb + 64 * kCodeB + half * 2 * kChunk, 2 * kChunk, bar);
    };
    if (lane == 0) {
        for (int i = 0; i < kStages && i < nmine; ++i) issue(i);
    }
    pdl_wait();                           // q' and u' come from the prologue kernel

    // B operands (constant): column n = gr of n-tile nt is head 4 nt + gr / 2, limb gr % 2
    uint32_t bq[NT][8][2], bu[NT][8][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hcol = 4 * nt + (gr >> 1);
        const bool live = hcol < G;
        const int64_t bh = (int64_t)b * a.Hq + (int64_t)hkv * G + (live ? hcol : 0);
        const float* qp = a.qp + bh * kD;
        const float* up = a.up + bh * kD;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            const int c0 = 16 * kc + 2 * tq4;
            float x[4] = {0.f, 0.f, 0.f, 0.f}, y[4] = {0.f, 0.f, 0.f, 0.f};
            if (live) {
                x[0] = qp[c0]; x[1] = qp[c0 + 1]; x[2] = qp[c0 + 8]; x[3] = qp[c0 + 9];
                y[0] = up[c0]; y[1] = up[c0 + 1]; y[2] = up[c0 + 8]; y[3] = up[c0 + 9];
            }
            uint32_t h0, l0, h1, l1;
            split_hilo(x[0], x[1], h0, l0);
            split_hilo(x[2], x[3], h1, l1);
            bq[nt][kc][0] = (gr & 1) ? l0 : h0;
            bq[nt][kc][1] = (gr & 1) ? l1 : h1;
            split_hilo(y[0], y[1], h0, l0);
            split_hilo(y[2], y[3], h1, l1);
            bu[nt][kc][0] = (gr & 1) ? l0 : h0;
            bu[nt][kc][1] = (gr & 1) ? l1 : h1;
        }
    }
    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
    const uint32_t* pw = a.cb.pow2;

    float o[NT][8][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    float mrun[NT], lrun[NT], live[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        mrun[nt] = -INFINITY;
        lrun[nt] = 0.f;
        live[nt] = (4 * nt + tq4 < G) ? 1.f : 0.f;   // this lane's head exists
    }
    bool failed = false;

    for (int i = 0; i < nmine; ++i) {
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        if (!mbar_wait_bounded(bar, (uint32_t)((i / kStages) & 1))) {
            failed = true;
            if (lane == 0) atomicExch(a.err, 1);
            for (int j = i; j < nmine && j < i + kStages; ++j)
                mbar_wait_bounded(smem_u32(&bars[warp * kStages + (j % kStages)]), (uint32_t)((j / kStages) & 1));
            break;
        }
        const uint8_t* st = ring + (i % kStages) * kStageB;
        const int64_t tok0 = s0 + (int64_t)(warp + i * NW) * kChunk;
        const int nvalid = (int)((s1 - tok0) < kChunk ? (s1 - tok0) : kChunk);

        // one 16-token tile; PARTIAL masks tokens beyond nvalid (only the last
        // chunk of a split can be partial)
        auto tile = [&](const int kt, auto partial_tag) {
            constexpr bool PARTIAL = decltype(partial_tag)::value;
            const int tA = kt * 16 + gr, tB = tA + 8;            // this lane's two tokens
            // ---------------- scores
            uint32_t selA[4], selB[4];
            code_selectors(st + kOffKc + tA * kCodeB + tq4 * 12, pw, selA);
            code_selectors(st + kOffKc + tB * kCodeB + tq4 * 12, pw, selB);
            const uint32_t sgA = *reinterpret_cast<const uint32_t*>(st + kOffKs + tA * kSignB + tq4 * 4);
            const uint32_t sgB = *reinterpret_cast<const uint32_t*>(st + kOffKs + tB * kSignB + tq4 * 4);
            const uint32_t gA = *reinterpret_cast<const uint16_t*>(st + kOffKg + 2 * tA);
            const uint32_t gB = *reinterpret_cast<const uint16_t*>(st + kOffKg + 2 * tB);
            const uint32_t ggA = gA | (gA << 16), ggB = gB | (gB << 16);
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                uint32_t ka[4];
                dequant4(sel_for(selA, pw, kc), lut, ka[0], ka[2]);
                dequant4(sel_for(selB, pw, kc), lut, ka[1], ka[3]);
                uint32_t sa[4];
                // sign bit 1 -> +gamma: the pair (2kc | 2kc+1) of a slot sits at bits (q, 16 + q)
                sa[0] = ggA ^ (~shl_m(sgA, pw, 15 - 2 * kc) & 0x80008000u);
                sa[1] = ggB ^ (~shl_m(sgB, pw, 15 - 2 * kc) & 0x80008000u);
                sa[2] = ggA ^ (~shl_m(sgA, pw, 14 - 2 * kc) & 0x80008000u);
                sa[3] = ggB ^ (~shl_m(sgB, pw, 14 - 2 * kc) & 0x80008000u);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma16816(acc[nt], ka, bq[nt][kc][0], bq[nt][kc][1]);
                    mma16816(acc[nt], sa, bu[nt][kc][0], bu[nt][kc][1]);
                }
            }
            // ---------------- online softmax per head (this lane: head 4 nt + tq4)
            const float2 nkA = __half22float2(__halves2half2(*reinterpret_cast<const __half*>(st + kOffKn + 2 * tA),
                                                             *reinterpret_cast<const __half*>(st + kOffKn + 2 * tB)));
            float2 nv = __half22float2(__halves2half2(*reinterpret_cast<const __half*>(st + kOffVn + 2 * tA),
                                                      *reinterpret_cast<const __half*>(st + kOffVn + 2 * tB)));
            const bool okA = tA < nvalid, okB = tB < nvalid;
            if constexpr (PARTIAL) {
                if (!okA) nv.x = 0.f;
                if (!okB) nv.y = 0.f;
            }
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float sA = a.scale_log2 * nkA.x * (acc[nt][0] + acc[nt][1]);
                float sB = a.scale_log2 * nkA.y * (acc[nt][2] + acc[nt][3]);
                if constexpr (PARTIAL) {
                    if (!okA) sA = -INFINITY;
                    if (!okB) sB = -INFINITY;
                }
                float mt = fmaxf(sA, sB);
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 4));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 16));
                const float mnew = fmaxf(mrun[nt], mt);
                if (__any_sync(kFull, mnew > mrun[nt])) {   // a new running maximum
                    const float corr = (mnew == -INFINITY) ? 1.f : fast_exp2(mrun[nt] - mnew);
                    lrun[nt] *= corr;
#pragma unroll
                    for (int mt2 = 0; mt2 < 8; ++mt2) {
                        o[nt][mt2][0] *= corr; o[nt][mt2][1] *= corr; o[nt][mt2][2] *= corr; o[nt][mt2][3] *= corr;
                    }
                    mrun[nt] = mnew;
                }
                // mrun >= sA, sB here, so the exponent is <= 0 (masked: -inf -> 0)
                const float pA = fast_exp2(sA - mrun[nt]);
                const float pB = fast_exp2(sB - mrun[nt]);
                lrun[nt] += pA + pB;
                uint32_t hi, lo, xA, xB;
                split_hilo(pA * nv.x * live[nt], pB * nv.y * live[nt], hi, lo);
                // (hi, lo) of token A and of token B as the two columns of head tq4
                xA = __byte_perm(hi, lo, 0x5410);
                xB = __byte_perm(hi, lo, 0x7632);
                pb[nt][0] = movmatrix_t(xA);
                pb[nt][1] = movmatrix_t(xB);
            }
            // ---------------- values: O^T += Vdeq^T P
            code_selectors(st + kOffVc + tA * kCodeB + tq4 * 12, pw, selA);
            code_selectors(st + kOffVc + tB * kCodeB + tq4 * 12, pw, selB);
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                uint32_t x0, x1, y0, y1;
                dequant4(sel_for(selA, pw, kc), lut, x0, x1);      // token tA: coords 16kc+2t(+1), +8
                dequant4(sel_for(selB, pw, kc), lut, y0, y1);      // token tB
                const uint32_t va[4] = {movmatrix_t(x0), movmatrix_t(x1), movmatrix_t(y0), movmatrix_t(y1)};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(o[nt][kc], va, pb[nt][0], pb[nt][1]);
            }
        };
        if (nvalid == kChunk) {
            tile(0, std::false_type{});
            tile(1, std::false_type{});
        } else {
            tile(0, std::true_type{});
            if (nvalid > 16) tile(1, std::true_type{});
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nmine) {
            fence_proxy_async();
            issue(i + kStages);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        if (failed) { mrun[nt] = -INFINITY; lrun[nt] = 0.f; }
        lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 4);
        lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 8);
        lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 16);
    }

    pdl_trigger();                        // the combine kernel may start launching
    // ---------------- merge the warps of the CTA into one partial per head
    __syncwarp();
    float* wbuf = reinterpret_cast<float*>(ring);             // [G][kD + 2], in this warp's own ring
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + tq4;
        if (h < G) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                wbuf[h * (kD + 2) + 16 * mt + gr] = o[nt][mt][0] + o[nt][mt][1];
                wbuf[h * (kD + 2) + 16 * mt + 8 + gr] = o[nt][mt][2] + o[nt][mt][3];
            }
            if (gr == 0) {
                wbuf[h * (kD + 2) + kD] = mrun[nt];
                wbuf[h * (kD + 2) + kD + 1] = lrun[nt];
            }
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kD; idx += NW * 32) {
        const int g = idx / kD, j = idx % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, reinterpret_cast<const float*>(smem + (size_t)w * kStages * kStageB)[g * (kD + 2) + kD]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float* wb = reinterpret_cast<const float*>(smem + (size_t)w * kStages * kStageB) + g * (kD + 2);
                const float f = exp2f(wb[kD] - M);
                L = fmaf(f, wb[kD + 1], L);
                A = fmaf(f, wb[j], A);
            }
        }
        const int64_t bh = (int64_t)b * a.Hq + (int64_t)hkv * G + g;
        const int64_t pidx = bh * a.nsplit + split;
        a.part_acc[pidx * kD + j] = A;
        if (j == 0) {
            a.part_ml[2 * pidx] = M;
            a.part_ml[2 * pidx + 1] = L;
        }
    }
}

}  // namespace

constexpr int kNW1 = 16;   // warps per CTA, up to 4 heads per kv head (one n-tile)
constexpr int kNW2 = 8;    // warps per CTA, 8 heads per kv head (two n-tiles, more registers)

template <int NT, int NW>
cudaError_t launch_mma_t(const DecArgs& a, int G, cudaStream_t s) {
    const size_t smem = (size_t)NW * kStages * kStageB + (size_t)NW * kStages * 8;
    auto kern = tq_decode_mma128_kernel<NT, NW>;
    cudaError_t e = set_smem_once<tq_decode_mma128_kernel<NT, NW>>((int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.nsplit, (unsigned)a.Hkv, (unsigned)a.B);
    return launch_pdl(kern, grid, dim3(NW * 32), smem, s, a, G);
}

cudaError_t launch_decode_mma(int d, int G, const DecArgs& a, cudaStream_t s) {
    if (d != kD || G < 1 || G > 8) return cudaErrorInvalidValue;
    if (a.B * a.Hkv == 0) return cudaSuccess;
    return G <= 4 ? launch_mma_t<1, kNW1>(a, G, s) : launch_mma_t<2, kNW2>(a, G, s);
}

int decode_mma_chunk_tokens() { return kChunk; }
int decode_mma_warps(int G) { return G <= 4 ? kNW1 : kNW2; }

}  // namespace tqi
