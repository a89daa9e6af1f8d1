// Split-K decode attention over the packed TurboQuant cache for head_dim 128
// on the 5th-generation tensor cores (tcgen05, operands and accumulators in
// tensor memory), for sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com), hybrid V2+V3 section: dequantisation is
// fused into the attention kernel.  Per token t and query head g:
//   s = scale * n_t * (<q', c[idx_t]> + gamma_t * <u', 2 sigma_t - 1>),  u' = sqrt(pi/2)/m * S q'
//   acc += softmax weight * nv_t * c[idxv_t]   (rotated domain)
// (K section: 3-bit codes plus the 1-bit QJL residual correction; V section:
// 3-bit codes and the norm.)
//
// A CTA of eight warps walks its split in tiles of 128 tokens (two cache
// blocks, staged by bulk copies into a ring).  Warp w works on tensor-memory
// lanes 32 (w % 4) .. + 31 (row r = 32 (w % 4) + lane: a token of the tile, or
// a coordinate) and half w / 4 of that row's work.  Per tile:
//   * keys, two threads per token (two of its four code slots each): the
//     token's 128 codes become two signed
//     byte limbs of the exact integer c[idx] 2^14 (one prmt per limb per four
//     codes, from byte look-up tables) and its 128 sign bits the bytes
//     -128 sigma; the three byte rows go to tensor memory (tcgen05.st) as the
//     A operand of int8 mma with M = 128 tokens:
//       D_lo = K_lo Q^T, D_hi = K_hi Q^T  (Q: q' of each head as 24-bit fixed point, three byte limbs)
//       D_s  = Sgn U^T                    (U: u' as 16-bit fixed point, two byte limbs)
//     all sums exact in int32, so <q', c[idx]> carries the precision of the
//     fixed point of q' alone (2^-23 of its largest entry);
//   * values, two threads per coordinate (one cache block each): V blocks
//     hold one row per coordinate (the codes of its 64 tokens), so the thread
//     expands its row straight
//     into fp16 centroid pairs along tokens -- the A operand of
//       D_O = V^T P  (M = 128 coordinates, K = 128 tokens, fp16, fp32 accumulation)
//     with no transpose;
//   * softmax, two threads per token (two of the four heads each): the
//     scores from D_lo, D_hi and D_s, the online softmax per group of 32
//     tokens (each lane quarter's tokens of every tile form their own running
//     maximum and sum), and p * nv of each head as fp16 hi and lo limbs into
//     the B operand P (shared memory), in columns of its token group, so that
//     D_O keeps the four groups' sums apart;
//   * the coordinate threads fold D_O into fp32 register accumulators (two
//     heads each), rescaled by each group's running-maximum correction.
// The mma of each stage runs while the threads expand the next operand; the
// CTA's four token-group partials are merged at the end into one split-K
// partial per head, as the decode's combine kernel expects.  Up to 4 query
// heads per CTA (kv heads with more are served by ceil(G / 4) CTAs); two CTAs
// per SM.
//
// Every wait is bounded: a wait that runs out sets the check word, every
// thread stops at the next barrier, the CTA waits (bounded) for its own
// copies and mma still in flight, releases its tensor memory and contributes
// an empty partial.
#include <type_traits>

#include "tq_frag.cuh"
#include "tq_tc.cuh"

namespace tqi {
namespace {

constexpr int kTD = 128;                 // head_dim
constexpr int kTT = 128;                 // tokens per tile (two cache blocks)
constexpr int kTH = 4;                   // query heads per CTA
constexpr int kTRing = 4;                // ring stages
constexpr int kNq = 16;                  // D_lo / D_hi columns: three q' limbs per head
constexpr int kNu = 16;                  // D_s columns: two u' limbs per head
constexpr int kNo = 8 * kTH;             // D_O columns: (warp, head, limb)
constexpr float kQScale = 8000000.f;     // q' fixed point: |q_int| <= 8e6 < 2^23
constexpr float kUScale = 32000.f;       // u' fixed point

template <bool QJL>
struct TcShape {
    static constexpr int kKB = 64 * 48 + (QJL ? 64 * 16 + 256 : 128);    // K block bytes
    static constexpr int kVB = kTD * kVRowB + 128;                        // V block bytes (code rows)
    static constexpr int kStage = 2 * (kKB + kVB);
    // tensor-memory columns
    static constexpr int kColAK = 0;                        // K operand: lo limbs, hi limbs, signs (32 each)
    static constexpr int kColAV = QJL ? 96 : 64;            // V operand (64)
    static constexpr int kColDlo = kColAV + 64;
    static constexpr int kColDhi = kColDlo + kNq;
    static constexpr int kColDs = kColDhi + kNq;
    static constexpr int kColDo = kColDs + (QJL ? kNu : 0);
    static constexpr int kCols = kColDo + kNo;
    static constexpr int kAlloc = 256;
    static_assert(kCols <= kAlloc, "tensor memory per CTA");
    // shared memory (offsets from a 1024-byte aligned base)
    static constexpr int kOffBq = 0;                        // 16 rows x 128 B, swizzled
    static constexpr int kOffBu = kOffBq + kNq * 128;
    static constexpr int kOffBp = kOffBu + kNu * 128;       // 32 rows x 256 B: two halves of 4 KB
    static constexpr int kOffRing = kOffBp + 2 * kNo * 128;
    static constexpr int kOffBar = kOffRing + kTRing * kStage;
    static constexpr int kOffMisc = kOffBar + 8 * (kTRing + 2);
    // + slack to align the base; at least 100 KB, so that two CTAs share an SM
    // (their two 256-column tensor-memory allocations fill it) and never three
    static constexpr int kSmemUsed = kOffMisc + 512 + 1024;
    static constexpr int kSmem = kSmemUsed > 100 * 1024 ? kSmemUsed : 100 * 1024;
    static_assert(2 * kSmem <= 227 * 1024 && 3 * kSmem > 228 * 1024, "two CTAs per SM");
};

// ---------------------------------------------------------------- kernel
constexpr int kTThreads = 256;

template <bool QJL>
__global__ void __launch_bounds__(kTThreads, 2) tq_decode_tc_kernel(const DecArgs a, int G) {
    using S = TcShape<QJL>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);       // ring [kTRing], K mma, V mma
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffMisc);
    float* sRed = reinterpret_cast<float*>(sm + S::kOffMisc + 16);       // [2 halves][4 groups][kTH]
    float* sFac = reinterpret_cast<float*>(sm + S::kOffMisc + 144);      // [kTH][3] fQ, fU, uS
    // [tile parity][4 groups][kTH]: a warp writes tile k's corrections while
    // another may still fold tile k - 1 with the other half
    float* sCorr = reinterpret_cast<float*>(sm + S::kOffMisc + 192);
    float* sML = reinterpret_cast<float*>(sm + S::kOffMisc + 320);       // [4 groups][kTH][2]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, hh = warp >> 2;                  // lane quarter, half of the row's work
    const int r = 32 * quad + lane;                             // token of the tile / coordinate
    const int split = blockIdx.x, b = blockIdx.z;
    const int hgroups = (G + kTH - 1) / kTH;
    const int hkv = blockIdx.y / hgroups;
    const int g0 = (blockIdx.y - hkv * hgroups) * kTH;
    const int Gl = G - g0 < kTH ? G - g0 : kTH;               // live query heads of this CTA
    const int64_t hbase = (int64_t)b * a.Hq + (int64_t)hkv * G + g0;
    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[b] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    const int64_t s0 = (int64_t)split * a.split_tokens;
    const int64_t s1 = (s0 + a.split_tokens < Tb) ? s0 + a.split_tokens : Tb;
    const int ntile = s1 > s0 ? (int)((s1 - s0 + kTT - 1) / kTT) : 0;
    const int64_t seq = (int64_t)b * a.Hkv + hkv;
    const uint32_t bar_k = smem_u32(&bars[kTRing]), bar_v = smem_u32(&bars[kTRing + 1]);

    if (tid == 0) {
        for (int s = 0; s < kTRing + 2; ++s) mbar_init(smem_u32(&bars[s]), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), S::kAlloc);
        tc_relinquish();
    }
    // B operands start as zeros (rows of absent heads, other groups' P columns)
    for (int i = tid; i < S::kOffRing / 16; i += kTThreads) reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);

    // tile k's blocks -> ring stage k % kTRing: [K block 0][K block 1][V block 0][V block 1];
    // a block starting at or beyond the split end is not copied
    auto issue = [&](int k) {
        const int64_t t0 = s0 + (int64_t)k * kTT;
        uint8_t* st = sm + S::kOffRing + (k % kTRing) * S::kStage;
        const uint32_t bar = smem_u32(&bars[k % kTRing]);
        const int nb = (t0 + 64 < s1) ? 2 : 1;
        mbar_expect_tx(bar, (uint32_t)(nb * (S::kKB + S::kVB)));
        for (int bi = 0; bi < nb; ++bi) {
            const int64_t lb = (t0 >> 6) + bi;
            const int64_t kblk = cache_block(a.ktable, a.kpool, a.NB, seq, lb, a.err);
            const int64_t vblk = cache_block(a.vtable, a.vpool, a.NB, seq, lb, a.err);
            bulk_g2s(smem_u32(st + bi * S::kKB), a.kc + (kblk >= 0 ? kblk : 0) * S::kKB, S::kKB, bar);
            bulk_g2s(smem_u32(st + 2 * S::kKB + bi * S::kVB), a.vc + (vblk >= 0 ? vblk : 0) * S::kVB, S::kVB, bar);
        }
    };
    // tiles holding tokens that a chained encode writes are fetched only after pdl_wait
    auto fresh = [&](int k) {
        const int64_t t0 = s0 + (int64_t)k * kTT;
        return t0 < a.fresh_hi && a.fresh_lo < t0 + kTT;
    };
    if (tid == 0)
        for (int k = 0; k < kTRing && k < ntile; ++k)
            if (!fresh(k)) issue(k);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tlane = tmem + ((uint32_t)(32 * quad) << 16);      // this warp's lanes

    pdl_wait();                                  // q' and u' come from the prologue kernel
    if (tid == 0) {
        bool any = false;
        for (int k = 0; k < kTRing && k < ntile; ++k) any |= fresh(k);
        if (any) {
            asm volatile("fence.proxy.async;" ::: "memory");
            for (int k = 0; k < kTRing && k < ntile; ++k)
                if (fresh(k)) issue(k);
        }
    }

    // ---- B operands of the score products: the first half's threads take
    // coordinate r of q', the second half's JL row r of u'.  K position of
    // coordinate r in the key operand: 32 t + p (slot t, slot position p of the
    // token record); of JL row r in the sign operand: 32 t + 4 k + e where the
    // row's sign is bit 8 e + 7 - k of sign word t.
    {
        const int t = slot_of(r), p = slot_pos(r);
        const int kq = 32 * t + p;
        const int l = (p & 1) ? 16 + (p >> 1) : (p >> 1);
        const int ks = 32 * t + 4 * (7 - (l & 7)) + (l >> 3);
        const float* src = hh == 0 ? a.qp : a.up;
        float v[kTH], m[kTH];
#pragma unroll
        for (int h = 0; h < kTH; ++h) {
            v[h] = (h < Gl && (QJL || hh == 0)) ? src[(hbase + h) * kTD + r] : 0.f;
            m[h] = fabsf(v[h]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(kFull, m[h], o));
        }
        if (lane == 0)
#pragma unroll
            for (int h = 0; h < kTH; ++h) sRed[(hh * 4 + quad) * kTH + h] = m[h];
        __syncthreads();
        int usum[kTH];
#pragma unroll
        for (int h = 0; h < kTH; ++h) {
            float mx = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) mx = fmaxf(mx, sRed[(hh * 4 + w) * kTH + h]);
            const float f = mx > 0.f ? (hh == 0 ? kQScale : kUScale) / mx : 0.f;
            const int vi = __float2int_rn(v[h] * f);
            usum[h] = 0;
            if (hh == 0) {
                const int c0 = ((vi + 128) & 255) - 128;
                const int r1 = (vi - c0) >> 8;
                const int c1 = ((r1 + 128) & 255) - 128;
                const int c2 = (r1 - c1) >> 8;
                sm[S::kOffBq + sw128_byte(3 * h + 0, kq, kNq)] = (uint8_t)(int8_t)c0;
                sm[S::kOffBq + sw128_byte(3 * h + 1, kq, kNq)] = (uint8_t)(int8_t)c1;
                sm[S::kOffBq + sw128_byte(3 * h + 2, kq, kNq)] = (uint8_t)(int8_t)c2;
                if (tid == 0) sFac[3 * h + 0] = mx > 0.f ? a.scale_log2 * a.cb.iscale / f : 0.f;
            } else if (QJL) {
                const int lo = ((vi + 128) & 255) - 128;
                sm[S::kOffBu + sw128_byte(2 * h + 0, ks, kNu)] = (uint8_t)(int8_t)((vi - lo) >> 8);
                sm[S::kOffBu + sw128_byte(2 * h + 1, ks, kNu)] = (uint8_t)(int8_t)lo;
                usum[h] = vi;
                if (tid == 128) sFac[3 * h + 1] = mx > 0.f ? a.scale_log2 / f : 0.f;
            }
        }
        if constexpr (QJL) {
#pragma unroll
            for (int h = 0; h < kTH; ++h)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) usum[h] += __shfl_xor_sync(kFull, usum[h], o);
            if (hh == 1 && lane == 0)
#pragma unroll
                for (int h = 0; h < kTH; ++h) reinterpret_cast<int*>(sCorr)[quad * kTH + h] = usum[h];
            __syncthreads();
            if (tid < kTH) {
                int sum = 0;
#pragma unroll
                for (int w = 0; w < 4; ++w) sum += reinterpret_cast<int*>(sCorr)[w * kTH + tid];
                sFac[3 * tid + 2] = (float)sum;
            }
        }
        fence_proxy_async();                     // B operands written by threads, read by the tensor core
        __syncthreads();
    }
    // this thread's two heads: hh * 2 + {0, 1}
    constexpr int kHH = kTH / 2;
    float fQ[kHH], fU[kHH], uS[kHH];
#pragma unroll
    for (int hl = 0; hl < kHH; ++hl) {
        const int h = kHH * hh + hl;
        fQ[hl] = sFac[3 * h];
        fU[hl] = sFac[3 * h + 1];
        uS[hl] = QJL ? sFac[3 * h + 2] : 0.f;
    }

    const uint32_t ilut[4] = {a.cb.ilut_lo[0], a.cb.ilut_lo[1], a.cb.ilut_hi[0], a.cb.ilut_hi[1]};
    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
    const uint32_t* pw = a.cb.pow2;
    constexpr uint32_t kIdQ = idesc_i8(128, kNq), kIdU = idesc_i8(128, kNu), kIdO = idesc_f16(128, kNo);
    // token r of a tile: block bi, row tau; its K position in P; this thread's
    // four P entries (two heads x hi, lo limbs)
    const int bi = r >> 6, tau = r & 63;
    const int kp = 64 * bi + 16 * (tau >> 4) + 4 * slot_of(tau) + 2 * ((tau >> 3) & 1) + (tau & 1);
    uint32_t poff[kHH][2];
#pragma unroll
    for (int hl = 0; hl < kHH; ++hl)
#pragma unroll
        for (int lb = 0; lb < 2; ++lb)
            poff[hl][lb] = S::kOffBp + sw128_byte((quad * kTH + kHH * hh + hl) * 2 + lb, 2 * kp, kNo);

    float o[4][kHH];                             // coordinate r, per token group and own head
    float mrun[kHH], lrun[kHH];                  // this group's running max (uniform) and this thread's sum
#pragma unroll
    for (int hl = 0; hl < kHH; ++hl) {
        mrun[hl] = -INFINITY;
        lrun[hl] = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) o[w][hl] = 0.f;
    }
    int nk_issued = 0, nk_seen = 0, nv_issued = 0, nv_seen = 0, n_issued = ntile < kTRing ? ntile : kTRing;
    bool failed = false;

    // fold tile kk's D_O into the accumulators (HH: this thread's half, a
    // compile-time constant so that the loaded columns stay in registers)
    auto fold_half = [&](int kk, auto hh_c) {
        constexpr int HH = decltype(hh_c)::value;
        uint32_t dv[kNo];
        tc_ld32(tlane + S::kColDo, dv);
        const float* corr = sCorr + (kk & 1) * 4 * kTH;
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int hl = 0; hl < kHH; ++hl) {
                constexpr int kBase = kHH * HH;
                const int col = (w * kTH + kBase + hl) * 2;
                o[w][hl] = fmaf(o[w][hl], corr[w * kTH + kBase + hl],
                                __uint_as_float(dv[col]) + __uint_as_float(dv[col + 1]));
            }
    };
    auto fold_o = [&](int kk) {
        if (hh == 0) fold_half(kk, std::integral_constant<int, 0>{});
        else fold_half(kk, std::integral_constant<int, 1>{});
    };

    for (int k = 0; k < ntile; ++k) {
        const uint8_t* st = sm + S::kOffRing + (k % kTRing) * S::kStage;
        const int64_t tk0 = s0 + (int64_t)k * kTT;
        // (bad is kept warp-uniform: the tensor-memory loads and stores below are warp-collective)
        bool bad = __any_sync(kFull, !mbar_wait_bounded(smem_u32(&bars[k % kTRing]), (uint32_t)((k / kTRing) & 1),
                                                        k == 0 ? a.first_wait : kWaitLimit));
        // ---------------- keys: slots 2 hh, 2 hh + 1 of token r -> tensor memory
        const uint8_t* kb = st + bi * S::kKB;
        float nk = 0.f, gk = 0.f;
        if (!bad) {
            const uint2* cw = reinterpret_cast<const uint2*>(kb + tau * 48 + 24 * hh);
            const uint2 c0 = cw[0], c1 = cw[1], c2 = cw[2];
            const uint32_t w6[6] = {c0.x, c0.y, c1.x, c1.y, c2.x, c2.y};
            uint2 sg2 = make_uint2(0u, 0u);
            if constexpr (QJL) sg2 = *reinterpret_cast<const uint2*>(kb + 64 * 48 + tau * 16 + 8 * hh);
            const uint32_t sgw[2] = {sg2.x, sg2.y};
            uint32_t lo[16], hi[16];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t sel[4];
                sel[0] = w6[3 * tt] & 0x77777777u;
                sel[1] = w6[3 * tt + 1] & 0x77777777u;
                sel[2] = w6[3 * tt + 2] & 0x77777777u;
                sel[3] = ((w6[3 * tt] >> 3) & 0x11111111u) | ((w6[3 * tt + 1] >> 2) & 0x22222222u) |
                         ((w6[3 * tt + 2] >> 1) & 0x44444444u);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint32_t s_lo = sel[s], s_hi = sel[s] >> 16;
                    lo[8 * tt + 2 * s] = __byte_perm(ilut[0], ilut[1], s_lo);
                    lo[8 * tt + 2 * s + 1] = __byte_perm(ilut[0], ilut[1], s_hi);
                    hi[8 * tt + 2 * s] = __byte_perm(ilut[2], ilut[3], s_lo);
                    hi[8 * tt + 2 * s + 1] = __byte_perm(ilut[2], ilut[3], s_hi);
                }
            }
            tc_st16(tlane + S::kColAK + 16 * hh, lo);
            tc_st16(tlane + S::kColAK + 32 + 16 * hh, hi);
            if constexpr (QJL) {
                uint32_t sb[16];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int q = 0; q < 8; ++q) sb[8 * tt + q] = shl_m(sgw[tt], pw, q) & 0x80808080u;
                tc_st16(tlane + S::kColAK + 64 + 16 * hh, sb);
            }
            const __half* kn = reinterpret_cast<const __half*>(kb + (QJL ? 64 * 64 : 64 * 48));
            nk = __half2float(kn[tau]);
            if constexpr (QJL) gk = __half2float(kn[64 + tau]);
        }
        tc_wait_st();
        tc_fence_before();
        if (__syncthreads_or(bad)) { failed = true; break; }
        if (tid == 0) {
            tc_fence_after();
            const uint32_t bq = sbase + S::kOffBq, bu = sbase + S::kOffBu;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                tc_mma_i8_ts(tmem + S::kColDlo, tmem + S::kColAK + 8 * s, sw128_desc(bq + 32 * s), kIdQ, s > 0);
                tc_mma_i8_ts(tmem + S::kColDhi, tmem + S::kColAK + 32 + 8 * s, sw128_desc(bq + 32 * s), kIdQ, s > 0);
                if constexpr (QJL)
                    tc_mma_i8_ts(tmem + S::kColDs, tmem + S::kColAK + 64 + 8 * s, sw128_desc(bu + 32 * s), kIdU, s > 0);
            }
            tc_commit(bar_k);
        }
        ++nk_issued;
        // ---------------- values: the previous tile's D_O, then coordinate r's row of block hh
        if (k > 0) {
            const bool okv = mbar_wait_bounded(bar_v, (uint32_t)(nv_seen & 1));
            nv_seen += okv ? 1 : 0;
            bad = __any_sync(kFull, bad || !okv);
            if (!bad) {
                tc_fence_after();
                fold_o(k - 1);
            }
        }
        if (!bad) {
            const uint2* rp = reinterpret_cast<const uint2*>(st + 2 * S::kKB + hh * S::kVB + r * kVRowB);
            const uint2 r0 = rp[0], r1 = rp[1], r2 = rp[2];
            const uint32_t W[6] = {r0.x, r0.y, r1.x, r1.y, r2.x, r2.y};
            uint32_t x[32];                          // column 8 q + 2 t + half: tokens 16 q + 2 t + 8 half + {0, 1}
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t w = W[t], hw = (W[4 + (t >> 1)] >> (16 * (t & 1))) & 0xFFFFu;
                const uint32_t m = w & 0x77777777u;
                const uint32_t sel[4] = {m, m >> 16, hw & 0x7777u,
                                         ((w >> 3) & 0x1111u) | ((w >> 18) & 0x2222u) | ((hw >> 1) & 0x4444u)};
#pragma unroll
                for (int q = 0; q < 4; ++q) dequant4(sel[q], lut, x[8 * q + 2 * t], x[8 * q + 2 * t + 1]);
            }
            uint32_t x16[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) x16[c] = x[c];
            tc_st16(tlane + S::kColAV + 32 * hh, x16);
#pragma unroll
            for (int c = 0; c < 16; ++c) x16[c] = x[16 + c];
            tc_st16(tlane + S::kColAV + 32 * hh + 16, x16);
        }
        // ---------------- scores and softmax: token r, heads 2 hh, 2 hh + 1
        const bool okk = mbar_wait_bounded(bar_k, (uint32_t)(nk_seen & 1));
        nk_seen += okk ? 1 : 0;
        bad = __any_sync(kFull, bad || !okk);
        auto softmax_half = [&](auto hh_c) {
            constexpr int HH = decltype(hh_c)::value;
            uint32_t dlo[16], dhi[16];
            [[maybe_unused]] uint32_t ds[16];
            tc_ld16(tlane + S::kColDlo, dlo);
            tc_ld16(tlane + S::kColDhi, dhi);
            if constexpr (QJL) tc_ld16(tlane + S::kColDs, ds);
            const bool valid = tk0 + r < s1;
            const float nv = __half2float(
                reinterpret_cast<const __half*>(st + 2 * S::kKB + bi * S::kVB + kTD * kVRowB)[tau]);
#pragma unroll
            for (int hl = 0; hl < kHH; ++hl) {
                const int h = kHH * HH + hl;
                const int X0 = (int)dlo[3 * h], X1 = (int)dlo[3 * h + 1], X2 = (int)dlo[3 * h + 2];
                const int Y0 = (int)dhi[3 * h], Y1 = (int)dhi[3 * h + 1], Y2 = (int)dhi[3 * h + 2];
                const int T1 = 256 * Y2 + X2 + Y1;
                const int T2 = 256 * (X1 + Y0) + X0;
                float sc = fQ[hl] * fmaf(65536.f, (float)T1, (float)T2);
                if constexpr (QJL) {
                    const int Z = 256 * (int)ds[2 * h] + (int)ds[2 * h + 1];
                    sc = fmaf(gk * fU[hl], fmaf((float)Z, -1.f / 64.f, -uS[hl]), sc);
                }
                sc = (valid && h < Gl) ? sc * nk : -INFINITY;
                // this group's maximum over its 32 tokens (order-preserving integer image of the floats)
                const int ib = __float_as_int(sc);
                const int key = ib ^ ((ib >> 31) & 0x7FFFFFFF);
                const int mk = __reduce_max_sync(kFull, key);
                const float tmax = __int_as_float(mk ^ ((mk >> 31) & 0x7FFFFFFF));
                const float mnew = fmaxf(mrun[hl], tmax);
                const float corr = (mnew == -INFINITY) ? 1.f : fast_exp2(mrun[hl] - mnew);
                const float pr = (sc == -INFINITY) ? 0.f : fast_exp2(sc - mnew);
                lrun[hl] = fmaf(lrun[hl], corr, pr);
                mrun[hl] = mnew;
                const float pv = valid ? pr * nv : 0.f;
                const __half hp = __float2half_rn(pv);
                const __half lp = __float2half_rn(pv - __half2float(hp));
                *reinterpret_cast<__half*>(sm + poff[hl][0]) = hp;
                *reinterpret_cast<__half*>(sm + poff[hl][1]) = lp;
                if (lane == 0) sCorr[(k & 1) * 4 * kTH + quad * kTH + h] = corr;
            }
        };
        if (!bad) {
            tc_fence_after();
            if (hh == 0) softmax_half(std::integral_constant<int, 0>{});
            else softmax_half(std::integral_constant<int, 1>{});
        }
        fence_proxy_async();                     // P written by threads, read by the tensor core
        tc_wait_st();
        tc_fence_before();
        if (__syncthreads_or(bad)) { failed = true; break; }
        if (tid == 0) {
            tc_fence_after();
            const uint32_t bp = sbase + S::kOffBp;
#pragma unroll
            for (int s = 0; s < kTT / 16; ++s)
                tc_mma_f16_ts(tmem + S::kColDo, tmem + S::kColAV + 8 * s,
                              sw128_desc(bp + (s >> 2) * (kNo * 128) + (s & 3) * 32), kIdO, s > 0);
            tc_commit(bar_v);
            if (k + kTRing < ntile) {
                fence_proxy_async();
                issue(k + kTRing);
            }
        }
        ++nv_issued;
        if (k + kTRing < ntile) ++n_issued;
    }
    if (!failed && nv_seen < nv_issued) {        // the last tile's D_O
        const bool ok = mbar_wait_bounded(bar_v, (uint32_t)(nv_seen & 1));
        nv_seen += ok ? 1 : 0;
        if (__syncthreads_or(!ok)) {
            failed = true;
        } else {
            tc_fence_after();
            fold_o(ntile - 1);
        }
    }
    if (failed) {
        if (tid == 0) atomicExch(a.err, 1);
        // wait (bounded) for this CTA's mma and copies still in flight
        for (; nk_seen < nk_issued; ++nk_seen) mbar_wait_bounded(bar_k, (uint32_t)(nk_seen & 1));
        for (; nv_seen < nv_issued; ++nv_seen) mbar_wait_bounded(bar_v, (uint32_t)(nv_seen & 1));
        for (int k = 0; k < n_issued; ++k) mbar_wait_bounded(smem_u32(&bars[k % kTRing]), (uint32_t)((k / kTRing) & 1));
    }
    pdl_trigger();                               // the combine kernel may start launching
    // ---------------- merge the four token groups' partials of every head
#pragma unroll
    for (int hl = 0; hl < kHH; ++hl) {
        float l = lrun[hl];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFull, l, off);
        if (lane == 0) {
            const int h = kHH * hh + hl;
            sML[(quad * kTH + h) * 2] = failed ? -INFINITY : mrun[hl];
            sML[(quad * kTH + h) * 2 + 1] = failed ? 0.f : l;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, S::kAlloc);
    }
#pragma unroll
    for (int hl = 0; hl < kHH; ++hl) {
        const int h = kHH * hh + hl;
        if (h >= Gl) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sML[(w * kTH + h) * 2]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = sML[(w * kTH + h) * 2];
                if (mw == -INFINITY) continue;
                const float f = exp2f(mw - M);
                L = fmaf(f, sML[(w * kTH + h) * 2 + 1], L);
                A = fmaf(f, o[w][hl], A);
            }
        }
        const int64_t pidx = (hbase + h) * a.nsplit + split;
        a.part_acc[pidx * kTD + r] = A;
        if (r == 0) {
            a.part_ml[2 * pidx] = M;
            a.part_ml[2 * pidx + 1] = L;
        }
    }
}

}  // namespace

constexpr int kTcHeads = kTH;

template <bool QJL>
cudaError_t launch_tc_q(int G, const DecArgs& a, cudaStream_t s) {
    constexpr int smem = TcShape<QJL>::kSmem;
    cudaError_t e = set_smem_once<tq_decode_tc_kernel<QJL>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.nsplit, (unsigned)(a.Hkv * ((G + kTcHeads - 1) / kTcHeads)), (unsigned)a.B);
    return launch_pdl(tq_decode_tc_kernel<QJL>, grid, dim3(kTThreads), smem, s, a, G);
}

cudaError_t launch_decode_tc(int d, int G, bool qjl, const DecArgs& a, cudaStream_t s) {
    if (d != kTD || G < 1) return cudaErrorInvalidValue;
    if (a.B * a.Hkv == 0) return cudaSuccess;
    return qjl ? launch_tc_q<true>(G, a, s) : launch_tc_q<false>(G, a, s);
}

int decode_tc_heads() { return kTcHeads; }
int decode_tc_tile_tokens() { return kTT; }

}  // namespace tqi
