// Tensor-core split-K decode attention over the packed TurboQuant cache
// (head_dim 64, 128 or 256, up to 8 query heads per kv head), for sm_100a.
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
//   * sign terms run on int8 mma (m16n8k32): each sign bit becomes an operand
//     byte -128 sigma, u' is 16-bit fixed point per head in two byte limbs, the
//     products accumulate exactly in int32 and gamma_t scales the sum;
//   * q' and the softmax weights p * nv are fp32, split into fp16 hi + lo
//     columns, so the products carry ~22 significant bits and the sums are
//     fp32.
// The packed layout is built for these fragments: a lane's codes for one
// token come as three words whose nibbles are prmt selectors into byte
// look-up tables of the fp16 centroids (lo bytes, hi bytes), and its sign
// bits come as one word of which a shift and a mask keep four signs, one per
// operand byte.  Value fragments are produced key-style and transposed in
// registers (movmatrix).
//
// Data movement: each warp owns a ring of STAGES shared-memory buffers of a
// chunk of tokens (32 at d = 128, 16 at d = 256; K codes, signs, norms,
// gammas, V codes, norms: six bulk copies, cp.async.bulk with an mbarrier
// transaction count, no multicast).  Waits are bounded: on timeout the kernel
// sets the handle's check word, waits (bounded) for its own copies, and
// contributes an empty partial.
//
// head_dim 256 is two 128-coordinate slices of the same record layout: the
// k-loop runs over 16 coordinate chunks and 8 sign blocks, the value tile
// over 16 coordinate tiles.  Its q'/u' fragments are read from shared memory
// (filled once per CTA) instead of being held in registers.  head_dim 64 is
// half a slice: 16 codes and 16 signs per slot (4 k-steps, 2 sign blocks),
// its sign halfword widened so that the same shifts pick its bits.
#include <type_traits>

#include "tq_frag.cuh"

namespace tqi {
namespace {

// ---------------------------------------------------------------- kernel
constexpr int kTabMax = 512;   // block-table entries of a split staged in shared memory (32768 tokens)

// Pool block of a paged cache from the staged table slice (contiguous cache:
// the logical block index); an entry outside the pool sets the check word and
// gives -1, as cache_block does.
__device__ __forceinline__ int64_t staged_block(const int32_t* table, const int32_t* st, int64_t pool,
                                                int64_t contiguous, int i, int* err) {
    if (!table) return contiguous;
    const int32_t p = st[i];
    if (p < 0 || (int64_t)p >= pool) {
        atomicExch(err, 1);
        return -1;
    }
    return p;
}
// Warps given to the first of two units sharing a stream-K CTA (nA and nB
// chunks): the split with the fewest chunk-steps for the slower group.
template <int NW>
__device__ __forceinline__ int streamk_split(int64_t nA, int64_t nB) {
    int best = 1;
    int64_t bt = INT64_MAX;
    for (int k = 1; k < NW; ++k) {
        const int64_t ta = (nA + k - 1) / k, tb = (nB + NW - k - 1) / (NW - k);
        const int64_t t = ta > tb ? ta : tb;
        if (t < bt) { bt = t; best = k; }
    }
    return best;
}

// Token-row orientation: each mma tile has 16 tokens on M and the (head,
// hi|lo) columns on N (NT n-tiles of 4 heads), so no M rows are wasted:
//   scores  S[16 tok][8] += Kdeq[16 tok][16 coords] * Q'[16 coords][8]   (D/16 coordinate chunks, fp16)
//           Z[16 tok][8]  += Sgn[16 tok][32 signs] * U'[32 signs][8]      (D/32 sign blocks, int8)
//   values  O^T[16 coords][8] += Vdeq^T[16 coords][16 tok] * P[16 tok][8] (D/16 coordinate tiles)
// Lane (g, t) = (lane / 4, lane % 4) dequantises tokens g and g + 8 of each
// 16-token tile; its score columns are head t (hi, lo), so its softmax state
// and output rows belong to head t (and head 4 + t when NT = 2).  A kv head
// with more than 8 query heads is served by ceil(G / 8) CTAs (grid.y = Hkv x
// head groups), each taking up to 8 of its query heads.
template <int D, int NT, int NW, bool QJL>
__global__ void __launch_bounds__(NW * 32, 1) tq_decode_mma_kernel(const DecArgs a, int G) {
    using C = Cfg<D, QJL>;
    constexpr int kKC = C::kKC;
    constexpr int kSBGroup = 2 * NT * kKC * 32;   // uint2 entries of one group's q'/u' fragments (d = 256)
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NW * kStages * C::kStageB);
    // per-warp (max, sum) of each head for the merge: [NW][8][2]
    float* sML = reinterpret_cast<float*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8);
    // d = 256: q'/u' fragments per (operand, n-tile, k-step, lane), filled once per CTA
    // paged caches: the split's slice of the K and V block tables, [2][kTabMax]
    int32_t* sTab = reinterpret_cast<int32_t*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                                               (size_t)NW * 8 * 2 * sizeof(float));
    uint2* sB = reinterpret_cast<uint2*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                                         (size_t)NW * 8 * 2 * sizeof(float) + 2 * kTabMax * sizeof(int32_t));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, tq4 = lane & 3;
    uint8_t* ring = smem + (size_t)warp * kStages * C::kStageB;
    const int hgroups = (G + 7) >> 3;

    // ---------------- this CTA's work: one or two (unit, token range) groups.
    // A unit is (batch, kv head, query-head group).  Uniform split grid: one
    // group, unit (blockIdx.z, blockIdx.y), split blockIdx.x.  Stream-K: the
    // CTA's chunk range lies in at most two units; its warps are divided
    // between them in proportion to their chunks (warps [0, kA) and [kA, NW)),
    // and each group writes one partial slot of its unit: slot c - (first CTA
    // of the unit).  The CTA holding a unit's last chunk also writes the
    // unit's unused slots as empty partials.
    int ngrp = 1, kA = NW;
    int64_t unitA = 0, s0A = 0, s1A = 0, unitB = 0, s0B = 0, s1B = 0;   // group 0 (A) and group 1 (B)
    int slotA = 0, slotB = 0;
    bool endA = false, endB = false;
    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[blockIdx.z] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    if (a.sk_ctas == 0) {
        unitA = (int64_t)blockIdx.z * a.Hkv * hgroups + blockIdx.y;
        s0A = (int64_t)blockIdx.x * a.split_tokens;
        s1A = (s0A + a.split_tokens < Tb) ? s0A + a.split_tokens : Tb;
        slotA = blockIdx.x;
    } else {
        const int64_t N = a.sk_total, nck = a.sk_nck, nC = a.sk_ctas, c = blockIdx.x;
        const int64_t lo = c * N / nC, hi = (c + 1) * N / nC;
        const int64_t u0 = lo / nck, u1 = (hi - 1) / nck;
        const int64_t cut = (u0 + 1) * nck < hi ? (u0 + 1) * nck : hi;
        auto tok = [&](int64_t x, int64_t u) {                 // chunk x of unit u as a token bound
            const int64_t t = (x - u * nck) * C::kChunk;
            return t < Tb ? t : Tb;
        };
        auto first_cta = [&](int64_t u) { return (int)(((u * nck + 1) * nC - 1) / N); };
        unitA = u0;
        s0A = tok(lo, u0);
        s1A = tok(cut, u0);
        slotA = (int)c - first_cta(u0);
        endA = cut == (u0 + 1) * nck;
        if (u1 != u0) {
            kA = streamk_split<NW>(cut - lo, hi - cut);
            ngrp = 2;
            unitB = u1;
            s0B = tok(cut, u1);
            s1B = tok(hi, u1);
            slotB = (int)c - first_cta(u1);
            endB = hi == (u1 + 1) * nck;
        }
    }
    const int grp = warp < kA ? 0 : 1;
    const int wi = grp ? warp - kA : warp;                     // this warp among its group's
    const int nw = grp ? NW - kA : kA;
    auto unit_rows = [&](int g, int64_t& hb, int& gl, int64_t& sq) {
        const int64_t u = g ? unitB : unitA;
        const int64_t bk = u / hgroups;                          // b * Hkv + kv head
        const int hg = (int)(u - bk * hgroups);
        const int64_t bb = bk / a.Hkv, kv = bk - bb * a.Hkv;
        gl = G - 8 * hg < 8 ? G - 8 * hg : 8;
        hb = bb * a.Hq + kv * G + 8 * hg;
        sq = bk;
    };
    int64_t hbase, seq;
    int Gl;
    unit_rows(grp, hbase, Gl, seq);
    const int64_t s0 = grp ? s0B : s0A, s1 = grp ? s1B : s1A;
    const int nchunk = s1 > s0 ? (int)((s1 - s0 + C::kChunk - 1) / C::kChunk) : 0;
    const int nmine = nchunk > wi ? (nchunk - wi + nw - 1) / nw : 0;
    // A paged cache's table entries for the CTA's token ranges go to shared
    // memory first (one coalesced load per CTA), so the per-chunk lookups that
    // feed the bulk copies do not wait on global memory; longer ranges keep the
    // direct lookups.
    const int64_t lb0A = s0A >> 6, lb0B = s0B >> 6;
    const int ntabA = s1A > s0A ? (int)(((s1A + 63) >> 6) - lb0A) : 0;
    const int ntabB = ngrp == 2 && s1B > s0B ? (int)(((s1B + 63) >> 6) - lb0B) : 0;
    const bool staged = (a.ktable || a.vtable) && ntabA + ntabB <= kTabMax;
    if (staged) {
        for (int g = 0; g < ngrp; ++g) {
            int64_t hb_, sq_;
            int gl_;
            unit_rows(g, hb_, gl_, sq_);
            const int off = g ? ntabA : 0, n = g ? ntabB : ntabA;
            const int64_t l0 = g ? lb0B : lb0A;
            for (int i = threadIdx.x; i < n; i += NW * 32) {
                sTab[off + i] = a.ktable ? __ldg(a.ktable + sq_ * a.NB + l0 + i) : 0;
                sTab[kTabMax + off + i] = a.vtable ? __ldg(a.vtable + sq_ * a.NB + l0 + i) : 0;
            }
        }
        __syncthreads();
    }
    const int64_t lb0 = grp ? lb0B : lb0A;
    const int toff = grp ? ntabA : 0;
    const int64_t kbb = block_bytes(D, QJL), vbb = block_bytes(D, false);

    if (lane == 0)
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[warp * kStages + s]), 1);
    fence_mbar_init();
    __syncwarp();

    // cache blocks (K, V) of this warp's chunk i; a paged cache reads its block table
    auto blocks_of = [&](int i, int64_t& kblk, int64_t& vblk) {
        const int64_t t0 = s0 + (int64_t)(wi + i * nw) * C::kChunk;
        if (staged) {
            const int ti = (int)((t0 >> 6) - lb0) + toff;
            kblk = staged_block(a.ktable, sTab, a.kpool, seq * a.NB + (t0 >> 6), ti, a.err);
            vblk = staged_block(a.vtable, sTab + kTabMax, a.vpool, seq * a.NB + (t0 >> 6), ti, a.err);
        } else {
            kblk = cache_block(a.ktable, a.kpool, a.NB, seq, t0 >> 6, a.err);
            vblk = cache_block(a.vtable, a.vpool, a.NB, seq, t0 >> 6, a.err);
        }
    };
    auto issue = [&](int i, int64_t kblk, int64_t vblk) {
        const int64_t t0 = s0 + (int64_t)(wi + i * nw) * C::kChunk;     // multiple of the chunk
        const int sub = (int)((t0 & 63) / C::kChunk);
        const uint8_t* kb = a.kc + (kblk >= 0 ? kblk : 0) * kbb;    // a bad table entry reads block 0
        const uint8_t* vb = a.vc + (vblk >= 0 ? vblk : 0) * vbb;
        uint8_t* st = ring + (i % kStages) * C::kStageB;
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        constexpr int cb = C::kCodeB, sb = C::kSignB, ch = C::kChunk;
        mbar_expect_tx(bar, C::kStageB);
        bulk_g2s(smem_u32(st + C::kOffKc), kb + sub * ch * cb, ch * cb, bar);
        if constexpr (QJL) {
            bulk_g2s(smem_u32(st + C::kOffKs), kb + 64 * cb + sub * ch * sb, ch * sb, bar);
            bulk_g2s(smem_u32(st + C::kOffKn), kb + 64 * (cb + sb) + sub * 2 * ch, 2 * ch, bar);
            bulk_g2s(smem_u32(st + C::kOffKg), kb + 64 * (cb + sb) + 128 + sub * 2 * ch, 2 * ch, bar);
        } else {
            bulk_g2s(smem_u32(st + C::kOffKn), kb + 64 * cb + sub * 2 * ch, 2 * ch, bar);
        }
        bulk_g2s(smem_u32(st + C::kOffVc), vb + sub * ch * cb, ch * cb, bar);
        bulk_g2s(smem_u32(st + C::kOffVn), vb + 64 * cb + sub * 2 * ch, 2 * ch, bar);
    };
    // chunks holding tokens that a chained encode writes are fetched only after pdl_wait
    auto fresh = [&](int i) {
        const int64_t t0 = s0 + (int64_t)(wi + i * nw) * C::kChunk;
        return t0 < a.fresh_hi && a.fresh_lo < t0 + C::kChunk;
    };
    if (lane == 0) {
        for (int i = 0; i < kStages && i < nmine; ++i)
            if (!fresh(i)) {
                int64_t kb_, vb_;
                blocks_of(i, kb_, vb_);
                issue(i, kb_, vb_);
            }
    }
    pdl_wait();                           // q' and u' come from the prologue kernel
    if (lane == 0) {
        bool any = false;
        for (int i = 0; i < kStages && i < nmine; ++i) any |= fresh(i);
        if (any) {
            asm volatile("fence.proxy.async;" ::: "memory");
            for (int i = 0; i < kStages && i < nmine; ++i)
                if (fresh(i)) {
                    int64_t kb_, vb_;
                    blocks_of(i, kb_, vb_);
                    issue(i, kb_, vb_);
                }
        }
    }
    // blocks of the next chunk to issue, looked up one chunk ahead so that a
    // block-table load overlaps a chunk of work
    int64_t next_k = 0, next_v = 0;
    if (lane == 0 && kStages < nmine) blocks_of(kStages, next_k, next_v);

    // B-operand fragment of k-step kc: column n = gr of n-tile nt is head
    // 4 nt + gr / 2, limb gr % 2; rows 16 kc + 2 tq4 (+1), +8 (+9)
    auto b_frag = [&](const float* base, int64_t hb, int gl, int nt, int kc, uint32_t& r0, uint32_t& r1) {
        const int hcol = 4 * nt + (gr >> 1);
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (hcol < gl) {
            const float* p = base + (hb + hcol) * D + 16 * kc + 2 * tq4;
            x[0] = p[0]; x[1] = p[1]; x[2] = p[8]; x[3] = p[9];
        }
        uint32_t h0, l0, h1, l1;
        split_hilo(x[0], x[1], h0, l0);
        split_hilo(x[2], x[3], h1, l1);
        r0 = (gr & 1) ? l0 : h0;
        r1 = (gr & 1) ? l1 : h1;
    };
    uint32_t bq[C::kBRegs ? NT : 1][C::kBRegs ? kKC : 1][2];
    if constexpr (C::kBRegs) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int kc = 0; kc < kKC; ++kc) b_frag(a.qp, hbase, Gl, nt, kc, bq[nt][kc][0], bq[nt][kc][1]);
    } else {
        // q' fragments of each group's unit, in that group's copy of sB
        for (int idx = warp; idx < ngrp * kKC; idx += NW) {
            const int g = idx >= kKC ? 1 : 0, kc = idx - g * kKC;
            int64_t hb_, sq_;
            int gl_;
            unit_rows(g, hb_, gl_, sq_);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint32_t r0, r1;
                b_frag(a.qp, hb_, gl_, nt, kc, r0, r1);
                sB[(size_t)g * kSBGroup + (nt * kKC + kc) * 32 + lane] = make_uint2(r0, r1);
            }
        }
    }
    [[maybe_unused]] const uint2* sBw = sB + (size_t)grp * kSBGroup;   // this warp's group's operands
    // QJL term on int8 operands.  u' of each head is taken to 16-bit fixed point,
    // u_int = rint(u' kQ / max|u'|), as two signed byte limbs (256 hi + lo): B column
    // n = gr of n-tile nt is head 4 nt + gr / 2, limb gr % 2.  The A operand byte e
    // of a0/a1 (a2/a3) in k-block kb is -128 times bit 8 e + 7 - 2 (kb % 4)
    // (8 e + 6 - 2 (kb % 4)) of lane tq4's sign word of slice kb / 4, so b0 (b1)
    // byte e holds u_int of that bit's JL row.  With acc = sum of the products,
    // sum_i u'_i (2 sigma_i - 1) = (max|u'| / kQ) (-acc / 64 - sum_i u_int_i), exact
    // up to the fixed point of u' (the term is scaled by gamma ~ 0.18 of the score).
    constexpr int kKB = D / 32;
    constexpr float kQ = 32000.f;
    [[maybe_unused]] uint32_t iu[QJL && C::kBRegs ? NT : 1][QJL && C::kBRegs ? kKB : 1][2];
    [[maybe_unused]] float fS[NT], uS[NT];   // factors of this lane's own head 4 nt + tq4
    if constexpr (QJL) {
        auto row_of = [&](int kb, int half, int e) {
            const int bit = 8 * e + 7 - 2 * (kb & 3) - half;
            if constexpr (D == 64) return slot_coord(0, tq4, e < 2 ? bit : bit - 20);   // h | h << 20
            return slot_coord(kb >> 2, tq4, bit < 16 ? 2 * bit : 2 * (bit - 16) + 1);
        };
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int hcol = 4 * nt + (gr >> 1);
            const bool live = hcol < Gl;
            const float* up = a.up + (hbase + (live ? hcol : 0)) * D;
            float um = 0.f;
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int e = 0; e < 4; ++e) um = fmaxf(um, fabsf(up[row_of(kb, hf, e)]));
            um = fmaxf(um, __shfl_xor_sync(kFull, um, 1));
            um = fmaxf(um, __shfl_xor_sync(kFull, um, 2));
            if (!live) um = 0.f;
            const float fu = um > 0.f ? kQ / um : 0.f;
            int usum = 0;
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb) {
                uint32_t w[2] = {0u, 0u};
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ui = __float2int_rn(up[row_of(kb, hf, e)] * fu);
                        const int lo = ((ui + 128) & 255) - 128;
                        w[hf] |= (uint32_t)(uint8_t)(int8_t)((gr & 1) ? lo : (ui - lo) >> 8) << (8 * e);
                        usum += ui;
                    }
                if constexpr (C::kBRegs) {
                    iu[nt][kb][0] = w[0];
                    iu[nt][kb][1] = w[1];
                } else if (wi == 0) {
                    sB[(size_t)grp * kSBGroup + ((NT + nt) * kKC + kb) * 32 + lane] = make_uint2(w[0], w[1]);
                }
            }
            usum += __shfl_xor_sync(kFull, usum, 1);
            usum += __shfl_xor_sync(kFull, usum, 2);
            // this lane's score columns are head 4 nt + tq4, whose factors sit in lane 8 tq4
            fS[nt] = a.scale_log2 * (__shfl_sync(kFull, um, 8 * tq4) / kQ) * (1.f / 64.f);
            uS[nt] = 64.f * (float)__shfl_sync(kFull, usum, 8 * tq4);
        }
    }
    if constexpr (!C::kBRegs) __syncthreads();
    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
    const uint32_t* pw = a.cb.pow2;
    [[maybe_unused]] const uint32_t m64 = pw[20] | 1u;    // d = 64 sign widening factor

    float o[NT][kKC][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int mt = 0; mt < kKC; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    float mrun[NT], lrun[NT], live[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        mrun[nt] = -INFINITY;
        lrun[nt] = 0.f;
        live[nt] = (4 * nt + tq4 < Gl) ? 1.f : 0.f;   // this lane's head exists
    }
    bool failed = false, drained = true;

    for (int i = 0; i < nmine; ++i) {
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        const bool ok = mbar_wait_bounded(bar, (uint32_t)((i / kStages) & 1), i == 0 ? a.first_wait : kWaitLimit);
        if (__any_sync(kFull, !ok)) {         // warp-uniform: no lane may run on alone into mma.sync
            failed = true;
            if (lane == 0) atomicExch(a.err, 1);
            // wait (bounded) for this warp's copies still in flight before its ring is reused
            bool all = true;
            for (int j = i; j < nmine && j < i + kStages; ++j)
                all &= mbar_wait_bounded(smem_u32(&bars[warp * kStages + (j % kStages)]), (uint32_t)((j / kStages) & 1));
            drained = __all_sync(kFull, all);
            break;
        }
        const uint8_t* st = ring + (i % kStages) * C::kStageB;
        const int64_t tok0 = s0 + (int64_t)(wi + i * nw) * C::kChunk;
        const int nvalid = (int)((s1 - tok0) < C::kChunk ? (s1 - tok0) : C::kChunk);

        // one 16-token tile; PARTIAL masks tokens beyond nvalid (only the last
        // chunk of a split can be partial)
        auto tile = [&](const int kt, auto partial_tag) {
            constexpr bool PARTIAL = decltype(partial_tag)::value;
            const int tA = kt * 16 + gr, tB = tA + 8;            // this lane's two tokens
            // ---------------- scores
            uint32_t selA[C::kS][4], selB[C::kS][4];
            [[maybe_unused]] uint32_t sgA[C::kS], sgB[C::kS];
#pragma unroll
            for (int sl = 0; sl < C::kS; ++sl) {
                token_selectors<D>(st + C::kOffKc + tA * C::kCodeB, sl, tq4, pw, selA[sl]);
                token_selectors<D>(st + C::kOffKc + tB * C::kCodeB, sl, tq4, pw, selB[sl]);
                if constexpr (QJL) {
                    sgA[sl] = token_signs<D>(st + C::kOffKs + tA * C::kSignB, sl, tq4, m64);
                    sgB[sl] = token_signs<D>(st + C::kOffKs + tB * C::kSignB, sl, tq4, m64);
                }
            }
            float acc[NT][4];
            [[maybe_unused]] int accS[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
                accS[nt][0] = accS[nt][1] = accS[nt][2] = accS[nt][3] = 0;
            }
#pragma unroll
            for (int kc = 0; kc < kKC; ++kc) {
                const int sl = kc >> 3, kk = kc & 7;
                uint32_t ka[4];
                dequant4(sel_for(selA[sl], pw, kk), lut, ka[0], ka[2]);
                dequant4(sel_for(selB[sl], pw, kk), lut, ka[1], ka[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if constexpr (C::kBRegs) {
                        mma16816(acc[nt], ka, bq[nt][kc][0], bq[nt][kc][1]);
                    } else {
                        const uint2 fq = sBw[(nt * kKC + kc) * 32 + lane];
                        mma16816(acc[nt], ka, fq.x, fq.y);
                    }
                }
                if constexpr (QJL) {
                    if ((kc & 1) == 0) {                        // one k32 block of signs per two k-steps
                        const int kb = kc >> 1, k4 = kb & 3;
                        const uint32_t sg[4] = {shl_m(sgA[sl], pw, 2 * k4) & 0x80808080u,
                                                shl_m(sgB[sl], pw, 2 * k4) & 0x80808080u,
                                                shl_m(sgA[sl], pw, 2 * k4 + 1) & 0x80808080u,
                                                shl_m(sgB[sl], pw, 2 * k4 + 1) & 0x80808080u};
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            if constexpr (C::kBRegs) {
                                imma16832(accS[nt], sg, iu[nt][kb][0], iu[nt][kb][1]);
                            } else {
                                const uint2 fu = sBw[((NT + nt) * kKC + kb) * 32 + lane];
                                imma16832(accS[nt], sg, fu.x, fu.y);
                            }
                        }
                    }
                }
            }
            [[maybe_unused]] float gAf = 0.f, gBf = 0.f;
            if constexpr (QJL) {
                gAf = __half2float(*reinterpret_cast<const __half*>(st + C::kOffKg + 2 * tA));
                gBf = __half2float(*reinterpret_cast<const __half*>(st + C::kOffKg + 2 * tB));
            }
            // ---------------- online softmax per head (this lane: head 4 nt + tq4)
            const float2 nkA = __half22float2(__halves2half2(*reinterpret_cast<const __half*>(st + C::kOffKn + 2 * tA),
                                                             *reinterpret_cast<const __half*>(st + C::kOffKn + 2 * tB)));
            float2 nv = __half22float2(__halves2half2(*reinterpret_cast<const __half*>(st + C::kOffVn + 2 * tA),
                                                      *reinterpret_cast<const __half*>(st + C::kOffVn + 2 * tB)));
            const bool okA = tA < nvalid, okB = tB < nvalid;
            if constexpr (PARTIAL) {
                if (!okA) nv.x = 0.f;
                if (!okB) nv.y = 0.f;
            }
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float sA = a.scale_log2 * (acc[nt][0] + acc[nt][1]);
                float sB_ = a.scale_log2 * (acc[nt][2] + acc[nt][3]);
                if constexpr (QJL) {
                    // + gamma (max|u'| / kQ) (-acc / 64 - sum u_int), acc = 256 hi-limb + lo-limb column
                    sA = fmaf(-gAf * fS[nt], (float)(accS[nt][0] * 256 + accS[nt][1]) + uS[nt], sA);
                    sB_ = fmaf(-gBf * fS[nt], (float)(accS[nt][2] * 256 + accS[nt][3]) + uS[nt], sB_);
                }
                sA *= nkA.x;
                sB_ *= nkA.y;
                if constexpr (PARTIAL) {
                    if (!okA) sA = -INFINITY;
                    if (!okB) sB_ = -INFINITY;
                }
                float mt = fmaxf(sA, sB_);
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 4));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 16));
                const float mnew = fmaxf(mrun[nt], mt);
                if (__any_sync(kFull, mnew > mrun[nt])) {   // a new running maximum
                    const float corr = (mnew == -INFINITY) ? 1.f : fast_exp2(mrun[nt] - mnew);
                    lrun[nt] *= corr;
#pragma unroll
                    for (int mt2 = 0; mt2 < kKC; ++mt2) {
                        o[nt][mt2][0] *= corr; o[nt][mt2][1] *= corr; o[nt][mt2][2] *= corr; o[nt][mt2][3] *= corr;
                    }
                    mrun[nt] = mnew;
                }
                // mrun >= sA, sB here, so the exponent is <= 0 (masked: -inf -> 0)
                const float pA = fast_exp2(sA - mrun[nt]);
                const float pB = fast_exp2(sB_ - mrun[nt]);
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
#pragma unroll
            for (int sl = 0; sl < C::kS; ++sl) {
                token_selectors<D>(st + C::kOffVc + tA * C::kCodeB, sl, tq4, pw, selA[sl]);
                token_selectors<D>(st + C::kOffVc + tB * C::kCodeB, sl, tq4, pw, selB[sl]);
            }
#pragma unroll
            for (int kc = 0; kc < kKC; ++kc) {
                const int sl = kc >> 3, kk = kc & 7;
                uint32_t x0, x1, y0, y1;
                dequant4(sel_for(selA[sl], pw, kk), lut, x0, x1);      // token tA: coords 16kc+2t(+1), +8
                dequant4(sel_for(selB[sl], pw, kk), lut, y0, y1);      // token tB
                const uint32_t va[4] = {movmatrix_t(x0), movmatrix_t(x1), movmatrix_t(y0), movmatrix_t(y1)};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(o[nt][kc], va, pb[nt][0], pb[nt][1]);
            }
        };
        if (nvalid == C::kChunk) {
#pragma unroll
            for (int kt = 0; kt < C::kTiles; ++kt) tile(kt, std::false_type{});
        } else {
            tile(0, std::true_type{});
            if (C::kTiles > 1 && nvalid > 16) tile(1, std::true_type{});
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nmine) {
            fence_proxy_async();
            issue(i + kStages, next_k, next_v);
            if (i + kStages + 1 < nmine) blocks_of(i + kStages + 1, next_k, next_v);
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
    // ---------------- merge the warps of the CTA into one partial per head.  Each
    // warp's (max, sum) go to sML; its accumulators to its own ring, unless a
    // failed wait left copies of unknown state there (then the warp is skipped:
    // its max is -inf and its accumulators are never read).
    __syncwarp();
    float* wbuf = reinterpret_cast<float*>(ring);             // [Gl][D], in this warp's own ring
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + tq4;
        if (h < Gl) {
            if (drained) {
#pragma unroll
                for (int mt = 0; mt < kKC; ++mt) {
                    wbuf[h * D + 16 * mt + gr] = o[nt][mt][0] + o[nt][mt][1];
                    wbuf[h * D + 16 * mt + 8 + gr] = o[nt][mt][2] + o[nt][mt][3];
                }
            }
            if (gr == 0) {
                sML[(warp * 8 + h) * 2] = mrun[nt];
                sML[(warp * 8 + h) * 2 + 1] = lrun[nt];
            }
        }
    }
    __syncthreads();
    for (int g = 0; g < ngrp; ++g) {
        int64_t hb_, sq_;
        int gl_;
        unit_rows(g, hb_, gl_, sq_);
        const int w0 = g ? kA : 0, w1 = g ? NW : kA;
        for (int idx = threadIdx.x; idx < gl_ * D; idx += NW * 32) {
            const int h = idx / D, j = idx % D;
            float M = -INFINITY;
            for (int w = w0; w < w1; ++w) M = fmaxf(M, sML[(w * 8 + h) * 2]);
            float L = 0.f, A = 0.f;
            if (M != -INFINITY) {
                for (int w = w0; w < w1; ++w) {
                    const float mw = sML[(w * 8 + h) * 2];
                    if (mw == -INFINITY) continue;                    // empty or failed warp
                    const float* wb = reinterpret_cast<const float*>(smem + (size_t)w * kStages * C::kStageB) + h * D;
                    const float f = exp2f(mw - M);
                    L = fmaf(f, sML[(w * 8 + h) * 2 + 1], L);
                    A = fmaf(f, wb[j], A);
                }
            }
            const int slot = g ? slotB : slotA;
            const int64_t pidx = (hb_ + h) * a.nsplit + slot;
            a.part_acc[pidx * D + j] = A;
            if (j == 0) {
                a.part_ml[2 * pidx] = M;
                a.part_ml[2 * pidx + 1] = L;
            }
            // the CTA holding the unit's last chunk empties the unit's unused slots
            if (g ? endB : endA)
                for (int sp = slot + 1; sp < a.nsplit; ++sp) {
                    const int64_t e = (hb_ + h) * a.nsplit + sp;
                    a.part_acc[e * D + j] = 0.f;
                    if (j == 0) {
                        a.part_ml[2 * e] = -INFINITY;
                        a.part_ml[2 * e + 1] = 0.f;
                    }
                }
        }
    }
}

}  // namespace

constexpr int kNW1 = 16;   // warps per CTA, up to 4 heads per kv head (one n-tile)
constexpr int kNW2 = 8;    // warps per CTA, 8 heads per kv head (two n-tiles, more registers)

template <int D, int NT, int NW, bool QJL>
cudaError_t launch_mma_t(const DecArgs& a, int G, cudaStream_t s) {
    using C = Cfg<D, QJL>;
    const size_t smem = (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                        (size_t)NW * 8 * 2 * sizeof(float) + 2 * kTabMax * sizeof(int32_t) +
                        (C::kBRegs ? 0 : (size_t)2 * 2 * NT * C::kKC * 32 * sizeof(uint2));
    auto kern = tq_decode_mma_kernel<D, NT, NW, QJL>;
    cudaError_t e = set_smem_once<tq_decode_mma_kernel<D, NT, NW, QJL>>((int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid = a.sk_ctas > 0 ? dim3((unsigned)a.sk_ctas)
                                    : dim3(a.nsplit, (unsigned)(a.Hkv * ((G + 7) / 8)), (unsigned)a.B);
    return launch_pdl(kern, grid, dim3(NW * 32), smem, s, a, G);
}

template <bool QJL>
cudaError_t launch_mma_q(int d, int G, const DecArgs& a, cudaStream_t s) {
    if (d == 64)
        return G <= 4 ? launch_mma_t<64, 1, kNW1, QJL>(a, G, s) : launch_mma_t<64, 2, kNW2, QJL>(a, G, s);
    if (d == 128)
        return G <= 4 ? launch_mma_t<128, 1, kNW1, QJL>(a, G, s) : launch_mma_t<128, 2, kNW2, QJL>(a, G, s);
    return G <= 4 ? launch_mma_t<256, 1, kNW1, QJL>(a, G, s) : launch_mma_t<256, 2, kNW2, QJL>(a, G, s);
}

cudaError_t launch_decode_mma(int d, int G, bool qjl, const DecArgs& a, cudaStream_t s) {
    if (!head_dim_ok(d) || G < 1) return cudaErrorInvalidValue;
    if (a.B * a.Hkv == 0) return cudaSuccess;
    return qjl ? launch_mma_q<true>(d, G, a, s) : launch_mma_q<false>(d, G, a, s);
}

int decode_mma_chunk_tokens(int d) {
    return d == 64 ? Cfg<64>::kChunk : d == 128 ? Cfg<128>::kChunk : Cfg<256>::kChunk;
}
int decode_mma_warps(int G) { return G <= 4 ? kNW1 : kNW2; }

}  // namespace tqi
