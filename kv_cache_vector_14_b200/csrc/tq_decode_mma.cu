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
// registers (movmatrix).  With at most two query heads per kv head at
// head_dim 128 (K8) the keys enter as int8 limbs of the integer centroids
// c 2^14 instead (one prmt per four codes and limb, no interleave) against q'
// in 22-bit fixed point as three byte limbs.
//
// Work partition: a uniform split of every (batch, kv head, head group) unit
// (grid = splits x units), or a stream-K grid over all units' chunks laid end
// to end (grid = CTAs, each warp a contiguous run of chunks, at most one warp
// per CTA crossing into a second unit); the host's cost model picks.
//
// Data movement: each warp owns a ring of STAGES shared-memory buffers of a
// chunk of tokens (32 at d = 128, 16 at d = 256; K codes, signs, norms,
// gammas, V codes, norms: six bulk copies issued by six lanes at once,
// cp.async.bulk with an mbarrier transaction count, no multicast).  Waits are
// bounded: on timeout the kernel
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
// Pool block of table row `row` (= sequence * blocks per sequence + logical
// block) of a paged cache, or `row` itself for a contiguous cache; an entry
// outside the pool sets the check word and gives -1, as cache_block does.
__device__ __forceinline__ int64_t table_block(const int32_t* table, int64_t pool, int64_t row, int* err) {
    if (!table) return row;
    const int32_t p = __ldg(table + row);
    if (p < 0 || (int64_t)p >= pool) {
        atomicExch(err, 1);
        return -1;
    }
    return p;
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
template <int D, int NT, int NW, bool QJL, bool K8>
__global__ void __launch_bounds__(NW * 32, 1) tq_decode_mma_kernel(const DecArgs a, int G) {
    using C = Cfg<D, QJL>;
    constexpr int kKC = C::kKC;
    static_assert(!K8 || (D == 128 && NT == 1), "int8 key operands: head_dim 128, up to two heads per kv head");
    constexpr int kSBGroup = 2 * NT * kKC * 32;   // uint2 entries of one unit's q'/u' fragments
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NW * kStages * C::kStageB);
    // per-warp (max, sum) of each head for the merge: [NW][8][2]
    float* sML = reinterpret_cast<float*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8);
    // paged caches: the CTA's slices of the K and V block tables, [2][kTabMax]
    // q'/u' fragments per (unit group, operand, n-tile, k-step, lane), filled once per CTA
    int32_t* sTab = reinterpret_cast<int32_t*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                                               (size_t)NW * 8 * 2 * sizeof(float));
    uint2* sB = reinterpret_cast<uint2*>(smem + (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                                         (size_t)NW * 8 * 2 * sizeof(float) + 2 * kTabMax * sizeof(int32_t));
    // score factors per (unit group, kind, head): [2][3][8] (u' factor, u' sum, int8 q' factor)
    float* sF = reinterpret_cast<float*>(sB + 2 * kSBGroup);
    // the crossing warp's unit-A result: accumulators [8][D], (max, sum) [8][2]
    float* xacc = sF + 2 * 3 * 8;
    float* xml = xacc + 8 * D;
    int64_t* sU = reinterpret_cast<int64_t*>(xml + 8 * 2);     // [NW][2][4] unit descriptors
    int* sMerge = reinterpret_cast<int*>(sU + NW * 8);          // [8] CTA merge facts
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, tq4 = lane & 3;
    uint8_t* ring = smem + (size_t)warp * kStages * C::kStageB;
    const int hgroups = (G + 7) >> 3;

    // ---------------- this CTA's work.  A unit is (batch, kv head, query-head
    // group).  Uniform split grid: unit (blockIdx.z, blockIdx.y), the tokens of
    // split blockIdx.x, chunks dealt to the warps in turn.  Stream-K: the CTA's
    // chunk range [lo, hi) of the units laid end to end lies in at most two
    // units, A and then B from chunk `cut`; warp w takes the contiguous chunks
    // [lo + w S / NW, lo + (w + 1) S / NW), S = hi - lo, so at most one warp
    // crosses from A to B, and it keeps its A result in shared memory (xacc,
    // xml) for the merge.  The CTA writes one partial slot of each unit it
    // touches, c - (first CTA of the unit); the CTA holding a unit's last chunk
    // also empties the unit's unused slots.
    int64_t unitA = 0, unitB = 0, s0A = 0, s1A = 0, s0B = 0, s1B = 0;   // token ranges of A and B
    int64_t cut = INT64_MAX, xw0 = 0, nck = 1;
    int slotA = 0, slotB = 0, ngrp = 1, nmine = 0, ipart = 0;
    bool endA = false, endB = false, firstB = false;
    int aEnd = NW, bBeg = NW;          // merge: warps [0, aEnd) feed unit A, [bBeg, NW) unit B
    bool aX = false;                   // the crossing warp's unit-A result feeds unit A too
    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[blockIdx.z] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    if (a.sk_ctas == 0) {
        unitA = (int64_t)blockIdx.z * a.Hkv * hgroups + blockIdx.y;
        s0A = (int64_t)blockIdx.x * a.split_tokens;
        s1A = (s0A + a.split_tokens < Tb) ? s0A + a.split_tokens : Tb;
        slotA = blockIdx.x;
        const int nchunk = s1A > s0A ? (int)((s1A - s0A + C::kChunk - 1) / C::kChunk) : 0;
        nmine = nchunk > warp ? (nchunk - warp + NW - 1) / NW : 0;
        ipart = nmine;
    } else {
        const int64_t N = a.sk_total, nC = a.sk_ctas, c = blockIdx.x;
        nck = a.sk_nck;
        const int64_t lo = c * N / nC, hi = (c + 1) * N / nC, S = hi - lo;
        const int64_t u0 = lo / nck, u1 = (hi - 1) / nck, nxt = (u0 + 1) * nck;
        auto tok = [&](int64_t x, int64_t u) {                 // chunk x of unit u as a token bound
            const int64_t t = (x - u * nck) * C::kChunk;
            return t < Tb ? t : Tb;
        };
        auto first_cta = [&](int64_t u) { return (int)(((u * nck + 1) * nC - 1) / N); };
        unitA = u0;
        s0A = tok(lo, u0);
        s1A = tok(nxt < hi ? nxt : hi, u0);
        slotA = (int)c - first_cta(u0);
        endA = nxt <= hi;
        if (u1 != u0) {
            ngrp = 2;
            cut = nxt;
            unitB = u1;
            s0B = tok(nxt, u1);
            s1B = tok(hi, u1);
            slotB = (int)c - first_cta(u1);
            endB = hi == (u1 + 1) * nck;
        }
        auto wlo = [&](int w) { return lo + (int64_t)w * S / NW; };
        xw0 = wlo(warp);
        const int64_t xw1 = wlo(warp + 1);
        nmine = (int)(xw1 - xw0);
        firstB = xw0 >= cut;
        ipart = (xw0 < cut && cut < xw1) ? (int)(cut - xw0) : nmine;
        if (ngrp == 2)
            for (int w = 0; w < NW; ++w) {
                const int64_t a0 = wlo(w), a1 = wlo(w + 1);
                if (a0 >= cut || cut < a1) {
                    aEnd = bBeg = w;
                    aX = a0 < cut;
                    break;
                }
            }
    }
    auto unit_rows = [&](int g, int64_t& hb, int& gl, int64_t& sq) {
        const int64_t u = g ? unitB : unitA;
        const int64_t bk = u / hgroups;                          // b * Hkv + kv head
        const int hg = (int)(u - bk * hgroups);
        const int64_t bb = bk / a.Hkv, kv = bk - bb * a.Hkv;
        gl = G - 8 * hg < 8 ? G - 8 * hg : 8;
        hb = bb * a.Hq + kv * G + 8 * hg;
        sq = bk;
    };
    int64_t hbA, seqA, hbB = 0, seqB = 0;
    int GlA, GlB = 0;
    unit_rows(0, hbA, GlA, seqA);
    if (ngrp == 2) unit_rows(1, hbB, GlB, seqB);
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
            const int off = g ? ntabA : 0, n = g ? ntabB : ntabA;
            const int64_t l0 = g ? lb0B : lb0A, sq_ = g ? seqB : seqA;
            for (int i = threadIdx.x; i < n; i += NW * 32) {
                sTab[off + i] = a.ktable ? __ldg(a.ktable + sq_ * a.NB + l0 + i) : 0;
                sTab[kTabMax + off + i] = a.vtable ? __ldg(a.vtable + sq_ * a.NB + l0 + i) : 0;
            }
        }
        __syncthreads();
    }
    const int64_t kbb = block_bytes(D, QJL), vbb = block_bytes(D, false);
    // Unit descriptors in shared memory, read by the producer lane per chunk,
    // at the crossing and in the merge (registers stay with the main loop):
    // per warp and unit group, block-table row of logical block 0, offset of
    // the staged table slice, first query row, query heads.  CTA-wide merge
    // facts in sMerge (written by thread 0, read after the next barrier).
    int64_t* myU = sU + warp * 8;
    if (lane == 0) {
        myU[0] = seqA * a.NB;
        myU[1] = -lb0A;
        myU[2] = hbA;
        myU[3] = GlA;
        myU[4] = seqB * a.NB;
        myU[5] = ntabA - lb0B;
        myU[6] = hbB;
        myU[7] = GlB;
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[warp * kStages + s]), 1);
    }
    if (threadIdx.x == 0) {
        sMerge[0] = ngrp; sMerge[1] = aEnd; sMerge[2] = bBeg; sMerge[3] = aX;
        sMerge[4] = slotA; sMerge[5] = slotB; sMerge[6] = endA; sMerge[7] = endB;
    }
    fence_mbar_init();
    __syncwarp();
    // chunk i of this warp is chunk (i < icut ? offA : offB) + i step of its unit
    int offA, offB = 0, icut, step;
    if (a.sk_ctas == 0) {
        offA = (int)(s0A / C::kChunk) + warp;
        icut = nmine;
        step = NW;
    } else {
        offA = (int)(xw0 - unitA * nck);
        offB = (int)(xw0 - unitB * nck);
        icut = firstB ? 0 : ipart;
        step = 1;
    }

    // token offset of this warp's chunk i in its unit, and whether the unit is B
    auto chunk_at = [&](int i, bool& inB) -> int64_t {
        inB = i >= icut;
        return (int64_t)((inB ? offB : offA) + i * step) * C::kChunk;
    };
    // cache blocks (K, V) of this warp's chunk i; a paged cache reads its block table
    auto blocks_of = [&](int i, int64_t& kblk, int64_t& vblk) {
        bool inB;
        const int64_t t0 = chunk_at(i, inB);
        const int64_t* u = myU + (inB ? 4 : 0);
        const int64_t row = u[0] + (t0 >> 6);
        if (staged) {
            const int ti = (int)((t0 >> 6) + u[1]);
            kblk = staged_block(a.ktable, sTab, a.kpool, row, ti, a.err);
            vblk = staged_block(a.vtable, sTab + kTabMax, a.vpool, row, ti, a.err);
        } else {
            kblk = table_block(a.ktable, a.kpool, row, a.err);
            vblk = table_block(a.vtable, a.vpool, row, a.err);
        }
    };
    // A stage is six bulk copies (four without the QJL bit): K codes, K signs, K
    // norms, gammas, V codes, V norms of one chunk.  Lane k issues copy k, so a
    // stage costs the warp one copy instruction rather than six in a row: its
    // source offset in the K or V block for sub-chunk 0, the step per sub-chunk,
    // its place in the stage and its size.
    constexpr int kCopies = QJL ? 6 : 4;
    int cp_off = 0, cp_step = 0, cp_dst = 0, cp_size = 0;
    bool cp_v = false;
    {
        constexpr int cb = C::kCodeB, sb = C::kSignB, ch = C::kChunk;
        const int k = QJL ? lane : (lane == 0 ? 0 : lane == 1 ? 2 : lane + 2);   // without QJL: 0, 2, 4, 5
        switch (k) {
            case 0: cp_off = 0; cp_step = ch * cb; cp_dst = C::kOffKc; cp_size = ch * cb; break;
            case 1: cp_off = 64 * cb; cp_step = ch * sb; cp_dst = C::kOffKs; cp_size = ch * sb; break;
            case 2: cp_off = QJL ? 64 * (cb + sb) : 64 * cb; cp_step = 2 * ch; cp_dst = C::kOffKn; cp_size = 2 * ch; break;
            case 3: cp_off = 64 * (cb + sb) + 128; cp_step = 2 * ch; cp_dst = C::kOffKg; cp_size = 2 * ch; break;
            case 4: cp_off = 0; cp_step = ch * cb; cp_dst = C::kOffVc; cp_size = ch * cb; cp_v = true; break;
            case 5: cp_off = 64 * cb; cp_step = 2 * ch; cp_dst = C::kOffVn; cp_size = 2 * ch; cp_v = true; break;
            default: break;
        }
    }
    // every lane of the warp: lane 0 arms the stage's barrier, then lanes 0 .. kCopies - 1 copy
    auto issue = [&](int i, int64_t kblk, int64_t vblk) {
        bool inB;
        const int64_t t0 = chunk_at(i, inB);                          // multiple of the chunk
        const int sub = (int)((t0 & 63) / C::kChunk);
        const uint8_t* kb = a.kc + (kblk >= 0 ? kblk : 0) * kbb;    // a bad table entry reads block 0
        const uint8_t* vb = a.vc + (vblk >= 0 ? vblk : 0) * vbb;
        uint8_t* st = ring + (i % kStages) * C::kStageB;
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        if (lane == 0) mbar_expect_tx(bar, C::kStageB);
        __syncwarp();
        if (lane < kCopies)
            bulk_g2s(smem_u32(st + cp_dst), (cp_v ? vb : kb) + cp_off + sub * cp_step, (uint32_t)cp_size, bar);
    };
    // chunks holding tokens that a chained encode writes are fetched only after pdl_wait
    auto fresh = [&](int i) {
        bool inB;
        const int64_t t0 = chunk_at(i, inB);
        return t0 < a.fresh_hi && a.fresh_lo < t0 + C::kChunk;
    };
    pdl_wait();                           // q' and u' come from the prologue kernel
    // blocks of the next chunk to issue, looked up one chunk ahead so that a
    // block-table load overlaps a chunk of work
    int64_t next_k = 0, next_v = 0;
    if (kStages < nmine) blocks_of(kStages, next_k, next_v);

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
    // The q' fragments of each unit the CTA touches go to sB (group g: unit A
    // or B), filled by all warps; so do the u' words and factors below.
    for (int idx = warp; !K8 && idx < ngrp * kKC; idx += NW) {
        const int g = idx >= kKC ? 1 : 0, kc = idx - g * kKC;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint32_t r0, r1;
            b_frag(a.qp, g ? hbB : hbA, g ? GlB : GlA, nt, kc, r0, r1);
            sB[(size_t)g * kSBGroup + (nt * kKC + kc) * 32 + lane] = make_uint2(r0, r1);
        }
    }
    // int8 key operands (K8, up to two heads): q' of each head in 22-bit fixed
    // point, q_int = rint(q' 2^22 / max|q'|) = l0 + 256 l1 + 65536 l2 (signed byte
    // limbs); B column n = gr is head gr / 4, limb gr % 4 (limb 3 zero).  K-block w
    // of the m16n8k32 operand: rows 4 tq4 + e and 16 + 4 tq4 + e are positions
    // 8 w + e and 8 w + 4 + e of slot tq4, i.e. coordinates 32 w + 2 tq4 + o(e)
    // and 32 w + 16 + 2 tq4 + o(e), o = (0, 1, 8, 9).  The factor of head h,
    // scale_log2 max|q'| 2^-22 2^-14 (the keys are c 2^14), goes to sF[g][2][h].
    if constexpr (K8) {
        for (int g = warp; g < ngrp; g += NW) {
            const int hq = gr >> 2, lq = gr & 3;
            const int gl_ = g ? GlB : GlA;
            const float* qrow = a.qp + ((g ? hbB : hbA) + (hq < gl_ ? hq : 0)) * D;
            float qv[4][8];
            float qm = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int o = (e & 1) + 8 * ((e >> 1) & 1);
                    qv[w][e] = qrow[32 * w + 16 * (e >> 2) + 2 * tq4 + o];
                    qm = fmaxf(qm, fabsf(qv[w][e]));
                }
            qm = fmaxf(qm, __shfl_xor_sync(kFull, qm, 1));
            qm = fmaxf(qm, __shfl_xor_sync(kFull, qm, 2));
            if (hq >= gl_) qm = 0.f;
            const float fq = qm > 0.f ? 4194304.f / qm : 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t b2[2] = {0u, 0u};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int qi = __float2int_rn(qv[w][e] * fq);
                    const int l0 = ((qi + 128) & 255) - 128;
                    const int r1 = (qi - l0) >> 8;
                    const int l1 = ((r1 + 128) & 255) - 128;
                    const int l2 = (r1 - l1) >> 8;
                    const int limb = lq == 0 ? l0 : lq == 1 ? l1 : lq == 2 ? l2 : 0;
                    b2[e >> 2] |= (uint32_t)(uint8_t)(int8_t)limb << (8 * (e & 3));
                }
                sB[(size_t)g * kSBGroup + w * 32 + lane] = make_uint2(b2[0], b2[1]);
            }
            if (lq == 0 && tq4 == 0) sF[(g * 3 + 2) * 8 + hq] = a.scale_log2 * (qm * (1.f / 4194304.f)) * (1.f / 16384.f);
        }
    }
    // QJL term on int8 operands.  u' of each head is taken to 16-bit fixed point,
    // u_int = rint(u' kQ / max|u'|), as two signed byte limbs (256 hi + lo): B column
    // n = gr of n-tile nt is head 4 nt + gr / 2, limb gr % 2.  The A operand byte e
    // of a0/a1 (a2/a3) in k-block kb is -128 times bit 8 e + 7 - 2 (kb % 4)
    // (8 e + 6 - 2 (kb % 4)) of lane tq4's sign word of slice kb / 4, so b0 (b1)
    // byte e holds u_int of that bit's JL row.  With acc = sum of the products,
    // sum_i u'_i (2 sigma_i - 1) = (max|u'| / kQ) (-acc / 64 - sum_i u_int_i), exact
    // up to the fixed point of u' (the term is scaled by gamma ~ 0.18 of the score).
    // The words of (unit g, n-tile nt) go to sB, and the factors of head h to
    // sF[g][0][h] (scale_log2 max|u'| / (64 kQ)) and sF[g][1][h] (64 sum u_int).  With int8
    // key operands (K8) the columns are head gr / 4, limb gr % 4 (limbs 2, 3 zero).
    constexpr int kKB = D / 32;
    constexpr float kQ = 32000.f;
    if constexpr (QJL) {
        auto row_of = [&](int kb, int half, int e) {
            const int bit = 8 * e + 7 - 2 * (kb & 3) - half;
            if constexpr (D == 64) return slot_coord(0, tq4, e < 2 ? bit : bit - 20);   // h | h << 20
            return slot_coord(kb >> 2, tq4, bit < 16 ? 2 * bit : 2 * (bit - 16) + 1);
        };
        for (int idx = warp; idx < ngrp * NT; idx += NW) {
            const int g = idx >= NT ? 1 : 0, nt = idx - g * NT;
            const int hcol = K8 ? (gr >> 2) : 4 * nt + (gr >> 1);
            const bool hlive = hcol < (g ? GlB : GlA);
            const bool zcol = K8 && (gr & 3) >= 2;               // K8: limb columns 2, 3 are zero
            const float* up = a.up + ((g ? hbB : hbA) + (hlive ? hcol : 0)) * D;
            float um = 0.f;
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int e = 0; e < 4; ++e) um = fmaxf(um, fabsf(up[row_of(kb, hf, e)]));
            um = fmaxf(um, __shfl_xor_sync(kFull, um, 1));
            um = fmaxf(um, __shfl_xor_sync(kFull, um, 2));
            if (!hlive) um = 0.f;
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
                        const int lb = (gr & 1) ? lo : (ui - lo) >> 8;
                        w[hf] |= (uint32_t)(uint8_t)(int8_t)(zcol ? 0 : lb) << (8 * e);
                        usum += ui;
                    }
                sB[(size_t)g * kSBGroup + ((NT + nt) * kKC + kb) * 32 + lane] = make_uint2(w[0], w[1]);
            }
            usum += __shfl_xor_sync(kFull, usum, 1);
            usum += __shfl_xor_sync(kFull, usum, 2);
            if ((gr & (K8 ? 3 : 1)) == 0 && tq4 == 0) {
                sF[(g * 3) * 8 + hcol] = a.scale_log2 * (um / kQ) * (1.f / 64.f);
                sF[(g * 3 + 1) * 8 + hcol] = 64.f * (float)usum;
            }
        }
    }
    {
        bool any = false;
        for (int i = 0; i < kStages && i < nmine; ++i) any |= fresh(i);
        if (any) asm volatile("fence.proxy.async;" ::: "memory");
        for (int i = 0; i < kStages && i < nmine; ++i) {
            int64_t kb_, vb_;
            blocks_of(i, kb_, vb_);
            issue(i, kb_, vb_);
        }
    }
    // the crossing warp's unit-A result starts empty (it stays so if a wait fails before the crossing)
    if (ipart < nmine && lane < 8) {
        xml[2 * lane] = -INFINITY;
        xml[2 * lane + 1] = 0.f;
    }
    __syncthreads();
    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
    [[maybe_unused]] const uint32_t l8[4] = {a.cb.lut8_lo[0], a.cb.lut8_lo[1], a.cb.lut8_hi[0], a.cb.lut8_hi[1]};
    const uint32_t* pw = a.cb.pow2;
    [[maybe_unused]] const uint32_t m64 = pw[20] | 1u;    // d = 64 sign widening factor

    // ---------------- this warp's unit: operands and softmax state
    int64_t hbase = hbA;
    int Gl = GlA;
    uint32_t bq[C::kBRegs ? NT : 1][C::kBRegs ? kKC : 1][2];
    [[maybe_unused]] uint32_t iu[QJL && C::kBRegs ? NT : 1][QJL && C::kBRegs ? kKB : 1][2];
    [[maybe_unused]] float fS[NT], uS[NT];   // factors of this lane's own head 4 nt + tq4
    [[maybe_unused]] float fK = 0.f;         // K8: factor of this lane's head's integer key score
    [[maybe_unused]] const uint2* sBw = sB;  // this warp's unit's fragments in sB
    float o[NT][kKC][4];
    float mrun[NT], lrun[NT], live[NT];
    auto load_unit = [&](int g) {
        hbase = myU[4 * g + 2];
        Gl = (int)myU[4 * g + 3];
        sBw = sB + (size_t)g * kSBGroup;
        if constexpr (C::kBRegs) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int kc = 0; kc < (K8 ? 4 : kKC); ++kc) {     // K8: the four k-blocks' q' limbs
                    const uint2 v = sBw[(nt * kKC + kc) * 32 + lane];
                    bq[nt][kc][0] = v.x;
                    bq[nt][kc][1] = v.y;
                }
            if constexpr (QJL) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int kb = 0; kb < kKB; ++kb) {
                        const uint2 v = sBw[((NT + nt) * kKC + kb) * 32 + lane];
                        iu[nt][kb][0] = v.x;
                        iu[nt][kb][1] = v.y;
                    }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            // this lane's head: 4 nt + tq4, or with int8 keys tq4 / 2 (even lanes own it,
            // odd lanes hold the same score and contribute nothing)
            const int hh = K8 ? (tq4 >> 1) : 4 * nt + tq4;
            const bool own = !K8 || (tq4 & 1) == 0;
            if constexpr (QJL) {
                fS[nt] = own ? sF[(g * 3) * 8 + hh] : 0.f;
                uS[nt] = own ? sF[(g * 3 + 1) * 8 + hh] : 0.f;
            }
            if constexpr (K8) fK = sF[(g * 3 + 2) * 8 + hh];
            live[nt] = (own && hh < Gl) ? 1.f : 0.f;      // this lane's head exists
            mrun[nt] = -INFINITY;
            lrun[nt] = 0.f;
#pragma unroll
            for (int mt = 0; mt < kKC; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        }
    };
    // softmax sums over the lanes of a head, then the result of the unit in
    // hand: accumulators to acc_dst [8][D] (if write_acc), (max, sum) of every
    // head this lane serves to ml_dst [8][2] (max -inf where the head is absent)
    auto finish_unit = [&](bool failed_, float* acc_dst, float* ml_dst, bool write_acc) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            if (failed_) { mrun[nt] = -INFINITY; lrun[nt] = 0.f; }
            lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 4);
            lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 8);
            lrun[nt] += __shfl_xor_sync(kFull, lrun[nt], 16);
            const int h = K8 ? (tq4 >> 1) : 4 * nt + tq4;
            const bool own = !K8 || (tq4 & 1) == 0;
            const bool hl = own && h < Gl;
            if (hl && write_acc) {
#pragma unroll
                for (int mt = 0; mt < kKC; ++mt) {
                    acc_dst[h * D + 16 * mt + gr] = o[nt][mt][0] + o[nt][mt][1];
                    acc_dst[h * D + 16 * mt + 8 + gr] = o[nt][mt][2] + o[nt][mt][3];
                }
            }
            if (gr == 0 && own) {
                ml_dst[h * 2] = hl ? mrun[nt] : -INFINITY;
                ml_dst[h * 2 + 1] = hl ? lrun[nt] : 0.f;
            }
        }
    };
    load_unit(firstB ? 1 : 0);
    bool failed = false, drained = true;

    for (int i = 0; i < nmine; ++i) {
        if (i == ipart) {                     // this warp crosses from unit A to unit B
            finish_unit(false, xacc, xml, true);
            load_unit(1);
        }
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
        bool inB_;
        const int64_t tok0 = chunk_at(i, inB_);
        const int nvalid = (int)((Tb - tok0) < C::kChunk ? (Tb - tok0) : C::kChunk);

        // one 16-token tile; PARTIAL masks tokens beyond nvalid (only the last
        // chunk of a sequence can be partial)
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
            // QJL term: int8 m16n8k32 over one k32 block of sign bits
            [[maybe_unused]] auto sign_mma = [&](int kb, int sl) {
                const int k4 = kb & 3;
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
            };
            if constexpr (K8) {
                // keys as int8 limbs of c 2^14: one prmt gives four codes' limb bytes,
                // which are the m16n8k32 A operand rows as they stand (no interleave)
                int accK[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t sa = selA[0][w], sb = selB[0][w];
                    const uint32_t sah = shr_m(sa, pw, 16), sbh = shr_m(sb, pw, 16);
                    const uint32_t alo[4] = {__byte_perm(l8[0], l8[1], sa), __byte_perm(l8[0], l8[1], sb),
                                             __byte_perm(l8[0], l8[1], sah), __byte_perm(l8[0], l8[1], sbh)};
                    const uint32_t ahi[4] = {__byte_perm(l8[2], l8[3], sa), __byte_perm(l8[2], l8[3], sb),
                                             __byte_perm(l8[2], l8[3], sah), __byte_perm(l8[2], l8[3], sbh)};
                    imma16832(accK[0], alo, bq[0][w][0], bq[0][w][1]);
                    imma16832(accK[1], ahi, bq[0][w][0], bq[0][w][1]);
                    if constexpr (QJL) sign_mma(w, 0);
                }
                // this lane's columns 2 tq4, 2 tq4 + 1 are q' limbs 2 (tq4 & 1), + 1 of head tq4 / 2
                const float w0 = (tq4 & 1) ? 65536.f : 1.f, w1 = (tq4 & 1) ? 0.f : 256.f;
                acc[0][0] = fmaf((float)accK[1][0], w0, fmaf((float)accK[1][1], w1, 0.f)) * 256.f +
                            fmaf((float)accK[0][0], w0, (float)accK[0][1] * w1);
                acc[0][2] = fmaf((float)accK[1][2], w0, fmaf((float)accK[1][3], w1, 0.f)) * 256.f +
                            fmaf((float)accK[0][2], w0, (float)accK[0][3] * w1);
            } else {
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
                        if ((kc & 1) == 0) sign_mma(kc >> 1, sl);   // one k32 block of signs per two k-steps
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
                float sA = K8 ? fK * acc[nt][0] : a.scale_log2 * (acc[nt][0] + acc[nt][1]);
                float sB_ = K8 ? fK * acc[nt][2] : a.scale_log2 * (acc[nt][2] + acc[nt][3]);
                if constexpr (QJL) {
                    // + gamma (max|u'| / kQ) (-acc / 64 - sum u_int), acc = 256 hi-limb + lo-limb column
                    // (K8: zero on the odd lanes, whose factors are zero)
                    sA = fmaf(-gAf * fS[nt], (float)(accS[nt][0] * 256 + accS[nt][1]) + uS[nt], sA);
                    sB_ = fmaf(-gBf * fS[nt], (float)(accS[nt][2] * 256 + accS[nt][3]) + uS[nt], sB_);
                }
                if constexpr (K8) {             // the head's q' limbs sit on lanes tq4 and tq4 ^ 1
                    sA += __shfl_xor_sync(kFull, sA, 1);
                    sB_ += __shfl_xor_sync(kFull, sB_, 1);
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
        if (i + kStages < nmine) {            // warp-uniform
            fence_proxy_async();
            issue(i + kStages, next_k, next_v);
            if (i + kStages + 1 < nmine) blocks_of(i + kStages + 1, next_k, next_v);
        }
    }
    pdl_trigger();                        // the combine kernel may start launching
    // ---------------- merge the warps of the CTA into one partial per unit and
    // head.  Each warp's (max, sum) go to sML; its accumulators to its own
    // ring, unless a failed wait left copies of unknown state there (then the
    // warp is skipped: its max is -inf and its accumulators are never read).
    __syncwarp();
    finish_unit(failed, reinterpret_cast<float*>(ring), sML + warp * 16, drained);
    __syncthreads();
    const int ngrp_ = sMerge[0];
    for (int g = 0; g < ngrp_; ++g) {
        const int64_t hb_ = myU[4 * g + 2];
        const int gl_ = (int)myU[4 * g + 3];
        const int w0 = g ? sMerge[2] : 0, w1 = g ? NW : sMerge[1];
        const bool withx = g == 0 && sMerge[3];                  // the crossing warp's unit-A result
        for (int idx = threadIdx.x; idx < gl_ * D; idx += NW * 32) {
            const int h = idx / D, j = idx % D;
            float M = withx ? xml[2 * h] : -INFINITY;
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
                if (withx && xml[2 * h] != -INFINITY) {
                    const float f = exp2f(xml[2 * h] - M);
                    L = fmaf(f, xml[2 * h + 1], L);
                    A = fmaf(f, xacc[h * D + j], A);
                }
            }
            const int slot = sMerge[4 + g];
            const int64_t pidx = (hb_ + h) * a.nsplit + slot;
            a.part_acc[pidx * D + j] = A;
            if (j == 0) {
                a.part_ml[2 * pidx] = M;
                a.part_ml[2 * pidx + 1] = L;
            }
            // the CTA holding the unit's last chunk empties the unit's unused slots
            if (sMerge[6 + g])
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

template <int D, int NT, int NW, bool QJL, bool K8 = false>
cudaError_t launch_mma_t(const DecArgs& a, int G, cudaStream_t s) {
    using C = Cfg<D, QJL>;
    const size_t smem = (size_t)NW * kStages * C::kStageB + (size_t)NW * kStages * 8 +
                        (size_t)NW * 8 * 2 * sizeof(float) + 2 * kTabMax * sizeof(int32_t) +
                        (size_t)2 * 2 * NT * C::kKC * 32 * sizeof(uint2) + (2 * 3 * 8 + 8 * D + 8 * 2) * sizeof(float) +
                        (size_t)NW * 8 * sizeof(int64_t) + 8 * sizeof(int);
    auto kern = tq_decode_mma_kernel<D, NT, NW, QJL, K8>;
    cudaError_t e = set_smem_once<tq_decode_mma_kernel<D, NT, NW, QJL, K8>>((int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid = a.sk_ctas > 0 ? dim3((unsigned)a.sk_ctas)
                                    : dim3(a.nsplit, (unsigned)(a.Hkv * ((G + 7) / 8)), (unsigned)a.B);
    return launch_pdl(kern, grid, dim3(NW * 32), smem, s, a, G);
}

template <bool QJL>
cudaError_t launch_mma_q(int d, int G, const DecArgs& a, cudaStream_t s) {
    if (d == 64)
        return G <= 4 ? launch_mma_t<64, 1, kNW1, QJL>(a, G, s) : launch_mma_t<64, 2, kNW2, QJL>(a, G, s);
    if (d == 128) {
        // up to two heads per kv head: keys as int8 limbs (half the byte look-ups)
        if (G <= 2 && a.cb.k8) return launch_mma_t<128, 1, kNW1, QJL, true>(a, G, s);
        return G <= 4 ? launch_mma_t<128, 1, kNW1, QJL>(a, G, s) : launch_mma_t<128, 2, kNW2, QJL>(a, G, s);
    }
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
