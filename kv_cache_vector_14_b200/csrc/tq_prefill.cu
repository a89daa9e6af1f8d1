// Chunked-prefill attention over the packed TurboQuant cache (head_dim 64, 128
// and 256), for sm_100a: a chunk of Lq new queries per sequence, query i attending
// causally over cache tokens [0, T0 + i] (the chunk's own K/V already
// appended at T0 .. T0 + Lq - 1).
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com): the same estimator as decode (K section
// and hybrid V2+V3 section), per query row q and cached token t:
//   s = scale * n_t * (<q', c[idx_t]> + gamma_t * <u', 2 sigma_t - 1>),  u' = sqrt(pi/2)/m * S q'
//   acc += softmax weight * nv_t * c[idxv_t]   (rotated domain)
// With many queries per kv head the contraction is dense, so the roles of the
// decode kernel flip: query rows (query i, head g of the kv group) are the M
// dimension and tokens the N dimension of mma.sync tiles.  A warp owns 16
// query rows; for each 16-token tile it dequantises the keys straight into B
// fragments (lane (g, t) expands token g's slot t: the coordinates an
// m16n8k16 B fragment needs), so one dequantisation serves 16 rows:
//   S[16 rows][8 tok] += Q'[16 rows][16 coords] Kdeq^T (fp16 hi and lo limbs of q')
//   Z[16 rows][8 tok] += U'[16 rows][32 rows of S] Sgn^T (int8: -128 sigma bytes,
//                        u' of each row as 16-bit fixed point in two byte limbs)
//   O[16 rows][8 coords] += P[16 rows][16 tok] Vdeq (P from the score
//                        accumulators, fp16 hi and lo limbs of p * nv;
//                        Vdeq^T from the same expansion plus movmatrix)
// with an online softmax per row and the causal mask per (row, token).  The
// rotated-domain accumulators and (max, sum) of every row are written as a
// single split, which the decode's combine kernel normalises and transforms
// back (D H).  Each warp streams the chunk's cache through its own ring of
// bulk copies (the four warps of a CTA read the same blocks; the repeats are
// served from L2).
#include <type_traits>

#include "tq_frag.cuh"

namespace tqi {
namespace {

constexpr int kPW = 4;                         // warps per CTA, 16 query rows each
constexpr int kPRows = 16 * kPW;
constexpr float kQfix = 32000.f;               // u' fixed-point scale

// Shared memory per CTA: per warp a ring of staged chunks, the fp16 q'
// fragments [k-step][limb][lane] and the int8 u' fragments [block][limb][lane].
template <int D>
struct PShape {
    using PC = Cfg<D, true>;
    static constexpr int kKC = D / 16;         // 16-coordinate k-steps
    static constexpr int kKB = D / 32;         // 32-row sign blocks
    static constexpr size_t kRing = (size_t)kPW * kStages * PC::kStageB;
    static constexpr size_t kQa = (size_t)kPW * kKC * 2 * 32 * 16;
    static constexpr size_t kUa = (size_t)kPW * kKB * 2 * 32 * 16;
    static constexpr size_t kSmem = kRing + kQa + kUa + (size_t)kPW * kStages * 8;
};

struct PrefillArgs {
    DecArgs a;          // caches, workspace, scale, partials (one split), check word
    int64_t Lq, T0;     // queries per sequence in the chunk; tokens cached before it
    int G;              // query heads per kv head
};

template <int D>
__global__ void __launch_bounds__(kPW * 32) tq_prefill_mma_kernel(const PrefillArgs pa) {
    using PC = Cfg<D, true>;
    constexpr int kPD = D;
    constexpr int kPKC = PShape<D>::kKC, kPKB = PShape<D>::kKB;
    constexpr int kVKC = D == 256 ? 8 : kPKC;            // 16-coordinate value tiles of this CTA
    constexpr size_t kPRing = PShape<D>::kRing, kPQa = PShape<D>::kQa, kPUa = PShape<D>::kUa;
    const DecArgs& a = pa.a;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, tq4 = lane & 3;
    uint8_t* ring = smem + (size_t)warp * kStages * PC::kStageB;
    uint4* qa = reinterpret_cast<uint4*>(smem + kPRing) + (size_t)warp * kPKC * 2 * 32;
    uint4* ua = reinterpret_cast<uint4*>(smem + kPRing + kPQa) + (size_t)warp * kPKB * 2 * 32;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPRing + kPQa + kPUa);
    const int hkv = blockIdx.y, b = blockIdx.z;
    const int G = pa.G;
    const int64_t nrows = pa.Lq * G;
    // head_dim 256: CTA pairs share their rows, each accumulating one half of the
    // value coordinates (both compute the scores)
    const int vh = D == 256 ? (int)(blockIdx.x & 1) : 0;
    const int64_t row0 = (int64_t)(D == 256 ? blockIdx.x >> 1 : blockIdx.x) * kPRows + 16 * warp;   // this warp's first row
    const int64_t seq = (int64_t)b * a.Hkv + hkv;
    const int64_t kbb = block_bytes(kPD, true), vbb = block_bytes(kPD, false);

    // rows r = i G + g (query i of the chunk, head g of the group); this lane's rows g and g + 8
    int64_t qrow[2];
    int64_t lim[2];                       // tokens visible to the row: [0, T0 + i]
    bool rvalid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t r = row0 + gr + 8 * h;
        rvalid[h] = r < nrows;
        const int64_t i = rvalid[h] ? r / G : 0, g = rvalid[h] ? r % G : 0;
        qrow[h] = ((int64_t)b * pa.Lq + i) * a.Hq + (int64_t)hkv * G + g;
        lim[h] = rvalid[h] ? pa.T0 + i + 1 : 0;
    }
    // tokens this warp needs: up to the last query among its 16 rows
    const int64_t rlast = (row0 + 15 < nrows ? row0 + 15 : nrows - 1);
    const int64_t tend = row0 < nrows ? pa.T0 + rlast / G + 1 : 0;
    const int nmine = (int)((tend + PC::kChunk - 1) / PC::kChunk);

    if (lane == 0)
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[warp * kStages + s]), 1);
    fence_mbar_init();
    __syncwarp();

    auto issue = [&](int i) {
        const int64_t t0 = (int64_t)i * PC::kChunk;
        const int64_t kblk = cache_block(a.ktable, a.kpool, a.NB, seq, t0 >> 6, a.err);
        const int64_t vblk = cache_block(a.vtable, a.vpool, a.NB, seq, t0 >> 6, a.err);
        const int sub = (int)((t0 & 63) / PC::kChunk);
        const uint8_t* kb = a.kc + (kblk >= 0 ? kblk : 0) * kbb;     // a bad table entry reads block 0
        const uint8_t* vb = a.vc + (vblk >= 0 ? vblk : 0) * vbb;
        uint8_t* st = ring + (i % kStages) * PC::kStageB;
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        constexpr int cb = PC::kCodeB, sb = PC::kSignB, ch = PC::kChunk;
        mbar_expect_tx(bar, PC::kStageB);
        bulk_g2s(smem_u32(st + PC::kOffKc), kb + sub * ch * cb, ch * cb, bar);
        bulk_g2s(smem_u32(st + PC::kOffKs), kb + 64 * cb + sub * ch * sb, ch * sb, bar);
        bulk_g2s(smem_u32(st + PC::kOffKn), kb + 64 * (cb + sb) + sub * 2 * ch, 2 * ch, bar);
        bulk_g2s(smem_u32(st + PC::kOffKg), kb + 64 * (cb + sb) + 128 + sub * 2 * ch, 2 * ch, bar);
        bulk_g2s(smem_u32(st + PC::kOffVc), vb + sub * ch * cb, ch * cb, bar);
        bulk_g2s(smem_u32(st + PC::kOffVn), vb + 64 * cb + sub * 2 * ch, 2 * ch, bar);
    };
    if (lane == 0)
        for (int i = 0; i < kStages && i < nmine; ++i) issue(i);
    pdl_wait();                           // q' and u' come from the prologue kernel

    // ---- A fragments of this warp's rows.  q' (m16n8k16, row-major A): a0 = row g,
    // coordinates 16 kc + 2t, +1; a1 = row g + 8, same; a2/a3 = coordinates +8, +9.
    // u' (m16n8k32): byte e of a0/a1 (a2/a3) in block kb is u_int of the JL row whose
    // sign sits at bit 8 e + 7 - 2 (kb % 4) (8 e + 6 - 2 (kb % 4)) of slot word tq4.
    // (d = 64: the slot's sign halfword h is widened to h | h << 20, see token_signs)
    auto row_of = [&](int kb, int half, int e) {
        const int bit = 8 * e + 7 - 2 * (kb & 3) - half;
        if constexpr (D == 64) return slot_coord(0, tq4, e < 2 ? bit : bit - 20);
        return slot_coord(kb >> 2, tq4, bit < 16 ? 2 * bit : 2 * (bit - 16) + 1);
    };
    float fS[2], uS[2];
    {
        const float* q0 = a.qp + qrow[0] * kPD;
        const float* q1 = a.qp + qrow[1] * kPD;
#pragma unroll
        for (int kc = 0; kc < kPKC; ++kc) {
            const int c = 16 * kc + 2 * tq4;
            float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (rvalid[0]) { x[0] = q0[c]; x[1] = q0[c + 1]; x[4] = q0[c + 8]; x[5] = q0[c + 9]; }
            if (rvalid[1]) { x[2] = q1[c]; x[3] = q1[c + 1]; x[6] = q1[c + 8]; x[7] = q1[c + 9]; }
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) split_hilo(x[2 * r], x[2 * r + 1], hi[r], lo[r]);
            qa[(kc * 2 + 0) * 32 + lane] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            qa[(kc * 2 + 1) * 32 + lane] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        float um[2] = {0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float* u = a.up + qrow[h] * kPD;
            if (rvalid[h])
                for (int kb = 0; kb < kPKB; ++kb)
                    for (int hf = 0; hf < 2; ++hf)
                        for (int e = 0; e < 4; ++e) um[h] = fmaxf(um[h], fabsf(u[row_of(kb, hf, e)]));
            um[h] = fmaxf(um[h], __shfl_xor_sync(kFull, um[h], 1));
            um[h] = fmaxf(um[h], __shfl_xor_sync(kFull, um[h], 2));
        }
        int usum[2] = {0, 0};
        const float fu[2] = {um[0] > 0.f ? kQfix / um[0] : 0.f, um[1] > 0.f ? kQfix / um[1] : 0.f};
#pragma unroll
        for (int kb = 0; kb < kPKB; ++kb) {
            uint32_t w[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};     // [limb][a0..a3]
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float* u = a.up + qrow[h] * kPD;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ui = rvalid[h] ? __float2int_rn(u[row_of(kb, hf, e)] * fu[h]) : 0;
                        const int lo = ((ui + 128) & 255) - 128;
                        const int hi = (ui - lo) >> 8;
                        w[0][2 * hf + h] |= (uint32_t)(uint8_t)(int8_t)hi << (8 * e);
                        w[1][2 * hf + h] |= (uint32_t)(uint8_t)(int8_t)lo << (8 * e);
                        usum[h] += ui;
                    }
            }
            ua[(kb * 2 + 0) * 32 + lane] = make_uint4(w[0][0], w[0][1], w[0][2], w[0][3]);
            ua[(kb * 2 + 1) * 32 + lane] = make_uint4(w[1][0], w[1][1], w[1][2], w[1][3]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            usum[h] += __shfl_xor_sync(kFull, usum[h], 1);
            usum[h] += __shfl_xor_sync(kFull, usum[h], 2);
            fS[h] = a.scale_log2 * (um[h] / kQfix) * (1.f / 64.f);
            uS[h] = 64.f * (float)usum[h];
        }
    }
    __syncwarp();

    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
    const uint32_t* pw = a.cb.pow2;
    [[maybe_unused]] const uint32_t m64 = pw[20] | 1u;    // d = 64 sign widening factor
    float o[2 * kVKC][4];                 // coordinate n-tiles of 8: rows g (0, 1), g + 8 (2, 3)
#pragma unroll
    for (int nc = 0; nc < 2 * kVKC; ++nc) o[nc][0] = o[nc][1] = o[nc][2] = o[nc][3] = 0.f;
    float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
    bool failed = false;

    for (int i = 0; i < nmine; ++i) {
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        const bool ok = mbar_wait_bounded(bar, (uint32_t)((i / kStages) & 1));
        if (__any_sync(kFull, !ok)) {         // warp-uniform: no lane may run on alone into mma.sync
            failed = true;
            if (lane == 0) atomicExch(a.err, 1);
            for (int j = i; j < nmine && j < i + kStages; ++j)
                mbar_wait_bounded(smem_u32(&bars[warp * kStages + (j % kStages)]), (uint32_t)((j / kStages) & 1));
            break;
        }
        const uint8_t* st = ring + (i % kStages) * PC::kStageB;
        const int64_t tok0 = (int64_t)i * PC::kChunk;
#pragma unroll
        for (int kt = 0; kt < PC::kTiles; ++kt) {
            // ---------------- scores of 16 rows x 16 tokens (two n-tiles of 8)
            const int tA = kt * 16 + gr, tB = tA + 8;            // B-fragment tokens of n-tiles 0, 1
            uint32_t selA[PC::kS][4], selB[PC::kS][4], sgA[PC::kS], sgB[PC::kS];
#pragma unroll
            for (int sl = 0; sl < PC::kS; ++sl) {                // 128-coordinate slices
                token_selectors<D>(st + PC::kOffKc + tA * PC::kCodeB, sl, tq4, pw, selA[sl]);
                token_selectors<D>(st + PC::kOffKc + tB * PC::kCodeB, sl, tq4, pw, selB[sl]);
                sgA[sl] = token_signs<D>(st + PC::kOffKs + tA * PC::kSignB, sl, tq4, m64);
                sgB[sl] = token_signs<D>(st + PC::kOffKs + tB * PC::kSignB, sl, tq4, m64);
            }
            float sacc[2][4];
            int iacc[2][2][4];                                  // [n-tile][u' limb]
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    sacc[nt][c] = 0.f;
                    iacc[nt][0][c] = iacc[nt][1][c] = 0;
                }
#pragma unroll
            for (int kc = 0; kc < kPKC; ++kc) {
                uint32_t kA0, kA1, kB0, kB1;
                dequant4(sel_for(selA[kc >> 3], pw, kc & 7), lut, kA0, kA1);
                dequant4(sel_for(selB[kc >> 3], pw, kc & 7), lut, kB0, kB1);
                const uint4 ah = qa[(kc * 2 + 0) * 32 + lane], al = qa[(kc * 2 + 1) * 32 + lane];
                const uint32_t aH[4] = {ah.x, ah.y, ah.z, ah.w}, aL[4] = {al.x, al.y, al.z, al.w};
                mma16816(sacc[0], aH, kA0, kA1);
                mma16816(sacc[0], aL, kA0, kA1);
                mma16816(sacc[1], aH, kB0, kB1);
                mma16816(sacc[1], aL, kB0, kB1);
                if ((kc & 1) == 0) {                            // one 32-row sign block per two k-steps
                    const int kb = kc >> 1, k4 = kb & 3;
                    const uint32_t bA0 = shl_m(sgA[kb >> 2], pw, 2 * k4) & 0x80808080u;
                    const uint32_t bA1 = shl_m(sgA[kb >> 2], pw, 2 * k4 + 1) & 0x80808080u;
                    const uint32_t bB0 = shl_m(sgB[kb >> 2], pw, 2 * k4) & 0x80808080u;
                    const uint32_t bB1 = shl_m(sgB[kb >> 2], pw, 2 * k4 + 1) & 0x80808080u;
                    const uint4 uh = ua[(kb * 2 + 0) * 32 + lane], ul = ua[(kb * 2 + 1) * 32 + lane];
                    const uint32_t uH[4] = {uh.x, uh.y, uh.z, uh.w}, uL[4] = {ul.x, ul.y, ul.z, ul.w};
                    imma16832(iacc[0][0], uH, bA0, bA1);
                    imma16832(iacc[0][1], uL, bA0, bA1);
                    imma16832(iacc[1][0], uH, bB0, bB1);
                    imma16832(iacc[1][1], uL, bB0, bB1);
                }
            }
            // element c of n-tile nt: row g (c < 2) or g + 8, token 8 nt + 2 tq4 + (c & 1)
            float s[2][4];
            bool vis[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int h = c >> 1;
                    const int tt = kt * 16 + 8 * nt + 2 * tq4 + (c & 1);
                    const float nk = __half2float(*reinterpret_cast<const __half*>(st + PC::kOffKn + 2 * tt));
                    const float gk = __half2float(*reinterpret_cast<const __half*>(st + PC::kOffKg + 2 * tt));
                    const float z = (float)(iacc[nt][0][c] * 256 + iacc[nt][1][c]) + uS[h];
                    vis[nt][c] = tok0 + tt < lim[h];
                    s[nt][c] = vis[nt][c] ? nk * fmaf(-gk * fS[h], z, a.scale_log2 * sacc[nt][c]) : -INFINITY;
                }
            // ---------------- online softmax per row (the quad's four lanes share rows g, g + 8)
            float pv[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mt = fmaxf(fmaxf(s[0][2 * h], s[0][2 * h + 1]), fmaxf(s[1][2 * h], s[1][2 * h + 1]));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 1));
                mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 2));
                const float mnew = fmaxf(mrun[h], mt);
                if (__any_sync(kFull, mnew > mrun[h])) {
                    const float corr = (mnew == -INFINITY) ? 1.f : fast_exp2(mrun[h] - mnew);
                    lrun[h] *= corr;
#pragma unroll
                    for (int nc = 0; nc < 2 * kVKC; ++nc) {
                        o[nc][2 * h] *= corr;
                        o[nc][2 * h + 1] *= corr;
                    }
                    mrun[h] = mnew;
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int c = 2 * h + j;
                        const float p = vis[nt][c] ? fast_exp2(s[nt][c] - mrun[h]) : 0.f;
                        lrun[h] += p;
                        const int tt = kt * 16 + 8 * nt + 2 * tq4 + j;
                        const float nv = __half2float(*reinterpret_cast<const __half*>(st + PC::kOffVn + 2 * tt));
                        pv[nt][c] = vis[nt][c] ? p * nv : 0.f;
                    }
            }
            // P as the A operand (k = tokens): a0 = row g, tokens 2t, 2t+1; a1 = row g + 8;
            // a2/a3 = tokens 8 + 2t, 9 + 2t; fp16 hi and lo limbs
            uint32_t pH[4], pL[4];
            split_hilo(pv[0][0], pv[0][1], pH[0], pL[0]);
            split_hilo(pv[0][2], pv[0][3], pH[1], pL[1]);
            split_hilo(pv[1][0], pv[1][1], pH[2], pL[2]);
            split_hilo(pv[1][2], pv[1][3], pH[3], pL[3]);
            // ---------------- values: O[16 rows][8 coords] += P Vdeq, Vdeq^T by movmatrix
            token_selectors<D>(st + PC::kOffVc + tA * PC::kCodeB, vh, tq4, pw, selA[0]);
            token_selectors<D>(st + PC::kOffVc + tB * PC::kCodeB, vh, tq4, pw, selB[0]);
#pragma unroll
            for (int kc = 0; kc < kVKC; ++kc) {
                uint32_t x0, x1, y0, y1;
                dequant4(sel_for(selA[0], pw, kc), lut, x0, x1);   // tokens 0..7 of the tile
                dequant4(sel_for(selB[0], pw, kc), lut, y0, y1);   // tokens 8..15
                const uint32_t mx0 = movmatrix_t(x0), mx1 = movmatrix_t(x1);
                const uint32_t my0 = movmatrix_t(y0), my1 = movmatrix_t(y1);
                mma16816(o[2 * kc], pH, mx0, my0);
                mma16816(o[2 * kc], pL, mx0, my0);
                mma16816(o[2 * kc + 1], pH, mx1, my1);
                mma16816(o[2 * kc + 1], pL, mx1, my1);
            }
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nmine) {
            fence_proxy_async();
            issue(i + kStages);
        }
    }
    pdl_trigger();                        // the combine kernel may start launching
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (failed) { mrun[h] = -INFINITY; lrun[h] = 0.f; }
        lrun[h] += __shfl_xor_sync(kFull, lrun[h], 1);
        lrun[h] += __shfl_xor_sync(kFull, lrun[h], 2);
        if (!rvalid[h]) continue;
        float* acc = a.part_acc + qrow[h] * kPD + 128 * vh;   // one split per row
#pragma unroll
        for (int nc = 0; nc < 2 * kVKC; ++nc)
            *reinterpret_cast<float2*>(acc + 8 * nc + 2 * tq4) = make_float2(o[nc][2 * h], o[nc][2 * h + 1]);
        if (tq4 == 0 && vh == 0) {
            a.part_ml[2 * qrow[h]] = mrun[h];
            a.part_ml[2 * qrow[h] + 1] = lrun[h];
        }
    }
}

template <int D>
cudaError_t launch_prefill_d(int G, const DecArgs& a, int64_t Lq, int64_t T0, cudaStream_t s) {
    constexpr size_t smem = PShape<D>::kSmem;
    PrefillArgs pa{a, Lq, T0, G};
    const int64_t tiles = (Lq * G + kPRows - 1) / kPRows;
    cudaError_t e = set_smem_once<tq_prefill_mma_kernel<D>>((int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(tiles * (D == 256 ? 2 : 1)), (unsigned)a.Hkv, (unsigned)a.B);
    return launch_pdl(tq_prefill_mma_kernel<D>, grid, dim3(kPW * 32), smem, s, pa);
}

}  // namespace

cudaError_t launch_prefill(int d, int G, const DecArgs& a, int64_t Lq, int64_t T0, cudaStream_t s) {
    if (!head_dim_ok(d) || G < 1) return cudaErrorInvalidValue;
    if (a.B * a.Hkv == 0 || Lq == 0) return cudaSuccess;
    if (d == 64) return launch_prefill_d<64>(G, a, Lq, T0, s);
    return d == 256 ? launch_prefill_d<256>(G, a, Lq, T0, s) : cudaErrorInvalidValue;
}

}  // namespace tqi
