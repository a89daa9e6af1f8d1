// Chunked-prefill attention over the packed TurboQuant cache for head_dim 128
// on the 5th-generation tensor cores (tcgen05, accumulators and the query
// operand in tensor memory), for sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com): the decode estimator (K section: 3-bit
// codes plus the 1-bit QJL residual correction; V section; hybrid V2+V3
// section: dequantisation fused into attention) for a chunk of Lq new queries
// per sequence, query i attending causally over cache tokens [0, T0 + i].
//
// A CTA owns 128 query rows (query i, head g of one kv head: row i G + g) and
// walks the cache in tiles of 64 tokens (one cache block).  With 128 rows per
// tile the contraction is dense, so the dequantised tile is built once in
// shared memory and consumed by the tensor core for all rows:
//   S[128 rows][64 tok] = [Q'hi | Q'lo | U'hi | U'lo] [Kdeq ; Kdeq ; Sgn ; Sgn]^T
//       (A in tensor memory: q' and u' of each row as fp16 hi and lo limbs,
//        K = 4 x 128; B in shared memory: the keys' fp16 centroids and the
//        sign operand +-gamma_t, both exact in fp16, so one fp32 accumulator
//        holds <q', c[idx]> + gamma <u', 2 sigma - 1>)
//   O[128 rows][128 coords] += [Phi | Plo] [Vdeq ; Vdeq]
//       (A in tensor memory: the softmax weights p * nv, scaled by 2^-6, as
//        fp16 hi and lo limbs; B in shared memory, MN-major: the values'
//        centroids, one 256-byte row per token, the coordinates in the same
//        slot order as the keys, so O's column 32 t + p is coordinate
//        slot_coord(0, t, p))
// Warp roles: warps 8-10 stage the cache blocks (bulk copies into a ring)
// and expand the codes into the B operands (three buffers, so they run up to
// two tiles ahead); warp 11 issues the mma (one thread); warps 0-7 own one
// half row each per thread (tensor-memory lane = row; warpgroup h takes
// tokens 32 h .. 32 h + 31 of a tile): they load S, apply the norms, the
// causal mask and the online softmax (the two halves of a row exchange their
// maxima through shared memory), and write P over S in tensor memory.
// S and P have two tensor-memory buffers, so the tensor core computes the
// scores of tile k + 1 while the softmax works on tile k; the mma of one
// thread run in issue order, so S(k + 2) cannot overwrite P(k) before O += P(k)
// V(k), issued earlier, has read it.  The running maximum used for P is moved
// only when it grows by more than 2^8, and then O in tensor memory is
// rescaled.  mbarriers order the roles and the tensor core; every wait is
// bounded.
#include <algorithm>
#include <vector>

#include "tq_frag.cuh"
#include "tq_tc.cuh"

namespace tqi {
namespace {

constexpr int kPD = 128;                 // head_dim
constexpr int kPT = 64;                  // tokens per tile (one cache block)
constexpr int kPRows = 128;              // query rows per CTA
constexpr int kPRing = 3;                // raw block stages
constexpr int kPBuf = 3;                 // B operand buffers
constexpr int kSoftmaxThreads = 256, kProducerThreads = 96;      // two softmax warpgroups, three producer warps
constexpr int kThreads = kSoftmaxThreads + kProducerThreads + 32;   // + the mma warp
constexpr float kRescaleLog2 = 8.f;      // move the maximum used for P only when it grows by more than this
constexpr float kPScale = 1.f / 64.f;    // P holds p nv 2^-6 (p <= 2^8, so fp16 holds it unless nv > 2^14)

struct PtcShape {
    static constexpr int kKB = 64 * 48 + 64 * 16 + 256;     // K block bytes
    static constexpr int kVB = 64 * 48 + 128;                // V block bytes
    // B buffers: keys [64 tok][128 coords] fp16, signs [64 tok][128 rows] fp16 (K-major),
    // values [64 tok][128 coords] fp16 (MN-major); 128-byte swizzled, coordinates in slot order
    static constexpr int kOffK = 0;
    static constexpr int kOffS = 16384;
    static constexpr int kOffV = 32768;
    static constexpr int kBuf = 49152;
    static constexpr int kOffScal = kPBuf * kBuf;            // per buffer: n scale log2(e) [64], nv 2^-6 [64]
    static constexpr int kOffRing = kOffScal + kPBuf * 512;
    static constexpr int kStage = kKB + kVB;
    static constexpr int kOffBar = kOffRing + kPRing * kStage;
    static constexpr int kNumBars = 16;
    static constexpr int kOffXchg = kOffBar + kNumBars * 8;  // row maxima [2 tiles][2 halves][128], sums [2][128]
    static constexpr int kOffMisc = kOffXchg + 6 * 128 * 4;
    static constexpr int kSmem = kOffMisc + 64 + 1024;       // + slack to align the base
    // tensor memory: the query operand (4 x 64 columns), S / P (two buffers), O
    static constexpr int kColA = 0;
    static constexpr int kColX = 256;                        // buffer x at kColX + 64 x
    static constexpr int kColO = 384;
    static constexpr int kAlloc = 512;
};
static_assert(PtcShape::kOffRing % 16 == 0 && PtcShape::kStage % 16 == 0, "bulk copy alignment");
static_assert(PtcShape::kSmem <= 227 * 1024, "shared memory per CTA");

// mbarriers (index into the barrier array)
enum : int {
    kBarRing = 0,     // [3] raw stage filled (bulk copy bytes)
    kBarBReady = 3,   // [3] B buffer built (96 producer arrivals)
    kBarBFree = 6,    // [3] B buffer read by S and O of its tile (commit)
    kBarSFull = 9,    // [2] S computed into buffer x (commit)
    kBarPReady = 11,  // [2] P written into buffer x (256 softmax arrivals)
    kBarODone = 13,   // O += P V of a tile done (commit)
    kBarAReady = 14,  // query operand in tensor memory (256 softmax arrivals)
    kBarDrain = 15,   // every mma issued by the mma thread done (commit, at exit)
};

constexpr int kMaxCtas = 160;            // CTAs of one launch (one per SM)

// Start of a CTA's range of the flattened (sequence, row tile, tile) space.
struct CtaStart {
    int64_t bh;   // sequence b * Hkv + h
    int32_t rt;   // row tile (rows 128 rt .. 128 rt + 127 of the sequence's Lq G rows)
    int32_t k;    // tile of the row tile's token range
};

struct PrefillTcArgs {
    DecArgs a;          // caches, workspace, scale, partials (nsplit per row), check word
    int64_t Lq, T0;     // queries per sequence in the chunk; tokens cached before it
    int64_t nrows;      // Lq G rows per sequence
    int64_t W1, W;      // tiles per sequence (over its row tiles); in all
    int G, R, nsplit;   // query heads per kv head; row tiles per sequence; partials per row
    CtaStart start[kMaxCtas];
};

// Tiles of row tile rt: tokens [0, T0 + (last row of the tile) / G + 1).
__device__ __forceinline__ int ntile_of(const PrefillTcArgs& pa, int rt) {
    const int64_t rl = (int64_t)rt * kPRows + kPRows - 1 < pa.nrows ? (int64_t)rt * kPRows + kPRows - 1 : pa.nrows - 1;
    return (int)((pa.T0 + rl / pa.G + 1 + kPT - 1) / kPT);
}
// Walks a CTA's range tile by tile: the sequence, the row tile, the tile and the row tile's length.
struct TileCursor {
    int64_t bh;
    int rt, k, nt;
    __device__ void init(const PrefillTcArgs& pa, const CtaStart& st) {
        bh = st.bh;
        rt = st.rt;
        k = st.k;
        nt = ntile_of(pa, rt);
    }
    __device__ void next(const PrefillTcArgs& pa) {
        if (++k == nt) {
            k = 0;
            if (++rt == pa.R) {
                rt = 0;
                ++bh;
            }
            nt = ntile_of(pa, rt);
        }
    }
};

// barrier id over n threads that also ORs v across them (every thread gets the result)
__device__ __forceinline__ bool bar_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
// warp-uniform bounded wait (the warp then runs warp-collective tensor-memory instructions)
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    return __all_sync(kFull, mbar_wait_bounded(bar, parity));
}

// One CTA per SM over an equal share (floor(c W / NC) .. floor((c + 1) W / NC)) of the
// flattened tiles, sequences outermost, then row tiles, then tiles of a row tile's token
// range.  A run of tiles of one row tile is a segment: the CTA loads that row tile's
// query operand, and at the segment's end writes the rows' partial (m, l, acc) into slot
// c - c_first of the row tile (c_first = the CTA holding its first tile); the CTA holding
// its last tile also fills the slots up to nsplit with empty partials.  The combine
// kernel merges the slots.
__global__ void __launch_bounds__(kThreads, 1) tq_prefill_tc_kernel(const __grid_constant__ PrefillTcArgs pa) {
    using S = PtcShape;
    const DecArgs& a = pa.a;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffMisc);
    float* scal = reinterpret_cast<float*>(sm + S::kOffScal);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int NC = (int)gridDim.x, c = (int)blockIdx.x;
    const int64_t g0 = (int64_t)c * pa.W / NC;
    const int J = (int)((int64_t)(c + 1) * pa.W / NC - g0);      // tiles of this CTA (>= 1)
    const CtaStart st0 = pa.start[c];

    if (tid == 0) {
        for (int i = 0; i < kPRing; ++i) mbar_init(bar(kBarRing + i), 1);
        for (int i = 0; i < kPBuf; ++i) {
            mbar_init(bar(kBarBReady + i), kProducerThreads);
            mbar_init(bar(kBarBFree + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kBarSFull + i), 1);
            mbar_init(bar(kBarPReady + i), kSoftmaxThreads);
        }
        mbar_init(bar(kBarODone), 1);
        mbar_init(bar(kBarAReady), kSoftmaxThreads);
        mbar_init(bar(kBarDrain), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), S::kAlloc);
        tc_relinquish();
    }
    // raw K and V blocks of the cursor's tile -> ring stage j % kPRing
    auto issue = [&](int j, const TileCursor& cu) {
        uint8_t* stg = sm + S::kOffRing + (j % kPRing) * S::kStage;
        const uint32_t br = bar(kBarRing + j % kPRing);
        const int64_t kblk = cache_block(a.ktable, a.kpool, a.NB, cu.bh, cu.k, a.err);
        const int64_t vblk = cache_block(a.vtable, a.vpool, a.NB, cu.bh, cu.k, a.err);
        mbar_expect_tx(br, (uint32_t)S::kStage);
        bulk_g2s(smem_u32(stg), a.kc + (kblk >= 0 ? kblk : 0) * S::kKB, S::kKB, br);
        bulk_g2s(smem_u32(stg + S::kKB), a.vc + (vblk >= 0 ? vblk : 0) * S::kVB, S::kVB, br);
    };
    tc_fence_before();
    __syncthreads();                       // the mbarriers are initialised before anyone uses them
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    TileCursor ci;                         // the ring's cursor (producer thread 0), kPRing tiles ahead
    if (tid == kSoftmaxThreads) {
        ci.init(pa, st0);
        for (int j = 0; j < kPRing && j < J; ++j) {
            issue(j, ci);
            ci.next(pa);
        }
    }
    pdl_wait();                            // q' and u' come from the prologue kernel

    bool failed = false;
    if (warp < 8) {
        // ======================================== softmax warps: thread = (row, half); warp w
        // reaches tensor-memory lanes 32 (w % 4) .. +31, warpgroup h = w / 4 takes tokens
        // 32 h .. 32 h + 31 of every tile and O columns 64 h .. 64 h + 63
        const int hh = warp >> 2;
        const int r = 32 * (warp & 3) + (tid & 31);
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        float* xm = reinterpret_cast<float*>(sm + S::kOffXchg);             // [2][2][128]
        float* xl = xm + 4 * 128;                                            // [2][128]
        TileCursor cs;
        cs.init(pa, st0);
        // the current segment's rows
        bool rvalid = false;
        int64_t qrow = 0, lim = 0;
        int sp = 0, seg = 0;
        bool unit_last = false;
        float m_run = -INFINITY, m_used = -INFINITY, l = 0.f;
        // query operand of row tile (bh, rt) (warpgroup 0: q', warpgroup 1: u'): column c of
        // each 64-column part holds K positions 2c, 2c + 1; K position kappa = 32 t + p is
        // coordinate (JL row) slot_coord(0, t, p)
        auto begin_segment = [&](int64_t gtile) {
            const int64_t b = cs.bh / a.Hkv, hkv = cs.bh - b * a.Hkv;
            const int64_t grow = (int64_t)cs.rt * kPRows + r;
            rvalid = grow < pa.nrows;
            const int64_t qi = rvalid ? grow / pa.G : 0, qg = rvalid ? grow % pa.G : 0;
            qrow = (b * pa.Lq + qi) * a.Hq + hkv * pa.G + qg;
            lim = rvalid ? pa.T0 + qi + 1 : 0;                 // tokens [0, lim) visible
            const int64_t gu = gtile - cs.k;                  // the row tile's first tile
            sp = c - (int)(((gu + 1) * NC - 1) / pa.W);
            m_run = m_used = -INFINITY;
            l = 0.f;
            const float* src = (hh == 0 ? a.qp : a.up) + qrow * kPD;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 16) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {
                    const int kap = 2 * (c0 + cc), t = kap >> 5, p = kap & 31;
                    const float x0 = rvalid ? src[slot_coord(0, t, p)] : 0.f;
                    const float x1 = rvalid ? src[slot_coord(0, t, p + 1)] : 0.f;
                    split_hilo(x0, x1, hi[cc], lo[cc]);
                }
                tc_st16(tl + S::kColA + 128 * hh + c0, hi);
                tc_st16(tl + S::kColA + 128 * hh + 64 + c0, lo);
            }
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kBarAReady));
        };
        // The segment's last tile jl: its P V, then the rows' partial (every softmax thread
        // gets here the same number of times; a failure seen by any of them zeroes the rows).
        auto end_segment = [&](int jl) {
            if (!failed && !warp_wait(bar(kBarODone), (uint32_t)(jl & 1))) failed = true;
            tc_fence_after();
            xl[((seg & 1) * 2 + hh) * 128 + r] = l;
            if (bar_or(2, kSoftmaxThreads, failed)) failed = true;
            // (the loads are warp-collective: every lane loads, valid rows store).  O's column
            // 32 t + p is coordinate slot_coord(0, t, p); positions 2i, 2i + 1 are adjacent
            // coordinates.
            float* acc = a.part_acc + (qrow * pa.nsplit + sp) * kPD;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t ov[32];
                tc_ld32(tl + S::kColO + 64 * hh + c0, ov);
                const int t = 2 * hh + (c0 >> 5);
                if (rvalid) {
#pragma unroll
                    for (int p = 0; p < 32; p += 2)
                        *reinterpret_cast<float2*>(acc + slot_coord(0, t, p)) =
                            failed ? make_float2(0.f, 0.f)
                                   : make_float2(__uint_as_float(ov[p]) * (1.f / kPScale),
                                                 __uint_as_float(ov[p + 1]) * (1.f / kPScale));
                }
            }
            if (rvalid) {
                if (hh == 0) {
                    a.part_ml[2 * (qrow * pa.nsplit + sp)] = failed ? -INFINITY : m_used;
                    a.part_ml[2 * (qrow * pa.nsplit + sp) + 1] =
                        failed ? 0.f : xl[((seg & 1) * 2) * 128 + r] + xl[((seg & 1) * 2 + 1) * 128 + r];
                }
                if (unit_last) {           // slots no CTA fills: empty partials
                    for (int s2 = sp + 1; s2 < pa.nsplit; ++s2) {
                        float* e = a.part_acc + (qrow * pa.nsplit + s2) * kPD + 64 * hh;
                        for (int i = 0; i < 64; i += 4) *reinterpret_cast<float4*>(e + i) = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (hh == 0) {
                            a.part_ml[2 * (qrow * pa.nsplit + s2)] = -INFINITY;
                            a.part_ml[2 * (qrow * pa.nsplit + s2) + 1] = 0.f;
                        }
                    }
                }
            }
            ++seg;
        };
        int b3 = 0, ph3 = 0;                                  // j % 3, (j / 3) & 1
        for (int j = 0; j < J; ++j) {
            const int x = j & 1;
            const uint32_t tx = tl + S::kColX + 64 * x;
            const bool first = j == 0 || cs.k == 0;
            if (first) {
                if (j > 0) end_segment(j - 1);
                if (failed) break;
                begin_segment(g0 + j);
            }
            unit_last = cs.k == cs.nt - 1;
            // A failed wait does not leave the loop at once: the two warpgroups meet at the
            // row-maximum exchange below, which also ORs their failures, and leave together.
            // (Within a warp the waits are uniform: the tensor-memory loads and stores are
            // warp-collective.)
            bool ok = !failed && warp_wait(bar(kBarSFull + x), (uint32_t)((j >> 1) & 1));
            tc_fence_after();
            uint32_t sv[32];
            tc_ld32(tx + 32 * hh, sv);
            // the tile's norms (written with its B operands)
            ok = ok && warp_wait(bar(kBarBReady + b3), (uint32_t)ph3);
            const float4* sn4 = reinterpret_cast<const float4*>(scal + b3 * 128 + 32 * hh);
            const int64_t tok0 = (int64_t)cs.k * kPT + 32 * hh;
            const int vis = lim - tok0 >= 32 ? 32 : (int)(lim > tok0 ? lim - tok0 : 0);
            float sc[32];
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
                const float4 n4 = sn4[t4];
                sc[4 * t4 + 0] = __uint_as_float(sv[4 * t4 + 0]) * n4.x;
                sc[4 * t4 + 1] = __uint_as_float(sv[4 * t4 + 1]) * n4.y;
                sc[4 * t4 + 2] = __uint_as_float(sv[4 * t4 + 2]) * n4.z;
                sc[4 * t4 + 3] = __uint_as_float(sv[4 * t4 + 3]) * n4.w;
            }
            if (vis < 32) {
#pragma unroll
                for (int t = 0; t < 32; ++t)
                    if (t >= vis) sc[t] = -INFINITY;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int t = 0; t < 32; ++t) mt = fmaxf(mt, sc[t]);
            xm[(x * 2 + hh) * 128 + r] = mt;
            if (bar_or(2, kSoftmaxThreads, !ok)) { failed = true; break; }
            mt = fmaxf(mt, xm[(x * 2 + (hh ^ 1)) * 128 + r]);
            const float m_new = fmaxf(m_run, mt);             // the same in both halves of the row
            m_run = m_new;
            // O += P(j-1) V(j-1) must be done before O is rescaled (and, for the barrier's
            // phase tracking, every tile but a segment's first waits for it: there the
            // segment's end waited); a failure here is acted on at the next exchange
            if (!first && !warp_wait(bar(kBarODone), (uint32_t)((j - 1) & 1))) failed = true;
            tc_fence_after();
            // Move this row's reference maximum when it grew by more than 2^8; O is rescaled
            // by each warp as a whole, with factor 1 on the rows that keep theirs.
            float f = 1.f;
            if (m_new != -INFINITY && (m_used == -INFINITY || m_new > m_used + kRescaleLog2)) {
                if (m_used != -INFINITY) {                    // O and l were built on m_used
                    f = fast_exp2(m_used - m_new);
                    l *= f;
                }
                m_used = m_new;
            }
            if (__any_sync(kFull, f != 1.f)) {
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t ov[32];
                    tc_ld32(tl + S::kColO + 64 * hh + c0, ov);
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) ov[cc] = __float_as_uint(__uint_as_float(ov[cc]) * f);
                    tc_st32(tl + S::kColO + 64 * hh + c0, ov);
                }
            }
            // P = 2^(s - m_used) nv 2^-6 over S: hi limbs in columns 0-31, lo limbs in
            // 32-63 (tokens 2c, 2c + 1; this half: columns 16 h .. 16 h + 15 of each).
            // A row that has seen nothing yet (an absent row) keeps P = 0.
            const float mu = m_used == -INFINITY ? 0.f : m_used;
            uint32_t ph[16], plo[16];
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 v4 = sn4[16 + c4];
                const float p0 = fast_exp2(sc[4 * c4 + 0] - mu), p1 = fast_exp2(sc[4 * c4 + 1] - mu);
                const float p2 = fast_exp2(sc[4 * c4 + 2] - mu), p3 = fast_exp2(sc[4 * c4 + 3] - mu);
                l += (p0 + p1) + (p2 + p3);
                split_hilo(p0 * v4.x, p1 * v4.y, ph[2 * c4], plo[2 * c4]);
                split_hilo(p2 * v4.z, p3 * v4.w, ph[2 * c4 + 1], plo[2 * c4 + 1]);
            }
            tc_st16(tx + 16 * hh, ph);
            tc_st16(tx + 32 + 16 * hh, plo);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kBarPReady + x));
            if (++b3 == kPBuf) { b3 = 0; ph3 ^= 1; }
            cs.next(pa);
        }
        // the last segment (or, after a failure, the segment in progress: its rows are zeroed)
        end_segment(J - 1);
        pdl_trigger();
        if (failed) atomicExch(a.err, 1);
    } else if (warp < 11) {
        // ======================================== producer warps: thread pt of 96; item
        // (token tau, slot group t) of the tile's 256
        const int pt = tid - kSoftmaxThreads;
        const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};
        const uint32_t* pw = a.cb.pow2;
        int n_ring = J < kPRing ? J : kPRing;
        int b3 = 0, ph3 = 0;                                  // j % 3 (B buffer and ring stage), (j / 3) & 1
        for (int j = 0; j < J; ++j) {
            const uint8_t* stg = sm + S::kOffRing + b3 * S::kStage;
            // every producer thread reaches the barrier below whatever happens, so that
            // the decision to stop is the same for all of them
            bool f = !mbar_wait_bounded(bar(kBarRing + b3), (uint32_t)ph3);
            // buffer b3 was last read by the mma of tile j - 3
            if (!f && j >= kPBuf) f = !mbar_wait_bounded(bar(kBarBFree + b3), (uint32_t)(ph3 ^ 1));
            if (!f) {
                uint8_t* Kt = sm + b3 * S::kBuf + S::kOffK;
                uint8_t* Sg = sm + b3 * S::kBuf + S::kOffS;
                uint8_t* Vt = sm + b3 * S::kBuf + S::kOffV;
                const uint8_t* kb = stg;
                const uint8_t* vb = stg + S::kKB;
                for (int it = pt; it < 4 * kPT; it += kProducerThreads) {
                    const int tau = it >> 2, t = it & 3;
                    const uint32_t gam = *reinterpret_cast<const uint16_t*>(kb + 64 * 64 + 128 + 2 * tau);
                    const uint32_t g2 = gam | (gam << 16);
                    uint32_t sel[4], vsel[4];
                    code_selectors(kb + tau * 48 + 12 * t, pw, sel);
                    code_selectors(vb + tau * 48 + 12 * t, pw, vsel);
                    // keys: K positions 32 t .. 32 t + 31 of row tau (four 16-byte chunks)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t xk[4];
                        dequant4(sel_for(sel, pw, 2 * c), lut, xk[0], xk[1]);
                        dequant4(sel_for(sel, pw, 2 * c + 1), lut, xk[2], xk[3]);
                        *reinterpret_cast<uint4*>(Kt + sw128_byte(tau, 2 * (32 * t + 8 * c), kPT)) =
                            make_uint4(xk[0], xk[1], xk[2], xk[3]);
                    }
                    // signs: +-gamma for JL rows at positions 2q, 2q + 1 (sign bits q, 16 + q)
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(kb + 64 * 48 + tau * 16 + 4 * t);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t xs[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int q = 4 * c + e;
                            const uint32_t sh = shl_m(w, pw, 15 - q);         // bits q, 16 + q -> 15, 31
                            xs[e] = g2 ^ (~sh & 0x80008000u);                 // sigma = 0: -gamma
                        }
                        *reinterpret_cast<uint4*>(Sg + sw128_byte(tau, 2 * (32 * t + 8 * c), kPT)) =
                            make_uint4(xs[0], xs[1], xs[2], xs[3]);
                    }
                    // values: row = token tau, positions 32 t .. 32 t + 31 (slot order, as the keys)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t xv[4];
                        dequant4(sel_for(vsel, pw, 2 * c), lut, xv[0], xv[1]);
                        dequant4(sel_for(vsel, pw, 2 * c + 1), lut, xv[2], xv[3]);
                        *reinterpret_cast<uint4*>(Vt + sw128_byte(tau, 2 * (32 * t + 8 * c), kPT)) =
                            make_uint4(xv[0], xv[1], xv[2], xv[3]);
                    }
                    if (t == 0) {          // the tile's per-token factors for the softmax
                        scal[b3 * 128 + tau] =
                            __half2float(*reinterpret_cast<const __half*>(kb + 64 * 64 + 2 * tau)) * a.scale_log2;
                        scal[b3 * 128 + 64 + tau] =
                            __half2float(*reinterpret_cast<const __half*>(vb + 64 * 48 + 2 * tau)) * kPScale;
                    }
                }
                fence_proxy_async();       // B operands written by threads, read by the tensor core
                mbar_arrive(bar(kBarBReady + b3));
            }
            // every producer thread is done with stage b3 (or one gave up)
            if (bar_or(1, kProducerThreads, f)) { failed = true; break; }
            if (pt == 0 && j + kPRing < J) {
                issue(j + kPRing, ci);
                ci.next(pa);
                ++n_ring;
            }
            if (++b3 == kPBuf) { b3 = 0; ph3 ^= 1; }
        }
        if (pt == 0) {
            // only the last copy into each stage can still be in flight: an earlier one was
            // waited for before its stage was refilled (and a wait on an older phase of the
            // same parity as the current one would not return)
            for (int j = n_ring > kPRing ? n_ring - kPRing : 0; j < n_ring; ++j)
                mbar_wait_bounded(bar(kBarRing + j % kPRing), (uint32_t)((j / kPRing) & 1));
            if (failed) atomicExch(a.err, 1);
        }
    } else if ((tid & 31) == 0) {
        // ======================================== the mma thread
        constexpr uint32_t kIdS = idesc_f16(128, kPT), kIdO = idesc_f16_bmn(128, kPD);
        auto mma_o = [&](int j, bool seg_first) {   // O (+)= P(j) V(j)
            const uint32_t vd = sbase + (uint32_t)((j % kPBuf) * S::kBuf + S::kOffV);
            const uint32_t pa_t = tmem + S::kColX + 64 * (j & 1);
            // K step s: tokens 16 (s % 4) .. + 15 (two 8-token atoms); the coordinates
            // 0-63 and 64-127 are the two halves of each token row, kPT * 128 bytes apart
#pragma unroll
            for (int s = 0; s < 8; ++s)
                tc_mma_f16_ts(tmem + S::kColO, pa_t + 8 * s,
                              sw128_desc_mn(vd + 2048 * (s & 3), (uint32_t)(kPT * 128), 1024u), kIdO,
                              (!seg_first || s > 0) ? 1u : 0u);
            tc_commit(bar(kBarODone));
            tc_commit(bar(kBarBFree + j % kPBuf));
        };
        TileCursor cm;
        cm.init(pa, st0);
        bool ok = true;
        int b3 = 0, ph3 = 0, seg = 0;
        int po = -1;                       // tile whose O mma is pending (its P not yet waited for)
        bool po_first = false;
        auto flush_o = [&]() -> bool {     // P(po) is written: O += P(po) V(po)
            if (po < 0) return true;
            if (!mbar_wait_bounded(bar(kBarPReady + (po & 1)), (uint32_t)((po >> 1) & 1))) return false;
            tc_fence_after();
            mma_o(po, po_first);
            po = -1;
            return true;
        };
        for (int j = 0; j < J; ++j) {
            const bool first = j == 0 || cm.k == 0;
            if (first) {                   // a new row tile: its query operand replaces the last one
                if (!(ok = flush_o())) break;
                if (!(ok = mbar_wait_bounded(bar(kBarAReady), (uint32_t)(seg & 1)))) break;
                ++seg;
            }
            // S(j) = [Q' | U'] [K ; K ; Sg ; Sg]^T into buffer j & 1 (its P(j - 2) was read by
            // the O mma issued before this one)
            if (!(ok = mbar_wait_bounded(bar(kBarBReady + b3), (uint32_t)ph3))) break;
            tc_fence_after();
            const uint32_t kd = sbase + (uint32_t)(b3 * S::kBuf + S::kOffK);
            const uint32_t sd = sbase + (uint32_t)(b3 * S::kBuf + S::kOffS);
            const uint32_t xd = tmem + S::kColX + 64 * (j & 1);
#pragma unroll
            for (int s = 0; s < 32; ++s) {
                const int ss = s & 7;
                const uint32_t base = s < 16 ? kd : sd;
                const uint32_t addr = base + (uint32_t)((ss >> 2) * (kPT * 128) + (ss & 3) * 32);
                tc_mma_f16_ts(xd, tmem + S::kColA + 8 * s, sw128_desc(addr), kIdS, s > 0 ? 1u : 0u);
            }
            tc_commit(bar(kBarSFull + (j & 1)));
            if (!(ok = flush_o())) break;  // O += P(j - 1) V(j - 1)
            po = j;
            po_first = first;
            if (++b3 == kPBuf) { b3 = 0; ph3 ^= 1; }
            cm.next(pa);
        }
        if (ok) ok = flush_o();
        // every mma this thread issued is done before tensor memory is released
        tc_commit(bar(kBarDrain));
        mbar_wait_bounded(bar(kBarDrain), 0u);
        if (!ok) atomicExch(a.err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, S::kAlloc);
    }
}

}  // namespace

int prefill_tc_split_cap(int num_sms, int64_t rows) {
    const int64_t units = (rows + kPRows - 1) / kPRows > 0 ? (rows + kPRows - 1) / kPRows : 1;
    int64_t cap = (4 * (int64_t)num_sms + units - 1) / units;
    return (int)(cap < 3 ? 3 : cap > 64 ? 64 : cap);
}

cudaError_t launch_prefill_tc(int G, const DecArgs& a, int64_t Lq, int64_t T0, int num_sms, int split_cap,
                              int* nsplit_out, cudaStream_t s) {
    PrefillTcArgs pa{};
    pa.a = a;
    pa.Lq = Lq;
    pa.T0 = T0;
    pa.G = G;
    pa.nrows = Lq * G;
    pa.R = (int)((pa.nrows + kPRows - 1) / kPRows);
    auto ntile = [&](int64_t rt) {
        const int64_t rl = rt * kPRows + kPRows - 1 < pa.nrows ? rt * kPRows + kPRows - 1 : pa.nrows - 1;
        return (T0 + rl / G + 1 + kPT - 1) / kPT;
    };
    static thread_local std::vector<int64_t> prefix;                 // tiles before row tile rt
    prefix.assign((size_t)pa.R + 1, 0);
    for (int rt = 0; rt < pa.R; ++rt) prefix[rt + 1] = prefix[rt] + ntile(rt);
    pa.W1 = prefix[pa.R];
    pa.W = a.B * a.Hkv * pa.W1;
    const int64_t ntmax = ntile(pa.R - 1);
    // CTAs: one per SM, at least 4 tiles each, and no more partials per row than the workspace
    // holds (a row tile of n tiles meets at most ceil((n - 1) / floor(W / NC)) + 1 CTAs)
    int64_t NC = num_sms < kMaxCtas ? num_sms : kMaxCtas;
    if (NC > pa.W / 4) NC = pa.W / 4 > 0 ? pa.W / 4 : 1;
    int64_t nsplit = 0;
    for (;; --NC) {
        const int64_t per = pa.W / NC;
        nsplit = (ntmax - 1 + per - 1) / per + 1;
        if (nsplit > NC) nsplit = NC;
        if (nsplit <= split_cap || NC == 1) break;
    }
    pa.nsplit = (int)nsplit;
    for (int64_t c = 0; c < NC; ++c) {
        const int64_t g0 = c * pa.W / NC;
        const int64_t bh = g0 / pa.W1, rem = g0 - bh * pa.W1;
        const int rt = (int)(std::upper_bound(prefix.begin(), prefix.end(), rem) - prefix.begin()) - 1;
        pa.start[c] = CtaStart{bh, rt, (int32_t)(rem - prefix[rt])};
    }
    *nsplit_out = pa.nsplit;
    constexpr int smem = PtcShape::kSmem;
    cudaError_t e = set_smem_once<tq_prefill_tc_kernel>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(tq_prefill_tc_kernel, dim3((unsigned)NC), dim3(kThreads), smem, s, pa);
}

}  // namespace tqi
