// TurboQuant K/V encode for head_dim 128 and 64 with the random rotation on
// the 5th-generation tensor cores, for bulk encodes of contiguous bf16 / fp16
// input on sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com), section "K-Cache圧縮：3-bit PolarQuant +
// 1-bit QJL = 4.25 bits/dim" (steps 1-5) and section "V-Cache圧縮：3-bit
// PolarQuant = 3.125 bits/dim" (steps 1-3, no QJL).
//
// One tile is 128 consecutive input vectors (rows of the flattened [B, Hkv,
// T, 128] input).  A TMA load brings the tile into shared memory in the
// 128-byte-swizzled K-major layout; the tensor core computes
//     Y = X (H D)^T          (8 tcgen05.mma, M = N = 128, K = 16)
// into tensor memory: H D has entries +-1, exact in bf16 and fp16, so every
// product is exact and only the fp32 accumulation rounds (as the butterflies
// of the per-lane path do).  Then each vector is quantised from its tensor-
// memory lane: ||Y||^2 = 128 ||x||^2 gives the norm, y = Y / ||Y|| the
// unit-sphere coordinates, the cell search and the centroid run on the FMA
// pipe (saturated fused multiply-adds against the boundaries), and the codes
// are packed into the token record.  For K, the residual r = y - c[idx] goes
// back into the same tensor-memory columns as fp16 hi and lo limbs of r 2^12
// (each 32-column chunk is overwritten only after it has been read), and the
// tensor core computes the QJL projection from there:
//     Z = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T   (24 tcgen05.mma, A in tensor memory)
// whose sign bits are read out one tile later.  Four threads share a vector
// (warps w, w + 4, w + 8, w + 12 reach the same tensor-memory lanes), each
// taking a 32-coordinate chunk; they add their parts of ||Y||^2 and gamma^2
// and merge the code words through shared memory.  Warp 16 issues the TMA
// loads (three tile buffers) and the mma (one thread); Y/R and Z are double-
// buffered in tensor memory, so the rotation of the next tile and the
// projection of this one overlap the quantisation.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tq_frag.cuh"
#include "tq_tc.cuh"

namespace tqi {
namespace {

constexpr int kRD = 128;                  // head_dim
constexpr int kRRows = 128;               // vectors per tile (tensor-memory lanes)
constexpr int kRQuant = 512;              // quantiser threads: four per vector (32 coordinates each)
constexpr int kRThreads = kRQuant + 32;   // + the copy / mma warp
constexpr int kRXBuf = 3;                 // input tile buffers
constexpr int kRTile = kRRows * kRD * 2;  // one 16-bit 128 x 128 operand (32 KB)
constexpr int64_t kRotMinVectors = 16384; // smaller encodes keep the per-lane kernels
constexpr float kRScale = 4096.f;         // residual scale before the fp16 split
// 3.5 (1 + 16 + 256 + 4096): the offset of four nibbles whose codes are held as code - 3.5
constexpr float kNib35 = 15291.5f;

template <bool IS_K>
struct RotShape {
    static constexpr int kOffM = 0;                              // rotation operand H D
    static constexpr int kOffS = kRTile;                         // K: JL operand, hi then lo limb
    static constexpr int kOffX = IS_K ? 3 * kRTile : kRTile;     // input tiles
    static constexpr int kOffBar = kOffX + kRXBuf * kRTile;
    // exchange between the four threads of a vector: ||Y||^2 and gamma^2 parts [4][128],
    // code words of chunks 0-2 and bit-3 planes of chunk 3 [12][128] each
    static constexpr int kOffXchg = kOffBar + 16 * 8;
    // K: address of each vector's sign words, per tile parity [2][128] (written with the
    // record, used for the projection's signs one tile later)
    static constexpr int kOffSgn = kOffXchg + (4 * 128 + 4 * 128 + 12 * 128 + 12 * 128) * 4;
    static constexpr int kOffMisc = kOffSgn + (IS_K ? 2 * 128 * 8 : 0);
    static constexpr int kSmem = kOffMisc + 16 + 1024;           // + slack to align the base
    static constexpr int kCols = IS_K ? 512 : 256;               // Y/R x 2 (+ Z x 2)
};
static_assert(RotShape<true>::kSmem <= 227 * 1024, "shared memory per CTA");

// mbarriers
enum : int {
    kRBarB = 0,       // JL operand copied (K)
    kRBarXFull = 1,   // [3] input tile landed (TMA bytes)
    kRBarXFree = 4,   // [3] input tile read by its rotation (commit)
    kRBarYFull = 7,   // [2] Y computed (commit)
    kRBarRFull = 9,   // [2] Y read and, for K, R written (512 quantiser arrivals)
    kRBarZFull = 11,  // [2] Z computed (commit)
    kRBarDrain = 13,  // every mma of the mma thread done (commit, at exit)
};

__device__ __forceinline__ bool warp_wait_r(uint32_t bar, uint32_t parity) {
    return __all_sync(kFull, mbar_wait_bounded(bar, parity));
}
__device__ __forceinline__ void named_bar_r(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// barrier id over n threads that also ORs v across them (every thread gets the result)
__device__ __forceinline__ bool bar_or_r(int id, int n, bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return res != 0;
}

// Eight entries (K indices i0 .. i0 + 7, i0 a multiple of 8) of row j of the rotation
// operand, (-1)^popcount(i & j) d_i as 16-bit +-1 (one: the bit pattern of 1.0).  The bits
// of i0 and of i - i0 < 8 are disjoint, so popcount(i & j) is popcount(i0 & j) plus that of
// (i - i0) & j: the chunk's sign bits are the byte of d's sign mask at i0, XOR the parity
// pattern of j & 7 over k = 0..7 (bit k: popcount(k & j) odd), XOR all ones when i0 & j has
// odd parity.  dword holds the sign bits of d_{32 (i0 / 32)} .. d_{32 (i0 / 32) + 31}.
__device__ __forceinline__ uint4 rot_chunk(int j, int i0, uint32_t dword, uint32_t one) {
    const uint32_t low = ((j & 1) ? 0xAAu : 0u) ^ ((j & 2) ? 0xCCu : 0u) ^ ((j & 4) ? 0xF0u : 0u);
    const uint32_t neg = ((dword >> (i0 & 31)) ^ low ^ ((__popc(i0 & j) & 1) ? 0xFFu : 0u)) & 0xFFu;
    const uint32_t one2 = one | (one << 16);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) w[e] = one2 | (((neg >> (2 * e)) & 1u) << 15) | (((neg >> (2 * e + 1)) & 1u) << 31);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// word i0 / 32 of the sign mask (a select chain: no dynamic index into the parameters)
__device__ __forceinline__ uint32_t dneg_word(const EncArgs& a, int i0) {
    const int k = i0 >> 5;
    return k == 0 ? a.dneg[0] : k == 1 ? a.dneg[1] : k == 2 ? a.dneg[2] : a.dneg[3];
}

template <int DT, bool IS_K>
__global__ void __launch_bounds__(kRThreads, 1)
    tq_encode_rot_kernel(const __grid_constant__ CUtensorMap tmap, const EncArgs a) {
    using S = RotShape<IS_K>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffMisc);
    pdl_trigger();                 // a chained kernel may start (it waits for this one's writes)

    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kRRows - 1) / kRRows;
    const int n = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);   // this CTA's tiles
    auto row0_of = [&](int j) { return ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kRRows; };
    const int64_t bb = block_bytes(kRD, IS_K);

    auto load = [&](int j) {           // input tile j -> buffer j % 3 (two 64-column boxes)
        const int bx = j % kRXBuf;
        const uint32_t dst = sbase + (uint32_t)(S::kOffX + bx * kRTile), br = bar(kRBarXFull + bx);
        mbar_expect_tx(br, (uint32_t)kRTile);
        const int r0 = (int)row0_of(j);
        tma_load_2d(dst, &tmap, 0, r0, br);
        tma_load_2d(dst + kRTile / 2, &tmap, 64, r0, br);
    };
    int n_load = n < kRXBuf ? n : kRXBuf;
    // The copy thread sets up the barriers and starts the JL operand copy and the first
    // input tiles before the rest of the set-up, which their latency then covers.
    if (tid == kRQuant) {
        mbar_init(bar(kRBarB), 1);
        for (int i = 0; i < kRXBuf; ++i) {
            mbar_init(bar(kRBarXFull + i), 1);
            mbar_init(bar(kRBarXFree + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kRBarYFull + i), 1);
            mbar_init(bar(kRBarRFull + i), kRQuant);
            mbar_init(bar(kRBarZFull + i), 1);
        }
        mbar_init(bar(kRBarDrain), 1);
        fence_mbar_init();
        if constexpr (IS_K) {
            mbar_expect_tx(bar(kRBarB), (uint32_t)(2 * kRTile));
            bulk_g2s(sbase + (uint32_t)S::kOffS, a.bimg, (uint32_t)(2 * kRTile), bar(kRBarB));
        }
        if (a.wait_x) pdl_wait();      // the input and the cache are the previous kernel's to finish
        for (int j = 0; j < n_load; ++j) load(j);
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), S::kCols);
        tc_relinquish();
    }
    // Rotation operand, row j (output coordinate), K index i (input coordinate):
    // (-1)^popcount(i & j) d_i, the Walsh-Hadamard matrix in natural order times
    // the random signs, as bf16 / fp16 +-1; eight entries per store, four per thread.
    if (tid < kRQuant) {
        const int i0 = (tid & 15) * 8;
        const uint32_t dw = dneg_word(a, i0), one = DT == TQ_BF16 ? 0x3F80u : 0x3C00u;
#pragma unroll
        static_assert((kRRows * kRD / 8) % kRQuant == 0 && kRQuant % 16 == 0, "whole chunks per thread");
        for (int m = 0; m < kRRows * kRD / 8 / kRQuant; ++m) {
            const int j = (tid >> 4) + (kRQuant / 16) * m;
            *reinterpret_cast<uint4*>(sm + S::kOffM + sw128_byte(j, 2 * i0, kRD)) = rot_chunk(j, i0, dw, one);
        }
        fence_proxy_async();           // written by threads, read by the tensor core
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == kRQuant) {
        // ======================================== copy and mma thread
        constexpr uint32_t kIdY = DT == TQ_BF16 ? idesc_bf16(kRRows, kRD) : idesc_f16(kRRows, kRD);
        constexpr uint32_t kIdZ = idesc_f16(kRRows, kRD);
        bool ok = true;
        if constexpr (IS_K) ok = mbar_wait_bounded(bar(kRBarB), 0u);
        // Z(j) = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T.  R(j) lies in Y(j)'s columns:
        // coordinates 16 s + 2 m, + 1 in column 16 s + m (hi) and 16 s + 8 + m (lo).
        auto qjl = [&](int j) {
            const uint32_t rb = tmem + (uint32_t)(128 * (j & 1)), zd = tmem + 256u + (uint32_t)(128 * (j & 1));
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (uint32_t)((ks >> 2) * (kRRows * 128) + (ks & 3) * 32);
                const uint32_t ahi = rb + (uint32_t)(16 * ks), alo = ahi + 8u;
                const uint64_t bhi = sw128_desc(sbase + (uint32_t)S::kOffS + koff);
                const uint64_t blo = sw128_desc(sbase + (uint32_t)(S::kOffS + kRTile) + koff);
                tc_mma_f16_ts(zd, ahi, bhi, kIdZ, ks > 0 ? 1u : 0u);
                tc_mma_f16_ts(zd, ahi, blo, kIdZ, 1u);
                tc_mma_f16_ts(zd, alo, bhi, kIdZ, 1u);
            }
            tc_commit(bar(kRBarZFull + (j & 1)));
        };
        for (int j = 0; ok && j < n; ++j) {
            const int bx = j % kRXBuf;
            if (!(ok = mbar_wait_bounded(bar(kRBarXFull + bx), (uint32_t)((j / kRXBuf) & 1)))) break;
            // Y(j) overwrites buffer j % 2: the quantisers are done with tile j - 2 there, and
            // (K) its R was read by the projection mma, issued before this one
            if (j >= 2 && !(ok = mbar_wait_bounded(bar(kRBarRFull + (j & 1)), (uint32_t)(((j - 2) >> 1) & 1)))) break;
            tc_fence_after();
            const uint32_t xa = sbase + (uint32_t)(S::kOffX + bx * kRTile);
            const uint32_t yd = tmem + (uint32_t)(128 * (j & 1));
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (uint32_t)((ks >> 2) * (kRRows * 128) + (ks & 3) * 32);
                tc_mma_f16_ss(yd, sw128_desc(xa + koff), sw128_desc(sbase + (uint32_t)S::kOffM + koff), kIdY,
                              ks > 0 ? 1u : 0u);
            }
            tc_commit(bar(kRBarYFull + (j & 1)));
            tc_commit(bar(kRBarXFree + bx));
            if constexpr (IS_K) {
                if (j >= 1) {          // R(j - 1) is written: its projection
                    if (!(ok = mbar_wait_bounded(bar(kRBarRFull + ((j - 1) & 1)), (uint32_t)(((j - 1) >> 1) & 1))))
                        break;
                    tc_fence_after();
                    qjl(j - 1);
                }
            }
            // tile j + 2 goes into tile j - 1's buffer once that tile's rotation is done
            if (j >= 1 && j + 2 < n) {
                if (!(ok = mbar_wait_bounded(bar(kRBarXFree + (j - 1) % kRXBuf), (uint32_t)(((j - 1) / kRXBuf) & 1))))
                    break;
                load(j + 2);
                ++n_load;
            }
        }
        if constexpr (IS_K) {
            if (ok && n > 0) {
                if ((ok = mbar_wait_bounded(bar(kRBarRFull + ((n - 1) & 1)), (uint32_t)(((n - 1) >> 1) & 1)))) {
                    tc_fence_after();
                    qjl(n - 1);
                }
            }
        }
        // every mma and copy this thread issued is done before shared and tensor memory are
        // released (only the last load into each buffer can still be in flight)
        tc_commit(bar(kRBarDrain));
        mbar_wait_bounded(bar(kRBarDrain), 0u);
        for (int j = n_load > kRXBuf ? n_load - kRXBuf : 0; j < n_load; ++j)
            mbar_wait_bounded(bar(kRBarXFull + j % kRXBuf), (uint32_t)((j / kRXBuf) & 1));
        if (!ok) atomicExch(a.err, 1);
    } else if (tid < kRQuant) {
        // ======================================== quantisers: threads r + 128 c (c = 0..3) share
        // vector r of the tile (tensor-memory lane r); thread c takes coordinates 32 c .. 32 c + 31
        const int cq = tid >> 7;
        const int r = tid & 127;
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        float* xss = reinterpret_cast<float*>(sm + S::kOffXchg);            // [4][128]
        float* xg = xss + 4 * 128;                                           // [4][128]
        uint32_t* xw = reinterpret_cast<uint32_t*>(xg + 4 * 128);            // [12][128]
        uint32_t* xp = xw + 12 * 128;                                        // [12][128]
        [[maybe_unused]] uint8_t** sgn_at = reinterpret_cast<uint8_t**>(sm + S::kOffSgn);   // K: [2][128]
        const Codebook& cb = a.cb;
        // Bucket index and centroid on the FMA pipe.  The codebook is antisymmetric
        // (b3 = 0, b[6-k] = -b[k], c[7-k] = -c[k]), so with a = |y| and
        // t_k = sat((b_k - a) 2^60) = [a < b_k] for k = 4, 5, 6 (the product is exact,
        // its sign decides, and any nonzero difference of two such floats saturates),
        // T = t4 + t5 + t6 boundaries lie above a: the code is 7 - T for y >= 0 and T
        // below, and |c| = c7 - t6 (c7 - c6) - t5 (c6 - c5) - t4 (c5 - c4), every partial
        // sum an exact centroid.  (Here the comparisons run on |Y| directly:
        // t_k = sat(fma(|Y|, -2^60 / ||Y||, b_k 2^60)), one rounding, so the sign of
        // b_k 2^60 - |Y| 2^60 / ||Y|| decides exactly; only the rounding of the per-vector
        // factor differs from forming y first.  The residual is kept in units of 2^-12, with
        // every constant scaled by a power of two.)
        constexpr float kBig = 1152921504606846976.f;        // 2^60
        const float bb4 = cb.b[4] * kBig, bb5 = cb.b[5] * kBig, bb6 = cb.b[6] * kBig;
        [[maybe_unused]] const float d3 = (cb.c[7] - cb.c[6]) * kRScale, d2 = (cb.c[6] - cb.c[5]) * kRScale,
                                     d1 = (cb.c[5] - cb.c[4]) * kRScale, c7 = cb.c[7] * kRScale;
        bool failed = false;
        [[maybe_unused]] bool nz_prev = true;                // the previous tile's vector is nonzero
        // sign word cq of tile jj (K): bit b is z[32 cq + b] >= 0
        auto signs = [&](int jj) -> bool {
            if (!warp_wait_r(bar(kRBarZFull + (jj & 1)), (uint32_t)((jj >> 1) & 1))) return false;
            tc_fence_after();
            uint32_t z[32];
            tc_ld32(tl + 256u + (uint32_t)(128 * (jj & 1) + 32 * cq), z);
            // the sign bits of z[31] .. z[0] shifted in one by one (one funnel shift each),
            // then inverted: bit b = 1 when z[b] >= 0 (a z of -0 would give 0; the
            // accumulation never yields one for a nonzero vector)
            uint32_t word = 0;
#pragma unroll
            for (int bt = 31; bt >= 0; --bt) word = __funnelshift_l(z[bt], word, 1);
            word = ~word;
            if (!nz_prev) word = 0xFFFFFFFFu;                // zero vector: z = 0, every sign bit 1
            uint8_t* sp = sgn_at[(jj & 1) * 128 + r];            // null: no record to write
            if (sp) *reinterpret_cast<uint32_t*>(sp + 4 * cq) = word;
            return true;
        };
        for (int j = 0; j < n; ++j) {
            const int64_t gv = row0_of(j) + r;
            // A failed wait does not leave the loop at once: the four threads of every vector
            // meet at the exchange below, which also ORs their failures, and leave together.
            // (Within a warp the waits are uniform: tensor-memory loads are warp-collective.)
            // Every exchange stays within a vector's four threads, so its barrier (id 1 + q)
            // spans only the four warps of lane quarter q and the quarters run out of step:
            // while one waits at its barrier the others issue.
            const bool ok = !failed && warp_wait_r(bar(kRBarYFull + (j & 1)), (uint32_t)((j >> 1) & 1));
            tc_fence_after();
            const uint32_t yb = tl + (uint32_t)(128 * (j & 1) + 32 * cq);
            {                              // ||Y||^2 = 128 ||x||^2, this chunk's part
                uint32_t v[32];
                tc_ld32(yb, v);
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 32; ++e) s4[e & 3] = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), s4[e & 3]);
                xss[cq * 128 + r] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            if (bar_or_r(1 + (warp & 3), 4 * 32, !ok)) { failed = true; break; }
            const float ss = (xss[r] + xss[128 + r]) + (xss[256 + r] + xss[384 + r]);
            const float nrm = sqrtf(ss * (1.f / 128.f));
            const bool nz = ss > 0.f;
            const float rcp = nz ? __frcp_rn(sqrtf(ss)) : 0.f;   // y = Y / ||Y||
            const float kneg = -kBig * rcp;
            [[maybe_unused]] const float rcpS = rcp * kRScale;
            // Codes in the token record: word 3 t + g holds, in nibble i, the code of slot
            // position 8 g + i (bits 0-2) and bit g of the code of position 24 + i (bit 3).
            // Position p of slot t is coordinate slot_coord(0, t, p), so chunk c gives words
            // 3 t + c for c < 3 and the bit-3 planes for c = 3; nibble i of slot t is the
            // chunk's coordinate o(t, i) = 16 (i / 4) + 2 t + (i % 2) + 8 ((i / 2) % 2): half
            // h of the chunk gives nibbles 4 h .. 4 h + 3.  W[t] collects the chunk's word of slot t.
            uint32_t W[4] = {0u, 0u, 0u, 0u};
            float g2 = 0.f;
#pragma unroll(IS_K ? 1 : 2)
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t v[16];
                tc_ld16(yb + (uint32_t)(16 * h2), v);
                float cf[16];
                [[maybe_unused]] uint32_t rh[8], rl[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    [[maybe_unused]] float rr[2];
#pragma unroll
                    for (int f = 0; f < 2; ++f) {
                        // the sign of Y decides the side of the code and of the residual (Y = -0,
                        // y = 0 on the boundary b3 = 0, counts as negative for both)
                        const uint32_t ybits = v[e + f], sgn = ybits & 0x80000000u;
                        const float av = __uint_as_float(ybits & 0x7FFFFFFFu);
                        const float t4 = __saturatef(fmaf(av, kneg, bb4));
                        const float t5 = __saturatef(fmaf(av, kneg, bb5));
                        const float t6 = __saturatef(fmaf(av, kneg, bb6));
                        const float T = (t4 + t5) + t6;
                        // 7 - T above zero, T below: 3.5 +- (3.5 - T); the 3.5 of all four
                        // nibbles is added once in the sum below (kNib35)
                        cf[e + f] = __uint_as_float(__float_as_uint(3.5f - T) ^ sgn);
                        if constexpr (IS_K) {
                            float m = fmaf(-t6, d3, c7);                // |c| 2^12
                            m = fmaf(-t5, d2, m);
                            m = fmaf(-t4, d1, m);
                            const float rv = __uint_as_float(__float_as_uint(fmaf(av, rcpS, -m)) ^ sgn);   // r 2^12
                            g2 = fmaf(rv, rv, g2);
                            rr[f] = rv;
                        }
                    }
                    if constexpr (IS_K) split_hilo(rr[0], rr[1], rh[e >> 1], rl[e >> 1]);
                }
                if constexpr (IS_K) {      // R over the columns just read: hi limbs, then lo
                    tc_st8(yb + (uint32_t)(16 * h2), rh);
                    tc_st8(yb + (uint32_t)(16 * h2 + 8), rl);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    // four nibbles as an exact float sum, read out of the mantissa (x + 2^23)
                    const float part = fmaf(cf[2 * t + 9], 4096.f,
                                            fmaf(cf[2 * t + 8], 256.f, fmaf(cf[2 * t + 1], 16.f, cf[2 * t] + kNib35)));
                    const uint32_t bits = __float_as_uint(part + 8388608.f);
                    W[t] = h2 == 0 ? bits : __byte_perm(W[t], bits, 0x5410);
                }
            }
            if constexpr (IS_K) tc_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kRBarRFull + (j & 1)));
            if (cq < 3) {
#pragma unroll
                for (int t = 0; t < 4; ++t) xw[(3 * t + cq) * 128 + r] = W[t];
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int g = 0; g < 3; ++g) xp[(3 * t + g) * 128 + r] = ((W[t] >> g) & 0x11111111u) << 3;
            }
            xg[cq * 128 + r] = g2;
            named_bar_r(1 + (warp & 3), 4 * 32);
            if (cq == 0) {
                int64_t xoff;
                uint8_t* blk = nullptr;
                int tau = 0;
                if (gv < N) encode_locate(a, (uint32_t)gv, bb, xoff, blk, tau);
                if constexpr (IS_K)
                    sgn_at[(j & 1) * 128 + r] = blk ? blk + kBlockT * code_bytes(kRD) + tau * sign_bytes(kRD) : nullptr;
                if (blk) {
                    uint32_t wd[12];
#pragma unroll
                    for (int k = 0; k < 12; ++k) wd[k] = xw[k * 128 + r] | xp[k * 128 + r];
                    uint4* rec = reinterpret_cast<uint4*>(blk + tau * code_bytes(kRD));
                    rec[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    rec[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
                    rec[2] = make_uint4(wd[8], wd[9], wd[10], wd[11]);
                    __half* nf = reinterpret_cast<__half*>(blk + kBlockT * (code_bytes(kRD) + (IS_K ? sign_bytes(kRD) : 0)));
                    nf[tau] = __float2half_rn(nrm);
                    if constexpr (IS_K) {        // gamma = ||r||; a zero vector has none
                        const float gs = (xg[r] + xg[128 + r]) + (xg[256 + r] + xg[384 + r]);
                        nf[kBlockT + tau] = __float2half_rn(nz ? sqrtf(gs) * (1.f / kRScale) : 0.f);
                    }
                }
            }
            if constexpr (IS_K) {          // the previous tile's projection ran meanwhile
                if (j >= 1 && !signs(j - 1)) failed = true;      // acted on at the next exchange
                nz_prev = nz;
            }
        }
        if constexpr (IS_K) {
            if (!failed && n > 0 && !signs(n - 1)) failed = true;
        }
        if (failed && (tid & 31) == 0) atomicExch(a.err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, S::kCols);
    }
    pdl_wait();                    // when chained: complete only after the previous kernel
}

// ---------------------------------------------------------------- head_dim 64
// The same scheme at d = 64: 128-vector tiles of 128-byte rows (one TMA box),
// Y = X (H D)^T with 4 tcgen05.mma (N = 64), the rotation's rows in slot order
// (Y's column 16 t + p is coordinate slot_coord(0, t, p), position p of slot t
// of the d = 64 record; the JL operand's K index follows), and two threads per
// vector (warps w and w + 4), each owning two 16-position slots: a thread
// writes its slots' code words and halfwords and its sign word itself, and
// only ||Y||^2 and gamma^2 are added across the two.  Two CTAs fit an SM
// (256 tensor-memory columns each).
constexpr int k6D = 64;
constexpr int k6Quant = 256;                 // two threads per vector
constexpr int k6Threads = k6Quant + 32;
constexpr int k6Tile = kRRows * k6D * 2;     // 16 KB
constexpr int k6Op = 64 * k6D * 2;           // a 64 x 64 16-bit operand (8 KB)

template <bool IS_K>
struct Rot64Shape {
    static constexpr int kOffM = 0;                              // rotation operand H D (rows in slot order)
    static constexpr int kOffS = k6Op;                           // K: JL operand, hi then lo limb
    static constexpr int kOffX = IS_K ? 3 * k6Op : k6Op;         // input tiles
    static constexpr int kOffBar = kOffX + kRXBuf * k6Tile;
    static constexpr int kOffXchg = kOffBar + 16 * 8;            // ||Y||^2 and gamma^2 parts [2 tiles][2][128] each
    static constexpr int kOffMisc = kOffXchg + 2 * (2 * 2 * 128) * 4;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr int kCols = 256;                            // Y/R x 2 at 0, 64; Z x 2 at 128, 192
};

template <int DT, bool IS_K>
__global__ void __launch_bounds__(k6Threads, 2)
    tq_encode_rot64_kernel(const __grid_constant__ CUtensorMap tmap, const EncArgs a) {
    using S = Rot64Shape<IS_K>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffMisc);
    pdl_trigger();                 // a chained kernel may start (it waits for this one's writes)

    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kRRows - 1) / kRRows;
    const int n = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);   // this CTA's tiles
    auto row0_of = [&](int j) { return ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kRRows; };
    const int64_t bb = block_bytes(k6D, IS_K);

    auto load = [&](int j) {           // input tile j -> buffer j % 3 (one 64-column box)
        const int bx = j % kRXBuf;
        const uint32_t dst = sbase + (uint32_t)(S::kOffX + bx * k6Tile), br = bar(kRBarXFull + bx);
        mbar_expect_tx(br, (uint32_t)k6Tile);
        tma_load_2d(dst, &tmap, 0, (int)row0_of(j), br);
    };
    int n_load = n < kRXBuf ? n : kRXBuf;
    // barriers, the JL operand copy and the first input tiles first (as at d = 128)
    if (tid == k6Quant) {
        mbar_init(bar(kRBarB), 1);
        for (int i = 0; i < kRXBuf; ++i) {
            mbar_init(bar(kRBarXFull + i), 1);
            mbar_init(bar(kRBarXFree + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kRBarYFull + i), 1);
            mbar_init(bar(kRBarRFull + i), k6Quant);
            mbar_init(bar(kRBarZFull + i), 1);
        }
        mbar_init(bar(kRBarDrain), 1);
        fence_mbar_init();
        if constexpr (IS_K) {
            mbar_expect_tx(bar(kRBarB), (uint32_t)(2 * k6Op));
            bulk_g2s(sbase + (uint32_t)S::kOffS, a.bimg, (uint32_t)(2 * k6Op), bar(kRBarB));
        }
        if (a.wait_x) pdl_wait();      // the input and the cache are the previous kernel's to finish
        for (int j = 0; j < n_load; ++j) load(j);
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), S::kCols);
        tc_relinquish();
    }
    // Rotation operand row nr (Y's column nr), K index i: (-1)^popcount(i & j) d_i with
    // j = slot_coord(0, nr / 16, nr % 16), as bf16 / fp16 +-1; eight entries per store,
    // two per thread.
    if (tid < k6Quant) {
        const int i0 = (tid & 7) * 8;
        const uint32_t dw = dneg_word(a, i0), one = DT == TQ_BF16 ? 0x3F80u : 0x3C00u;
        static_assert((64 * k6D / 8) % k6Quant == 0 && k6Quant % 8 == 0, "whole chunks per thread");
#pragma unroll
        for (int m = 0; m < 64 * k6D / 8 / k6Quant; ++m) {
            const int nr = (tid >> 3) + (k6Quant / 8) * m;
            const int j = slot_coord(0, nr >> 4, nr & 15);
            *reinterpret_cast<uint4*>(sm + S::kOffM + sw128_byte(nr, 2 * i0, 64)) = rot_chunk(j, i0, dw, one);
        }
        fence_proxy_async();           // written by threads, read by the tensor core
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == k6Quant) {
        // ======================================== copy and mma thread
        constexpr uint32_t kIdY = DT == TQ_BF16 ? idesc_bf16(kRRows, k6D) : idesc_f16(kRRows, k6D);
        constexpr uint32_t kIdZ = idesc_f16(kRRows, k6D);
        bool ok = true;
        if constexpr (IS_K) ok = mbar_wait_bounded(bar(kRBarB), 0u);
        // Z(j) = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T over the coordinates in slot order.
        // R(j) lies in Y(j)'s columns: K positions 16 s + 2 m, + 1 in column 16 s + m (hi)
        // and 16 s + 8 + m (lo).
        auto qjl = [&](int j) {
            const uint32_t rb = tmem + (uint32_t)(64 * (j & 1)), zd = tmem + 128u + (uint32_t)(64 * (j & 1));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint32_t ahi = rb + (uint32_t)(16 * ks), alo = ahi + 8u;
                const uint64_t bhi = sw128_desc(sbase + (uint32_t)S::kOffS + 32u * ks);
                const uint64_t blo = sw128_desc(sbase + (uint32_t)(S::kOffS + k6Op) + 32u * ks);
                tc_mma_f16_ts(zd, ahi, bhi, kIdZ, ks > 0 ? 1u : 0u);
                tc_mma_f16_ts(zd, ahi, blo, kIdZ, 1u);
                tc_mma_f16_ts(zd, alo, bhi, kIdZ, 1u);
            }
            tc_commit(bar(kRBarZFull + (j & 1)));
        };
        for (int j = 0; ok && j < n; ++j) {
            const int bx = j % kRXBuf;
            if (!(ok = mbar_wait_bounded(bar(kRBarXFull + bx), (uint32_t)((j / kRXBuf) & 1)))) break;
            if (j >= 2 && !(ok = mbar_wait_bounded(bar(kRBarRFull + (j & 1)), (uint32_t)(((j - 2) >> 1) & 1)))) break;
            tc_fence_after();
            const uint32_t xa = sbase + (uint32_t)(S::kOffX + bx * k6Tile);
            const uint32_t yd = tmem + (uint32_t)(64 * (j & 1));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma_f16_ss(yd, sw128_desc(xa + 32u * ks), sw128_desc(sbase + (uint32_t)S::kOffM + 32u * ks), kIdY,
                              ks > 0 ? 1u : 0u);
            tc_commit(bar(kRBarYFull + (j & 1)));
            tc_commit(bar(kRBarXFree + bx));
            if constexpr (IS_K) {
                if (j >= 1) {
                    if (!(ok = mbar_wait_bounded(bar(kRBarRFull + ((j - 1) & 1)), (uint32_t)(((j - 1) >> 1) & 1))))
                        break;
                    tc_fence_after();
                    qjl(j - 1);
                }
            }
            if (j >= 1 && j + 2 < n) {
                if (!(ok = mbar_wait_bounded(bar(kRBarXFree + (j - 1) % kRXBuf), (uint32_t)(((j - 1) / kRXBuf) & 1))))
                    break;
                load(j + 2);
                ++n_load;
            }
        }
        if constexpr (IS_K) {
            if (ok && n > 0) {
                if ((ok = mbar_wait_bounded(bar(kRBarRFull + ((n - 1) & 1)), (uint32_t)(((n - 1) >> 1) & 1)))) {
                    tc_fence_after();
                    qjl(n - 1);
                }
            }
        }
        tc_commit(bar(kRBarDrain));
        mbar_wait_bounded(bar(kRBarDrain), 0u);
        for (int j = n_load > kRXBuf ? n_load - kRXBuf : 0; j < n_load; ++j)
            mbar_wait_bounded(bar(kRBarXFull + j % kRXBuf), (uint32_t)((j / kRXBuf) & 1));
        if (!ok) atomicExch(a.err, 1);
    } else if (tid < k6Quant) {
        // ======================================== quantisers: threads r and r + 128 share vector r
        // (tensor-memory lane r); thread h owns slots 2 h, 2 h + 1, Y's columns 32 h .. 32 h + 31
        const int hv = tid >> 7;
        const int r = tid & 127;
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        float* xss = reinterpret_cast<float*>(sm + S::kOffXchg);            // [2][2][128]
        [[maybe_unused]] float* xg = xss + 2 * 2 * 128;                      // [2][2][128]
        const Codebook& cb = a.cb;
        // the cell search and residual of the d = 128 kernel, with this head_dim's codebook
        constexpr float kBig = 1152921504606846976.f;        // 2^60
        const float bb4 = cb.b[4] * kBig, bb5 = cb.b[5] * kBig, bb6 = cb.b[6] * kBig;
        [[maybe_unused]] const float d3 = (cb.c[7] - cb.c[6]) * kRScale, d2 = (cb.c[6] - cb.c[5]) * kRScale,
                                     d1 = (cb.c[5] - cb.c[4]) * kRScale, c7 = cb.c[7] * kRScale;
        bool failed = false;
        [[maybe_unused]] bool nz_prev = true;                // the previous tile's vector is nonzero
        // K: address of the sign words of this thread's vector in the previous tile (null: none)
        [[maybe_unused]] uint8_t* sgn_prev = nullptr;
        // sign word hv of tile jj (K): bit b is z[32 hv + b] >= 0
        auto signs = [&](int jj) -> bool {
            if (!warp_wait_r(bar(kRBarZFull + (jj & 1)), (uint32_t)((jj >> 1) & 1))) return false;
            tc_fence_after();
            uint32_t z[32];
            tc_ld32(tl + 128u + (uint32_t)(64 * (jj & 1) + 32 * hv), z);
            // the sign bits of z[31] .. z[0] shifted in one by one (one funnel shift each),
            // then inverted: bit b = 1 when z[b] >= 0 (a z of -0 would give 0; the
            // accumulation never yields one for a nonzero vector)
            uint32_t word = 0;
#pragma unroll
            for (int bt = 31; bt >= 0; --bt) word = __funnelshift_l(z[bt], word, 1);
            word = ~word;
            if (!nz_prev) word = 0xFFFFFFFFu;                // zero vector: z = 0, every sign bit 1
            if (sgn_prev) *reinterpret_cast<uint32_t*>(sgn_prev + 4 * hv) = word;
            return true;
        };
        for (int j = 0; j < n; ++j) {
            const int64_t gv = row0_of(j) + r;
            const int x = j & 1;
            // A failed wait does not leave the loop at once: both threads of every vector meet
            // at the exchange below, which also ORs their failures, and leave together.
            // The exchange barrier (id 1 + q) spans only the two warps of lane quarter q.
            const bool ok = !failed && warp_wait_r(bar(kRBarYFull + x), (uint32_t)((j >> 1) & 1));
            tc_fence_after();
            const uint32_t yb = tl + (uint32_t)(64 * x + 32 * hv);
            {                              // ||Y||^2 = 64 ||x||^2, this thread's part
                uint32_t v[32];
                tc_ld32(yb, v);
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 32; ++e) s4[e & 3] = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), s4[e & 3]);
                xss[(x * 2 + hv) * 128 + r] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            if (bar_or_r(1 + (warp & 3), 2 * 32, !ok)) { failed = true; break; }
            const float ss = xss[(x * 2) * 128 + r] + xss[(x * 2 + 1) * 128 + r];
            const float nrm = sqrtf(ss * (1.f / 64.f));
            const bool nz = ss > 0.f;
            const float rcp = nz ? __frcp_rn(sqrtf(ss)) : 0.f;   // y = Y / ||Y||
            const float kneg = -kBig * rcp;
            [[maybe_unused]] const float rcpS = rcp * kRScale;
            // d = 64 record, slot t: word t holds in nibble i the code of position i (bits 0-2)
            // and, for i < 4 bit 0, for i >= 4 bit 1 of the code of position 12 + i % 4 (bit 3);
            // halfword t holds the codes of positions 8..11 and bit 2 of those of 12..15.
            uint32_t wd0 = 0, wd1 = 0, hw0 = 0, hw1 = 0;
            float g2 = 0.f;
#pragma unroll(IS_K ? 1 : 2)
            for (int h2 = 0; h2 < 2; ++h2) {           // slot 2 hv + h2
                uint32_t v[16];
                tc_ld16(yb + (uint32_t)(16 * h2), v);
                float cf[16];
                [[maybe_unused]] uint32_t rh[8], rl[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    [[maybe_unused]] float rr[2];
#pragma unroll
                    for (int f = 0; f < 2; ++f) {
                        const uint32_t ybits = v[e + f], sgn = ybits & 0x80000000u;
                        const float av = __uint_as_float(ybits & 0x7FFFFFFFu);
                        const float t4 = __saturatef(fmaf(av, kneg, bb4));
                        const float t5 = __saturatef(fmaf(av, kneg, bb5));
                        const float t6 = __saturatef(fmaf(av, kneg, bb6));
                        const float T = (t4 + t5) + t6;
                        cf[e + f] = __uint_as_float(__float_as_uint(3.5f - T) ^ sgn);   // code - 3.5
                        if constexpr (IS_K) {
                            float m = fmaf(-t6, d3, c7);
                            m = fmaf(-t5, d2, m);
                            m = fmaf(-t4, d1, m);
                            const float rv = __uint_as_float(__float_as_uint(fmaf(av, rcpS, -m)) ^ sgn);
                            g2 = fmaf(rv, rv, g2);
                            rr[f] = rv;
                        }
                    }
                    if constexpr (IS_K) split_hilo(rr[0], rr[1], rh[e >> 1], rl[e >> 1]);
                }
                if constexpr (IS_K) {
                    tc_st8(yb + (uint32_t)(16 * h2), rh);
                    tc_st8(yb + (uint32_t)(16 * h2 + 8), rl);
                }
                // nibble sums as exact floats, read out of the mantissa (x + 2^23)
                const float n0 = fmaf(cf[3], 4096.f, fmaf(cf[2], 256.f, fmaf(cf[1], 16.f, cf[0] + kNib35)));
                const float n1 = fmaf(cf[7], 4096.f, fmaf(cf[6], 256.f, fmaf(cf[5], 16.f, cf[4] + kNib35)));
                const float n2 = fmaf(cf[11], 4096.f, fmaf(cf[10], 256.f, fmaf(cf[9], 16.f, cf[8] + kNib35)));
                const float n3 = fmaf(cf[15], 4096.f, fmaf(cf[14], 256.f, fmaf(cf[13], 16.f, cf[12] + kNib35)));
                const uint32_t na = __byte_perm(__float_as_uint(n0 + 8388608.f), __float_as_uint(n1 + 8388608.f), 0x5410);
                const uint32_t nb = __float_as_uint(n2 + 8388608.f) & 0xFFFFu;
                const uint32_t nc = __float_as_uint(n3 + 8388608.f) & 0xFFFFu;
                const uint32_t w = na | ((nc & 0x1111u) << 3) | (((nc >> 1) & 0x1111u) << 19);
                const uint32_t hw = nb | (((nc >> 2) & 0x1111u) << 3);
                wd0 = h2 == 0 ? w : wd0;
                wd1 = h2 == 1 ? w : wd1;
                hw0 = h2 == 0 ? hw : hw0;
                hw1 = h2 == 1 ? hw : hw1;
            }
            if constexpr (IS_K) tc_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kRBarRFull + x));
            if constexpr (IS_K) xg[(x * 2 + hv) * 128 + r] = g2;
            uint8_t* blk = nullptr;
            int tau = 0;
            if (gv < N) {
                int64_t xoff;
                encode_locate(a, (uint32_t)gv, bb, xoff, blk, tau);
                if (blk) {
                    uint8_t* rec = blk + tau * code_bytes(k6D);
                    *reinterpret_cast<uint2*>(rec + 8 * hv) = make_uint2(wd0, wd1);     // words 2 hv, 2 hv + 1
                    *reinterpret_cast<uint32_t*>(rec + 16 + 4 * hv) = hw0 | (hw1 << 16);    // their halfwords
                    if (hv == 0)
                        reinterpret_cast<__half*>(blk + kBlockT * (code_bytes(k6D) + (IS_K ? sign_bytes(k6D) : 0)))[tau] =
                            __float2half_rn(nrm);
                }
            }
            if constexpr (IS_K) {
                named_bar_r(1 + (warp & 3), 2 * 32);   // both gamma^2 parts are written
                if (hv == 0 && blk) {
                    const float gs = xg[(x * 2) * 128 + r] + xg[(x * 2 + 1) * 128 + r];
                    reinterpret_cast<__half*>(blk + kBlockT * (code_bytes(k6D) + sign_bytes(k6D)))[kBlockT + tau] =
                        __float2half_rn(nz ? sqrtf(gs) * (1.f / kRScale) : 0.f);     // a zero vector has no residual
                }
                if (j >= 1 && !signs(j - 1)) failed = true;      // acted on at the next exchange
                sgn_prev = blk ? blk + kBlockT * code_bytes(k6D) + tau * sign_bytes(k6D) : nullptr;
                nz_prev = nz;
            }
        }
        if constexpr (IS_K) {
            if (!failed && n > 0 && !signs(n - 1)) failed = true;
        }
        if (failed && (tid & 31) == 0) atomicExch(a.err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, S::kCols);
    }
    pdl_wait();                    // when chained: complete only after the previous kernel
}

// ---------------------------------------------------------------- head_dim 128, V, two threads per vector
// The V encode at d = 128 with the d = 64 kernel's organisation: Y = X (H D)^T
// with the rotation's rows in slot order (Y's column 32 t + p is coordinate
// slot_coord(0, t, p), position p of slot t), two threads per vector (warps w
// and w + 4), each owning two 32-position slots: a thread builds its slots'
// three code words (Wa, Wb, Wc of each slot, the bit-3 planes from positions
// 24..31 included) in registers and stores its 24 bytes of the record itself,
// so the two threads meet once per tile, for ||Y||^2.  Two input buffers and
// 256 tensor-memory columns (Y x 2), so two CTAs fit an SM.
constexpr int kVQuant = 256;                 // two threads per vector
constexpr int kVThreads = kVQuant + 32;
constexpr int kVXBuf = 2;                    // input tile buffers

struct RotVShape {
    static constexpr int kOffM = 0;                              // rotation operand H D (rows in slot order)
    static constexpr int kOffX = kRTile;                         // input tiles
    static constexpr int kOffBar = kOffX + kVXBuf * kRTile;
    static constexpr int kOffXchg = kOffBar + 16 * 8;            // ||Y||^2 parts [2 tiles][2][128]
    static constexpr int kOffMisc = kOffXchg + 2 * 2 * 128 * 4;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr int kCols = 256;                            // Y x 2 at 0, 128
};
static_assert(2 * (RotVShape::kSmem + 1024) <= 228 * 1024, "two CTAs per SM");

template <int DT>
__global__ void __launch_bounds__(kVThreads, 2)
    tq_encode_rotv_kernel(const __grid_constant__ CUtensorMap tmap, const EncArgs a) {
    using S = RotVShape;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffMisc);
    pdl_trigger();                 // a chained kernel may start (it waits for this one's writes)

    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kRRows - 1) / kRRows;
    const int n = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);   // this CTA's tiles
    auto row0_of = [&](int j) { return ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kRRows; };
    const int64_t bb = block_bytes(kRD, false);

    auto load = [&](int j) {           // input tile j -> buffer j % 2 (two 64-column boxes)
        const int bx = j % kVXBuf;
        const uint32_t dst = sbase + (uint32_t)(S::kOffX + bx * kRTile), br = bar(kRBarXFull + bx);
        mbar_expect_tx(br, (uint32_t)kRTile);
        const int r0 = (int)row0_of(j);
        tma_load_2d(dst, &tmap, 0, r0, br);
        tma_load_2d(dst + kRTile / 2, &tmap, 64, r0, br);
    };
    int n_load = n < kVXBuf ? n : kVXBuf;
    // barriers and the first input tiles first (as in the K kernel)
    if (tid == kVQuant) {
        for (int i = 0; i < kVXBuf; ++i) {
            mbar_init(bar(kRBarXFull + i), 1);
            mbar_init(bar(kRBarXFree + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kRBarYFull + i), 1);
            mbar_init(bar(kRBarRFull + i), kVQuant);
        }
        mbar_init(bar(kRBarDrain), 1);
        fence_mbar_init();
        if (a.wait_x) pdl_wait();      // the input and the cache are the previous kernel's to finish
        for (int j = 0; j < n_load; ++j) load(j);
    }
    if (warp == 0) {
        tc_alloc(smem_u32(tmem_slot), S::kCols);
        tc_relinquish();
    }
    // Rotation operand row nr (Y's column nr), K index i: (-1)^popcount(i & j) d_i with
    // j = slot_coord(0, nr / 32, nr % 32), as bf16 / fp16 +-1; eight entries per store,
    // eight per thread.
    if (tid < kVQuant) {
        const int i0 = (tid & 15) * 8;
        const uint32_t dw = dneg_word(a, i0), one = DT == TQ_BF16 ? 0x3F80u : 0x3C00u;
        static_assert((kRRows * kRD / 8) % kVQuant == 0 && kVQuant % 16 == 0, "whole chunks per thread");
#pragma unroll
        for (int m = 0; m < kRRows * kRD / 8 / kVQuant; ++m) {
            const int nr = (tid >> 4) + (kVQuant / 16) * m;
            const int j = slot_coord(0, nr >> 5, nr & 31);
            *reinterpret_cast<uint4*>(sm + S::kOffM + sw128_byte(nr, 2 * i0, kRD)) = rot_chunk(j, i0, dw, one);
        }
        fence_proxy_async();           // written by threads, read by the tensor core
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == kVQuant) {
        // ======================================== copy and mma thread
        constexpr uint32_t kIdY = DT == TQ_BF16 ? idesc_bf16(kRRows, kRD) : idesc_f16(kRRows, kRD);
        bool ok = true;
        for (int j = 0; ok && j < n; ++j) {
            const int bx = j % kVXBuf;
            if (!(ok = mbar_wait_bounded(bar(kRBarXFull + bx), (uint32_t)((j / kVXBuf) & 1)))) break;
            // Y(j) overwrites buffer j % 2: the quantisers are done with tile j - 2 there
            if (j >= 2 && !(ok = mbar_wait_bounded(bar(kRBarRFull + (j & 1)), (uint32_t)(((j - 2) >> 1) & 1)))) break;
            tc_fence_after();
            const uint32_t xa = sbase + (uint32_t)(S::kOffX + bx * kRTile);
            const uint32_t yd = tmem + (uint32_t)(128 * (j & 1));
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (uint32_t)((ks >> 2) * (kRRows * 128) + (ks & 3) * 32);
                tc_mma_f16_ss(yd, sw128_desc(xa + koff), sw128_desc(sbase + (uint32_t)S::kOffM + koff), kIdY,
                              ks > 0 ? 1u : 0u);
            }
            tc_commit(bar(kRBarYFull + (j & 1)));
            tc_commit(bar(kRBarXFree + bx));
            // tile j + 1 goes into tile j - 1's buffer once that tile's rotation is done
            if (j >= 1 && j + 1 < n) {
                if (!(ok = mbar_wait_bounded(bar(kRBarXFree + (j - 1) % kVXBuf), (uint32_t)(((j - 1) / kVXBuf) & 1))))
                    break;
                load(j + 1);
                ++n_load;
            }
        }
        // every mma and copy this thread issued is done before shared and tensor memory are
        // released (only the last load into each buffer can still be in flight)
        tc_commit(bar(kRBarDrain));
        mbar_wait_bounded(bar(kRBarDrain), 0u);
        for (int j = n_load > kVXBuf ? n_load - kVXBuf : 0; j < n_load; ++j)
            mbar_wait_bounded(bar(kRBarXFull + j % kVXBuf), (uint32_t)((j / kVXBuf) & 1));
        if (!ok) atomicExch(a.err, 1);
    } else if (tid < kVQuant) {
        // ======================================== quantisers: threads r and r + 128 share vector r
        // (tensor-memory lane r); thread h owns slots 2 h, 2 h + 1, Y's columns 64 h .. 64 h + 63
        const int hv = tid >> 7;
        const int r = tid & 127;
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        float* xss = reinterpret_cast<float*>(sm + S::kOffXchg);            // [2][2][128]
        const Codebook& cb = a.cb;
        // the cell search of the four-thread kernel
        constexpr float kBig = 1152921504606846976.f;        // 2^60
        const float bb4 = cb.b[4] * kBig, bb5 = cb.b[5] * kBig, bb6 = cb.b[6] * kBig;
        bool failed = false;
        for (int j = 0; j < n; ++j) {
            const int64_t gv = row0_of(j) + r;
            const int x = j & 1;
            // A failed wait does not leave the loop at once: both threads of every vector meet
            // at the exchange below, which also ORs their failures, and leave together.
            // The exchange barrier (id 1 + q) spans only the two warps of lane quarter q.
            const bool ok = !failed && warp_wait_r(bar(kRBarYFull + x), (uint32_t)((j >> 1) & 1));
            tc_fence_after();
            const uint32_t yb = tl + (uint32_t)(128 * x + 64 * hv);
            {                              // ||Y||^2 = 128 ||x||^2, this thread's part
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t v[32];
                    tc_ld32(yb + (uint32_t)(32 * q), v);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        s4[e & 3] = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), s4[e & 3]);
                }
                xss[(x * 2 + hv) * 128 + r] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            if (bar_or_r(1 + (warp & 3), 2 * 32, !ok)) { failed = true; break; }
            const float ss = xss[(x * 2) * 128 + r] + xss[(x * 2 + 1) * 128 + r];
            const float nrm = sqrtf(ss * (1.f / 128.f));
            const float rcp = ss > 0.f ? __frcp_rn(sqrtf(ss)) : 0.f;   // y = Y / ||Y||
            const float kneg = -kBig * rcp;
            // slot 2 hv + s2: word a holds in nibble k the code of position k (bits 0-2) and
            // bit 0 of the code of position 24 + k (bit 3); words b, c positions 8 + k, 16 + k
            // and bits 1, 2 of the code of 24 + k
            uint32_t wd[6];
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                uint32_t nib[4];       // nibble words of positions 0-7, 8-15, 16-23, 24-31
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[16];
                    tc_ld16(yb + (uint32_t)(32 * s2 + 16 * h2), v);
                    float cf[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint32_t ybits = v[e], sgn = ybits & 0x80000000u;
                        const float av = __uint_as_float(ybits & 0x7FFFFFFFu);
                        const float t4 = __saturatef(fmaf(av, kneg, bb4));
                        const float t5 = __saturatef(fmaf(av, kneg, bb5));
                        const float t6 = __saturatef(fmaf(av, kneg, bb6));
                        const float T = (t4 + t5) + t6;
                        cf[e] = __uint_as_float(__float_as_uint(3.5f - T) ^ sgn);   // code - 3.5
                    }
                    // nibble sums as exact floats, read out of the mantissa (x + 2^23)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float lo = fmaf(cf[8 * q + 3], 4096.f,
                                              fmaf(cf[8 * q + 2], 256.f, fmaf(cf[8 * q + 1], 16.f, cf[8 * q] + kNib35)));
                        const float hi = fmaf(cf[8 * q + 7], 4096.f,
                                              fmaf(cf[8 * q + 6], 256.f, fmaf(cf[8 * q + 5], 16.f, cf[8 * q + 4] + kNib35)));
                        nib[2 * h2 + q] = __byte_perm(__float_as_uint(lo + 8388608.f), __float_as_uint(hi + 8388608.f), 0x5410);
                    }
                }
                const uint32_t p3 = nib[3];
#pragma unroll
                for (int g = 0; g < 3; ++g) wd[3 * s2 + g] = nib[g] | (((p3 >> g) & 0x11111111u) << 3);
            }
            tc_fence_before();
            mbar_arrive(bar(kRBarRFull + x));
            if (gv < N) {
                int64_t xoff;
                uint8_t* blk;
                int tau;
                encode_locate(a, (uint32_t)gv, bb, xoff, blk, tau);
                if (blk) {
                    uint2* rec = reinterpret_cast<uint2*>(blk + tau * code_bytes(kRD) + 24 * hv);   // slots 2 hv, 2 hv + 1
                    rec[0] = make_uint2(wd[0], wd[1]);
                    rec[1] = make_uint2(wd[2], wd[3]);
                    rec[2] = make_uint2(wd[4], wd[5]);
                    if (hv == 0) reinterpret_cast<__half*>(blk + kBlockT * code_bytes(kRD))[tau] = __float2half_rn(nrm);
                }
            }
        }
        if (failed && (tid & 31) == 0) atomicExch(a.err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, S::kCols);
    }
    pdl_wait();                    // when chained: complete only after the previous kernel
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

template <int DT, bool IS_K>
cudaError_t launch_rot_t(const CUtensorMap& tm, const EncArgs& a, int grid, bool pdl, cudaStream_t s) {
    constexpr int smem = RotShape<IS_K>::kSmem;
    cudaError_t e = set_smem_once<tq_encode_rot_kernel<DT, IS_K>>(smem);
    if (e != cudaSuccess) return e;
    if (pdl) return launch_pdl(tq_encode_rot_kernel<DT, IS_K>, dim3(grid), dim3(kRThreads), smem, s, tm, a);
    tq_encode_rot_kernel<DT, IS_K><<<grid, kRThreads, smem, s>>>(tm, a);
    return cudaGetLastError();
}

template <int DT>
cudaError_t launch_rotv_t(const CUtensorMap& tm, const EncArgs& a, int grid, bool pdl, cudaStream_t s) {
    constexpr int smem = RotVShape::kSmem;
    cudaError_t e = set_smem_once<tq_encode_rotv_kernel<DT>>(smem);
    if (e != cudaSuccess) return e;
    if (pdl) return launch_pdl(tq_encode_rotv_kernel<DT>, dim3(grid), dim3(kVThreads), smem, s, tm, a);
    tq_encode_rotv_kernel<DT><<<grid, kVThreads, smem, s>>>(tm, a);
    return cudaGetLastError();
}

template <int DT, bool IS_K>
cudaError_t launch_rot64_t(const CUtensorMap& tm, const EncArgs& a, int grid, bool pdl, cudaStream_t s) {
    constexpr int smem = Rot64Shape<IS_K>::kSmem;
    cudaError_t e = set_smem_once<tq_encode_rot64_kernel<DT, IS_K>>(smem);
    if (e != cudaSuccess) return e;
    if (pdl) return launch_pdl(tq_encode_rot64_kernel<DT, IS_K>, dim3(grid), dim3(k6Threads), smem, s, tm, a);
    tq_encode_rot64_kernel<DT, IS_K><<<grid, k6Threads, smem, s>>>(tm, a);
    return cudaGetLastError();
}

// 2-D tensor map over the flattened [N, d] input when its rows are consecutive (16-bit
// elements, 16-byte aligned); false when the call does not qualify.
bool rot_tensor_map(int d, tq_dtype dt, const EncArgs& a, CUtensorMap* tm) {
    if (dt != TQ_BF16 && dt != TQ_F16) return false;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    if (N < kRotMinVectors || !a.vec16) return false;
    if (a.st != d || (a.Hkv > 1 && a.sh != a.Tnew * d) || (a.B > 1 && a.sb != a.Hkv * a.Tnew * d)) return false;
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kRRows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, dt == TQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(a.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Every launch is a programmatic dependent of the previous kernel on the stream, so that the
// set-up (barriers, tensor memory, the rotation operand, the JL operand copy) overlaps that
// kernel's end.  A chained launch (pdl: the previous kernel writes neither this input nor the
// cache range) loads at once; any other waits for the previous kernel before its first input
// load, and every write of the kernel follows that load.
EncArgs dependent_args(const EncArgs& a, bool chained) {
    EncArgs b = a;
    b.wait_x = chained ? 0 : 1;
    return b;
}

}  // namespace

cudaError_t launch_encode64_rot(bool is_k, tq_dtype dt, const EncArgs& a0, int num_sms, bool pdl, cudaStream_t s) {
    CUtensorMap tm;
    if (!a0.bimg || !rot_tensor_map(k6D, dt, a0, &tm)) return cudaErrorNotSupported;
    const EncArgs a = dependent_args(a0, pdl);
    pdl = true;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kRRows - 1) / kRRows;
    const int grid = (int)(ntiles < 2 * (int64_t)num_sms ? ntiles : 2 * (int64_t)num_sms);
    if (dt == TQ_BF16)
        return is_k ? launch_rot64_t<TQ_BF16, true>(tm, a, grid, pdl, s) : launch_rot64_t<TQ_BF16, false>(tm, a, grid, pdl, s);
    return is_k ? launch_rot64_t<TQ_F16, true>(tm, a, grid, pdl, s) : launch_rot64_t<TQ_F16, false>(tm, a, grid, pdl, s);
}

cudaError_t launch_encode128_rot(bool is_k, tq_dtype dt, const EncArgs& a0, int num_sms, bool pdl, cudaStream_t s) {
    CUtensorMap tm;
    if (!rot_tensor_map(kRD, dt, a0, &tm)) return cudaErrorNotSupported;
    const EncArgs a = dependent_args(a0, pdl);
    pdl = true;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kRRows - 1) / kRRows;
    const int grid = (int)(ntiles < num_sms ? ntiles : num_sms);
    if (!is_k) {                   // V: two threads per vector, two CTAs per SM
        const int gv = (int)(ntiles < 2 * num_sms ? ntiles : 2 * num_sms);
        return dt == TQ_BF16 ? launch_rotv_t<TQ_BF16>(tm, a, gv, pdl, s) : launch_rotv_t<TQ_F16>(tm, a, gv, pdl, s);
    }
    return dt == TQ_BF16 ? launch_rot_t<TQ_BF16, true>(tm, a, grid, pdl, s) : launch_rot_t<TQ_F16, true>(tm, a, grid, pdl, s);
}

}  // namespace tqi
