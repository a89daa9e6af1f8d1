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
#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kD = 128;
constexpr int kNW = 8;                 // warps per CTA
constexpr int kStages = 4;             // ring depth per warp
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
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
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

// Selector words for the 32 slot codes of one token: sel[w] holds, in its
// nibbles, the codes of slot positions 8w .. 8w+7.
__device__ __forceinline__ void code_selectors(const uint8_t* rec, uint32_t (&sel)[4]) {
    const uint32_t wa = *reinterpret_cast<const uint32_t*>(rec);
    const uint32_t wb = *reinterpret_cast<const uint32_t*>(rec + 4);
    const uint32_t wc = *reinterpret_cast<const uint32_t*>(rec + 8);
    sel[0] = wa & 0x77777777u;
    sel[1] = wb & 0x77777777u;
    sel[2] = wc & 0x77777777u;
    sel[3] = ((wa >> 3) & 0x11111111u) | ((wb >> 2) & 0x22222222u) | ((wc >> 1) & 0x44444444u);
}

// fp16 centroid pairs for slot positions 4kc .. 4kc+3: e=0,1 -> x0, e=2,3 -> x1
__device__ __forceinline__ void dequant4(uint32_t sel16, const uint32_t (&lut)[4], uint32_t& x0, uint32_t& x1) {
    const uint32_t lo4 = __byte_perm(lut[0], lut[1], sel16);
    const uint32_t hi4 = __byte_perm(lut[2], lut[3], sel16);
    x0 = __byte_perm(lo4, hi4, 0x5140);
    x1 = __byte_perm(lo4, hi4, 0x7362);
}

__device__ __forceinline__ uint32_t sel_for(const uint32_t (&sel)[4], int kc) {
    return (kc & 1) ? (sel[kc >> 1] >> 16) : sel[kc >> 1];
}

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kNW * 32, 1) tq_decode_mma128_kernel(const DecArgs a, int G) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kNW * kStages * kStageB);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, tq4 = lane & 3;
    uint8_t* ring = smem + (size_t)warp * kStages * kStageB;
    const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;

    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[b] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    const int64_t s0 = (int64_t)split * a.split_tokens;
    const int64_t s1 = (s0 + a.split_tokens < Tb) ? s0 + a.split_tokens : Tb;
    const int nchunk = s1 > s0 ? (int)((s1 - s0 + kChunk - 1) / kChunk) : 0;
    const int nmine = nchunk > warp ? (nchunk - warp + kNW - 1) / kNW : 0;
    const int64_t seq = (int64_t)b * a.Hkv + hkv;
    const int64_t kbb = block_bytes(kD, true), vbb = block_bytes(kD, false);

    if (lane == 0)
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&bars[warp * kStages + s]), 1);
    fence_mbar_init();
    __syncwarp();

    // issue the six bulk copies of chunk i of this warp into stage i % kStages
    auto issue = [&](int i) {
        const int64_t t0 = s0 + (int64_t)(warp + i * kNW) * kChunk;     // multiple of 32
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

    // A operands: rows gr (hi) and gr + 8 (lo) of query head gr of this kv head
    uint32_t aq[8][4], au[8][4];
    {
        const bool live = gr < G;
        const int64_t bh = (int64_t)b * a.Hq + (int64_t)hkv * G + (live ? gr : 0);
        const float* qp = a.qp + bh * kD;
        const float* up = a.up + bh * kD;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            const int c0 = 16 * kc + 2 * tq4;
            float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f, y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
            if (live) {
                x0 = qp[c0]; x1 = qp[c0 + 1]; x2 = qp[c0 + 8]; x3 = qp[c0 + 9];
                y0 = up[c0]; y1 = up[c0 + 1]; y2 = up[c0 + 8]; y3 = up[c0 + 9];
            }
            split_hilo(x0, x1, aq[kc][0], aq[kc][1]);
            split_hilo(x2, x3, aq[kc][2], aq[kc][3]);
            split_hilo(y0, y1, au[kc][0], au[kc][1]);
            split_hilo(y2, y3, au[kc][2], au[kc][3]);
        }
    }
    const uint32_t lut[4] = {a.cb.lut_lo[0], a.cb.lut_lo[1], a.cb.lut_hi[0], a.cb.lut_hi[1]};

    float o[16][4];
#pragma unroll
    for (int ct = 0; ct < 16; ++ct) o[ct][0] = o[ct][1] = o[ct][2] = o[ct][3] = 0.f;
    float mrun = -INFINITY, lrun = 0.f;
    bool failed = false;

    for (int i = 0; i < nmine; ++i) {
        const uint32_t bar = smem_u32(&bars[warp * kStages + (i % kStages)]);
        if (!mbar_wait_bounded(bar, (uint32_t)((i / kStages) & 1))) {
            failed = true;
            if (lane == 0) atomicExch(a.err, 1);
            // bounded wait for this warp's copies still in flight, then stop
            for (int j = i; j < nmine && j < i + kStages; ++j)
                mbar_wait_bounded(smem_u32(&bars[warp * kStages + (j % kStages)]), (uint32_t)((j / kStages) & 1));
            break;
        }
        const uint8_t* st = ring + (i % kStages) * kStageB;
        const int64_t tok0 = s0 + (int64_t)(warp + i * kNW) * kChunk;
        const int nvalid = (int)((s1 - tok0) < kChunk ? (s1 - tok0) : kChunk);

#pragma unroll 1
        for (int kt = 0; kt < kChunk / 16; ++kt) {
            if (kt * 16 >= nvalid) break;
            // ---------------- scores for the two 8-token tiles
            float sc[2][4];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int tok = kt * 16 + tt * 8 + gr;                      // B column of this lane
                uint32_t sel[4];
                code_selectors(st + kOffKc + tok * kCodeB + tq4 * 12, sel);
                const uint32_t nsg = ~*reinterpret_cast<const uint32_t*>(st + kOffKs + tok * kSignB + tq4 * 4);
                const uint32_t gb = *reinterpret_cast<const uint16_t*>(st + kOffKg + 2 * tok);
                const uint32_t gg = gb | (gb << 16);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kc = 0; kc < 8; ++kc) {
                    uint32_t b0, b1;
                    dequant4(sel_for(sel, kc), lut, b0, b1);
                    mma16816(acc, aq[kc], b0, b1);
                }
#pragma unroll
                for (int kc = 0; kc < 8; ++kc) {
                    const uint32_t b0 = gg ^ ((nsg << (15 - 2 * kc)) & 0x80008000u);
                    const uint32_t b1 = gg ^ ((nsg << (14 - 2 * kc)) & 0x80008000u);
                    mma16816(acc, au[kc], b0, b1);
                }
                sc[tt][0] = acc[0] + acc[2];                                 // token 2 tq4, head gr
                sc[tt][1] = acc[1] + acc[3];                                 // token 2 tq4 + 1
            }
            // ---------------- online softmax (log2 units), per head gr
            float s[4], nvv[4];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t0 = kt * 16 + tt * 8 + 2 * tq4;
                const float2 nk = __half22float2(*reinterpret_cast<const __half2*>(st + kOffKn + 2 * t0));
                const float2 nv = __half22float2(*reinterpret_cast<const __half2*>(st + kOffVn + 2 * t0));
                s[2 * tt] = (t0 < nvalid) ? a.scale_log2 * nk.x * sc[tt][0] : -INFINITY;
                s[2 * tt + 1] = (t0 + 1 < nvalid) ? a.scale_log2 * nk.y * sc[tt][1] : -INFINITY;
                nvv[2 * tt] = nv.x;
                nvv[2 * tt + 1] = nv.y;
            }
            float mt = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
            mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 2));
            const float mnew = fmaxf(mrun, mt);
            if (__any_sync(kFull, mnew > mrun)) {
                const float corr = (mnew == -INFINITY) ? 1.f : exp2f(mrun - mnew);
                lrun *= corr;
#pragma unroll
                for (int ct = 0; ct < 16; ++ct) {
                    o[ct][0] *= corr; o[ct][1] *= corr; o[ct][2] *= corr; o[ct][3] *= corr;
                }
                mrun = mnew;
            }
            float pv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float p = (s[k] == -INFINITY) ? 0.f : exp2f(s[k] - mrun);
                lrun += p;
                pv[k] = (p == 0.f) ? 0.f : p * nvv[k];
            }
            uint32_t ap[4];
            split_hilo(pv[0], pv[1], ap[0], ap[1]);
            split_hilo(pv[2], pv[3], ap[2], ap[3]);
            if (gr >= G) ap[0] = ap[1] = ap[2] = ap[3] = 0u;
            // ---------------- values: O += P V
            uint32_t vs0[4], vs1[4];
            code_selectors(st + kOffVc + (kt * 16 + gr) * kCodeB + tq4 * 12, vs0);
            code_selectors(st + kOffVc + (kt * 16 + 8 + gr) * kCodeB + tq4 * 12, vs1);
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                uint32_t x0, x1, y0, y1;
                dequant4(sel_for(vs0, kc), lut, x0, x1);       // tokens 0..7 of the tile
                dequant4(sel_for(vs1, kc), lut, y0, y1);       // tokens 8..15
                mma16816(o[2 * kc], ap, movmatrix_t(x0), movmatrix_t(y0));
                mma16816(o[2 * kc + 1], ap, movmatrix_t(x1), movmatrix_t(y1));
            }
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nmine) {
            fence_proxy_async();
            issue(i + kStages);
        }
    }
    if (failed) {
        mrun = -INFINITY;
        lrun = 0.f;
    }
    lrun += __shfl_xor_sync(kFull, lrun, 1);
    lrun += __shfl_xor_sync(kFull, lrun, 2);

    // ---------------- merge the warps of the CTA into one partial per head
    __syncwarp();
    float* wbuf = reinterpret_cast<float*>(ring);             // [G][kD + 2], in this warp's own ring
    if (gr < G) {
#pragma unroll
        for (int ct = 0; ct < 16; ++ct) {
            const int c = 8 * ct + 2 * tq4;
            wbuf[gr * (kD + 2) + c] = o[ct][0] + o[ct][2];
            wbuf[gr * (kD + 2) + c + 1] = o[ct][1] + o[ct][3];
        }
        if (tq4 == 0) {
            wbuf[gr * (kD + 2) + kD] = mrun;
            wbuf[gr * (kD + 2) + kD + 1] = lrun;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kD; idx += kNW * 32) {
        const int g = idx / kD, j = idx % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNW; ++w)
            M = fmaxf(M, reinterpret_cast<const float*>(smem + (size_t)w * kStages * kStageB)[g * (kD + 2) + kD]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kNW; ++w) {
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

size_t decode_mma_smem_bytes() { return (size_t)kNW * kStages * kStageB + (size_t)kNW * kStages * 8; }

cudaError_t launch_decode_mma(int d, int G, const DecArgs& a, cudaStream_t s) {
    if (d != kD || G < 1 || G > 8) return cudaErrorInvalidValue;
    if (a.B * a.Hkv == 0) return cudaSuccess;
    const size_t smem = decode_mma_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(tq_decode_mma128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.nsplit, (unsigned)a.Hkv, (unsigned)a.B);
    tq_decode_mma128_kernel<<<grid, kNW * 32, smem, s>>>(a, G);
    return cudaGetLastError();
}

int decode_mma_chunk_tokens() { return kChunk; }
int decode_mma_warps() { return kNW; }

}  // namespace tqi
