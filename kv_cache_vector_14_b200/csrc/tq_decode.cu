// Decode attention over the packed TurboQuant cache, for sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com): hybrid V2+V3 section (dequantisation fused
// into the attention kernel), K section (the QJL bit corrects inner-product
// scores), V section (V carries no QJL bit).  Per query head, with
// q' = H D q and u = S q':
//   s_t = scale * n_t * (<q', c[idx_t]> + gamma_t * sqrt(pi/2)/m * <u, 2 sigma_t - 1>)
//   out = D H sum_t softmax(s)_t * nv_t * c[idxv_t]
// Three kernels: the query prologue (q', u), split-K attention over token
// ranges writing (max, sum, rotated accumulator) partials, and the combine
// kernel (log-sum-exp merge, one inverse transform per head).
#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;

template <int DT>
__device__ __forceinline__ float load_q(const void* p, int64_t i) {
    if constexpr (DT == TQ_F32) return __ldg(static_cast<const float*>(p) + i);
    else if constexpr (DT == TQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    else return __half2float(static_cast<const __half*>(p)[i]);
}

// In-place unnormalised Walsh-Hadamard butterflies of NH vectors [NH][D] in
// shared memory, D threads; caller synchronises before and after.
template <int D, int NH>
__device__ void smem_fwht(float* v) {
    const int j = threadIdx.x;
#pragma unroll 1
    for (int h = 1; h < D; h <<= 1) {
        if ((j & h) == 0) {
#pragma unroll
            for (int k = 0; k < NH; ++k) {
                const float a = v[k * D + j], b = v[k * D + j + h];
                v[k * D + j] = a + b;
                v[k * D + j + h] = a - b;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- prologue
// q' = H D q / sqrt(d) and up = sqrt(pi/2)/m * S q'.  A CTA takes QH = D / kRC
// query heads and one chunk of kRC rows of S: warp k transforms head k in
// registers (coordinate lane + 32 r in element r; butterflies over the lane
// bits by shuffles, then over r, the levels in the same order as a butterfly
// over the whole index, so the sums are the same) while the kRC columns of
// S^T it needs are staged (one L2 read of S per head group).  Warp w then sums coordinates [32 w, 32 w + 32) for row
// `lane` of the chunk and all QH heads at once (each staged S value is read
// once per CTA), and the QH partial sums of every output are added in warp
// order.  The CTAs of row chunk 0 also store q'.
constexpr int kRC = 32;

template <int D, int DT>
__global__ void __launch_bounds__(D) tq_prologue_kernel(const void* q, int64_t BHq, const float* dsign,
                                                        const float* ST, float* qp, float* up) {
    constexpr int QH = D / kRC;                           // heads per CTA = warps per CTA
    __shared__ __align__(16) float v[QH * D];
    __shared__ __align__(16) float sst[D * kRC];          // sst[j][i] = S[rc*kRC + i][j]; then partial sums
    pdl_trigger();                                        // the split-K kernel may start its set-up
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t h0 = (int64_t)blockIdx.x * QH;
    const int rc = blockIdx.y;
    // the query loads go out first: the rotation waits for them, not for S
    constexpr int R = D / 32;
    const int64_t hw = h0 + warp;                        // this warp's head
    float x[R];
#pragma unroll
    for (int r = 0; r < R; ++r) x[r] = (hw < BHq) ? load_q<DT>(q, hw * D + lane + 32 * r) : 0.f;
    for (int i = t; i < D * kRC / 4; i += D) {          // in flight during the rotation below
        const int jr = i / (kRC / 4), c4 = i % (kRC / 4);
        cp_async16(reinterpret_cast<float4*>(sst) + i, reinterpret_cast<const float4*>(ST + (size_t)jr * D + rc * kRC) + c4);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) x[r] *= dsign[lane + 32 * r];
#pragma unroll
    for (int hb = 1; hb < 32; hb <<= 1)
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float p = __shfl_xor_sync(kFull, x[r], hb);
            x[r] = (lane & hb) ? (p - x[r]) : (x[r] + p);
        }
#pragma unroll
    for (int hb = 1; hb < R; hb <<= 1)
#pragma unroll
        for (int r = 0; r < R; ++r)
            if ((r & hb) == 0) {
                const float u = x[r], w = x[r | hb];
                x[r] = u + w;
                x[r | hb] = u - w;
            }
    const float inv = 1.0f / sqrtf((float)D);
#pragma unroll
    for (int r = 0; r < R; ++r) v[warp * D + lane + 32 * r] = x[r] * inv;
    cp_async_wait_all();
    __syncthreads();
    float acc[QH];
#pragma unroll
    for (int k = 0; k < QH; ++k) acc[k] = 0.f;
#pragma unroll 2
    for (int jj = 32 * warp; jj < 32 * warp + 32; jj += 4) {
        const float s0 = sst[jj * kRC + lane], s1 = sst[(jj + 1) * kRC + lane];
        const float s2 = sst[(jj + 2) * kRC + lane], s3 = sst[(jj + 3) * kRC + lane];
#pragma unroll
        for (int k = 0; k < QH; ++k) {
            const float4 vv = *reinterpret_cast<const float4*>(&v[k * D + jj]);
            acc[k] = fmaf(s3, vv.w, fmaf(s2, vv.z, fmaf(s1, vv.y, fmaf(s0, vv.x, acc[k]))));
        }
    }
    __syncthreads();                                      // sst is reused for the partial sums
#pragma unroll
    for (int k = 0; k < QH; ++k) sst[(warp * QH + k) * 32 + lane] = acc[k];
    __syncthreads();
    const int i = t % kRC, k = t / kRC;
    float u = 0.f;
#pragma unroll
    for (int w = 0; w < QH; ++w) u += sst[(w * QH + k) * 32 + i];
    const float cq = 1.2533141373155003f / (float)D;       // sqrt(pi/2) / m
    const int64_t h = h0 + k;
    if (h < BHq) up[h * D + rc * kRC + i] = cq * u;
    if (rc == 0) {
#pragma unroll
        for (int kk = 0; kk < QH; ++kk)
            if (h0 + kk < BHq) qp[(h0 + kk) * D + t] = v[kk * D + t];
    }
    pdl_wait();          // chained after an encode (fused step): complete only after it
}

// Query heads per SIMT CTA: G itself for 1, 2 and 4, else groups of up to 8.
int simt_heads_per_cta(int G) { return G <= 2 ? G : (G <= 4 ? 4 : 8); }

// ---------------------------------------------------------------- SIMT decode
// One CTA (4 warps) per (split, kv head, batch) and group of up to GT of the
// kv head's G query heads (grid.y = Hkv x head groups).  Each warp walks a quarter of
// the split's token range one token at a time; lane l owns coordinates
// j = l + 32 r.  Partial scores are reduced across the warp, the online
// softmax runs in log2 units, and the four warps are merged through shared
// memory into one partial per query head.
template <int D>
__device__ __forceinline__ int code_from_words(const uint32_t* w, int j) {
    const int s = j >> 7, t = slot_of(j), i = slot_pos(j);
    if constexpr (D == 64) {             // word t: codes 0..7; halfword t (words 4, 5): codes 8..11
        const uint32_t H = w[4 + (t >> 1)] >> (16 * (t & 1));
        if (i < 8) return (int)((w[t] >> (4 * i)) & 7u);
        if (i < 12) return (int)((H >> (4 * (i - 8))) & 7u);
        const int k = i - 12;
        return (int)(((w[t] >> (4 * k + 3)) & 1u) | (((w[t] >> (4 * k + 19)) & 1u) << 1) |
                     (((H >> (4 * k + 3)) & 1u) << 2));
    }
    const uint32_t* W = w + 12 * s + 3 * t;
    if (i < 24) return (int)((W[i >> 3] >> (4 * (i & 7))) & 7u);
    const int k = i - 24;
    return (int)(((W[0] >> (4 * k + 3)) & 1u) | (((W[1] >> (4 * k + 3)) & 1u) << 1) |
                 (((W[2] >> (4 * k + 3)) & 1u) << 2));
}
template <int D>
__device__ __forceinline__ int sign_from_words(const uint32_t* w, int j) {
    const int s = j >> 7, t = slot_of(j), i = slot_pos(j);
    if constexpr (D == 64) return (int)((w[t >> 1] >> (16 * (t & 1) + i)) & 1u);
    const int bit = (i & 1) ? 16 + (i >> 1) : (i >> 1);
    return (int)((w[4 * s + t] >> bit) & 1u);
}

template <int D, int GT, bool QJL>
__global__ void __launch_bounds__(128) tq_decode_simt_kernel(const DecArgs a, int Gq) {
    constexpr int R = D / 32;
    constexpr int G = GT;                                  // query heads per CTA (slots; Gl of them live)
    __shared__ float sC[8];
    __shared__ float sm[4][G][2];
    __shared__ float sacc[4][G][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, b = blockIdx.z;
    const int hgroups = (Gq + GT - 1) / GT;
    const int hkv = blockIdx.y / hgroups;
    const int g0 = (blockIdx.y - hkv * hgroups) * GT;
    const int Gl = Gq - g0 < GT ? Gq - g0 : GT;
    const int64_t hbase = (int64_t)b * a.Hq + (int64_t)hkv * Gq + g0;
    if (threadIdx.x < 8) sC[threadIdx.x] = a.cb.c[threadIdx.x];

    int64_t Tb = a.seq_lens ? (int64_t)a.seq_lens[b] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.Tcap ? a.Tcap : Tb);
    const int64_t s0 = (int64_t)split * a.split_tokens;
    const int64_t s1 = (s0 + a.split_tokens < Tb) ? s0 + a.split_tokens : Tb;
    const int64_t len = s1 > s0 ? s1 - s0 : 0;
    const int64_t per = (len + 3) / 4;
    const int64_t w0 = s0 + warp * per;
    const int64_t w1 = (w0 + per < s1) ? w0 + per : s1;

    const int64_t seq = (int64_t)b * a.Hkv + hkv;
    const int64_t kbb = block_bytes(D, QJL), vbb = block_bytes(D, false);
    const int64_t knorm = kBlockT * (code_bytes(D) + (QJL ? sign_bytes(D) : 0));
    pdl_wait();                                           // q' and u' from the prologue
    float q[G][R], u[G][R], acc[G][R], mrun[G], lrun[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int64_t bh = hbase + (g < Gl ? g : 0);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            q[g][r] = g < Gl ? a.qp[bh * D + lane + 32 * r] : 0.f;
            u[g][r] = g < Gl ? a.up[bh * D + lane + 32 * r] : 0.f;
            acc[g][r] = 0.f;
        }
        mrun[g] = -INFINITY;
        lrun[g] = 0.f;
    }
    __syncthreads();

    for (int64_t t = w0; t < w1; ++t) {
        const int64_t kblk = cache_block(a.ktable, a.kpool, a.NB, seq, t >> 6, a.err);
        const int64_t vblk = cache_block(a.vtable, a.vpool, a.NB, seq, t >> 6, a.err);
        const uint8_t* kb = a.kc + (kblk >= 0 ? kblk : 0) * kbb;    // a bad table entry reads block 0
        const uint8_t* vb = a.vc + (vblk >= 0 ? vblk : 0) * vbb;
        const int tau = (int)(t & 63);
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(kb + tau * code_bytes(D));
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(kb + kBlockT * code_bytes(D) + tau * sign_bytes(D));
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(vb + tau * code_bytes(D));
        const float nk = __half2float(reinterpret_cast<const __half*>(kb + knorm)[tau]);
        const float gk = QJL ? __half2float(reinterpret_cast<const __half*>(kb + knorm + 2 * kBlockT)[tau]) : 0.f;
        const float nv = __half2float(reinterpret_cast<const __half*>(vb + kBlockT * code_bytes(D))[tau]);
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = 0.f;
        float cv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int j = lane + 32 * r;
            const float ck = sC[code_from_words<D>(kw, j)];
            cv[r] = sC[code_from_words<D>(vw, j)];
            if constexpr (QJL) {
                const float sg = sign_from_words<D>(sw, j) ? gk : -gk;
#pragma unroll
                for (int g = 0; g < G; ++g) part[g] = fmaf(q[g][r], ck, fmaf(u[g][r], sg, part[g]));
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g) part[g] = fmaf(q[g][r], ck, part[g]);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part[g] += __shfl_xor_sync(kFull, part[g], o);
            const float s = a.scale_log2 * nk * part[g];
            const float mnew = fmaxf(mrun[g], s);
            const float corr = exp2f(mrun[g] - mnew);
            const float p = exp2f(s - mnew);
            lrun[g] = lrun[g] * corr + p;
            const float pv = p * nv;
#pragma unroll
            for (int r = 0; r < R; ++r) acc[g][r] = fmaf(pv, cv[r], acc[g][r] * corr);
            mrun[g] = mnew;
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) { sm[warp][g][0] = mrun[g]; sm[warp][g][1] = lrun[g]; }
#pragma unroll
        for (int r = 0; r < R; ++r) sacc[warp][g][lane + 32 * r] = acc[g][r];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < Gl * D; idx += 128) {
        const int g = idx / D, j = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w][g][0]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = exp2f(sm[w][g][0] - M);   // empty warps: exp2(-inf) = 0
                L = fmaf(f, sm[w][g][1], L);
                A = fmaf(f, sacc[w][g][j], A);
            }
        }
        const int64_t bh = hbase + g;
        const int64_t pidx = bh * a.nsplit + split;
        a.part_acc[pidx * D + j] = A;
        if (j == 0) { a.part_ml[2 * pidx] = M; a.part_ml[2 * pidx + 1] = L; }
    }
}

// ---------------------------------------------------------------- combine
// One CTA of D threads per (batch, query head): log-sum-exp merge of the
// split partials, division by the softmax sum, one inverse transform D H.
// The per-split (max, sum) pairs go through shared memory once; each thread
// then sums its coordinate over the splits with independent loads.
constexpr int kMaxSplitSmem = kMaxSplits;

template <int D>
__global__ void __launch_bounds__(D) tq_combine_kernel(const float* part_ml, const float* part_acc, int nsplit,
                                                       const float* dsign, float* out) {
    __shared__ float v[D];
    __shared__ float wgt[kMaxSplitSmem];
    __shared__ float red[D / 32];
    __shared__ float sM, sL;
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    const int64_t bh = blockIdx.x;
    pdl_wait();                                           // partials of the split-K kernel
    const float* ml = part_ml + bh * nsplit * 2;
    const int ns = nsplit < kMaxSplitSmem ? nsplit : kMaxSplitSmem;
    float m = -INFINITY;
    for (int s = j; s < ns; s += D) m = fmaxf(m, ml[2 * s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (j == 0) {
        float M = -INFINITY;
        for (int w = 0; w < D / 32; ++w) M = fmaxf(M, red[w]);
        sM = M;
    }
    __syncthreads();
    const float M = sM;
    float l = 0.f;
    for (int s = j; s < ns; s += D) {
        const float f = (M == -INFINITY) ? 0.f : exp2f(ml[2 * s] - M);
        wgt[s] = f;
        l = fmaf(f, ml[2 * s + 1], l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(kFull, l, o);
    __syncthreads();
    if (lane == 0) red[warp] = l;
    __syncthreads();
    if (j == 0) {
        float L = 0.f;
        for (int w = 0; w < D / 32; ++w) L += red[w];
        sL = L;
    }
    __syncthreads();
    const float* acc = part_acc + bh * nsplit * D + j;
    float A0 = 0.f, A1 = 0.f, A2 = 0.f, A3 = 0.f;
    int s = 0;
    for (; s + 4 <= ns; s += 4) {
        A0 = fmaf(wgt[s], acc[(size_t)s * D], A0);
        A1 = fmaf(wgt[s + 1], acc[(size_t)(s + 1) * D], A1);
        A2 = fmaf(wgt[s + 2], acc[(size_t)(s + 2) * D], A2);
        A3 = fmaf(wgt[s + 3], acc[(size_t)(s + 3) * D], A3);
    }
    for (; s < ns; ++s) A0 = fmaf(wgt[s], acc[(size_t)s * D], A0);
    const float L = sL;
    v[j] = (L > 0.f) ? ((A0 + A1) + (A2 + A3)) / L : 0.f;
    __syncthreads();
    smem_fwht<D, 1>(v);
    out[bh * D + j] = dsign[j] * v[j] * (1.0f / sqrtf((float)D));
}

template <int D, int DT>
cudaError_t launch_prologue_t(dim3 grid, bool pdl, const void* q, int64_t BHq, const float* dsign, const float* st,
                              float* qp, float* up, cudaStream_t s) {
    const cudaError_t e = set_carveout_once<tq_prologue_kernel<D, DT>>();
    if (e != cudaSuccess) return e;
    if (pdl) return launch_pdl(tq_prologue_kernel<D, DT>, grid, dim3(D), 0, s, q, BHq, dsign, st, qp, up);
    tq_prologue_kernel<D, DT><<<grid, D, 0, s>>>(q, BHq, dsign, st, qp, up);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_prologue_d(const void* q, tq_dtype dt, int64_t BHq, const float* dsign, const float* st,
                              float* qp, float* up, bool pdl, cudaStream_t s) {
    const int64_t groups = (BHq + D / kRC - 1) / (D / kRC);
    if (groups == 0) return cudaSuccess;
    const dim3 grid((unsigned)groups, D / kRC);
    switch (dt) {
        case TQ_F32: return launch_prologue_t<D, TQ_F32>(grid, pdl, q, BHq, dsign, st, qp, up, s);
        case TQ_BF16: return launch_prologue_t<D, TQ_BF16>(grid, pdl, q, BHq, dsign, st, qp, up, s);
        case TQ_F16: return launch_prologue_t<D, TQ_F16>(grid, pdl, q, BHq, dsign, st, qp, up, s);
    }
    return cudaErrorInvalidValue;
}

template <int D, int GT, bool QJL>
cudaError_t launch_simt(int G, const DecArgs& a, cudaStream_t s) {
    dim3 grid(a.nsplit, (unsigned)(a.Hkv * ((G + GT - 1) / GT)), (unsigned)a.B);
    return launch_pdl(tq_decode_simt_kernel<D, GT, QJL>, grid, dim3(128), 0, s, a, G);
}

template <int D, bool QJL>
cudaError_t launch_simt_g(int G, const DecArgs& a, cudaStream_t s) {
    switch (simt_heads_per_cta(G)) {
        case 1: return launch_simt<D, 1, QJL>(G, a, s);
        case 2: return launch_simt<D, 2, QJL>(G, a, s);
        case 4: return launch_simt<D, 4, QJL>(G, a, s);
        case 8: return launch_simt<D, 8, QJL>(G, a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prologue(int d, const void* q, tq_dtype dt, int64_t BHq, const float* dsign, const float* st,
                            float* qp, float* up, bool pdl, cudaStream_t s) {
    if (d == 64) return launch_prologue_d<64>(q, dt, BHq, dsign, st, qp, up, pdl, s);
    if (d == 128) return launch_prologue_d<128>(q, dt, BHq, dsign, st, qp, up, pdl, s);
    if (d == 256) return launch_prologue_d<256>(q, dt, BHq, dsign, st, qp, up, pdl, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_simt(int d, int G, bool qjl, const DecArgs& a, cudaStream_t s) {
    if (a.B * a.Hkv == 0) return cudaSuccess;
    if (d == 64) return qjl ? launch_simt_g<64, true>(G, a, s) : launch_simt_g<64, false>(G, a, s);
    if (d == 128) return qjl ? launch_simt_g<128, true>(G, a, s) : launch_simt_g<128, false>(G, a, s);
    if (d == 256) return qjl ? launch_simt_g<256, true>(G, a, s) : launch_simt_g<256, false>(G, a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_combine(int d, int64_t BHq, int nsplit, const float* part_ml, const float* part_acc,
                           const float* dsign, float* out, cudaStream_t s) {
    if (BHq == 0) return cudaSuccess;
    cudaError_t e = d == 64 ? set_carveout_once<tq_combine_kernel<64>>()
                    : d == 128 ? set_carveout_once<tq_combine_kernel<128>>() : set_carveout_once<tq_combine_kernel<256>>();
    if (e != cudaSuccess) return e;
    if (d == 64)
        return launch_pdl(tq_combine_kernel<64>, dim3((unsigned)BHq), dim3(64), 0, s, part_ml, part_acc, nsplit, dsign, out);
    if (d == 128)
        return launch_pdl(tq_combine_kernel<128>, dim3((unsigned)BHq), dim3(128), 0, s, part_ml, part_acc, nsplit, dsign, out);
    if (d == 256)
        return launch_pdl(tq_combine_kernel<256>, dim3((unsigned)BHq), dim3(256), 0, s, part_ml, part_acc, nsplit, dsign, out);
    return cudaErrorInvalidValue;
}

}  // namespace tqi

namespace tqi {

cudaError_t launch_decode_simt(int d, int G, bool qjl, const DecArgs& a, cudaStream_t s);
cudaError_t launch_decode_mma(int d, int G, bool qjl, const DecArgs& a, cudaStream_t s);
int decode_mma_chunk_tokens(int d);
int decode_mma_warps(int G);

// The tensor-core kernel covers head_dim 64, 128 and 256 and any group size
// (query heads in CTAs of up to 8 per kv head).
bool mma_supported(int d, int G) { return head_dim_ok(d) && G >= 1; }

// CTAs per (split, kv head, batch): query-head groups of the kernel that runs.
int decode_head_groups(bool use_mma, int G) {
    const int per = use_mma ? 8 : simt_heads_per_cta(G);
    return (G + per - 1) / per;
}

int decode_ctas_per_sm(bool use_mma) { return use_mma ? 1 : 4; }
int decode_chunk_tokens(int d, bool use_mma) { return use_mma ? decode_mma_chunk_tokens(d) : kBlockT; }
int decode_warps(bool use_mma, int G) { return use_mma ? decode_mma_warps(G) : 4; }

cudaError_t launch_decode(int d, int G, bool use_mma, bool qjl, const DecArgs& a, cudaStream_t s) {
    return use_mma ? launch_decode_mma(d, G, qjl, a, s) : launch_decode_simt(d, G, qjl, a, s);
}

}  // namespace tqi
