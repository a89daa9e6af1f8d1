// TurboQuant K/V encode kernels for sm_100a.
//
// Page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD Expert
// Streamingを実装" (ai-heartland.com), section "K-Cache圧縮：3-bit PolarQuant +
// 1-bit QJL = 4.25 bits/dim" (steps 1-5) and section "V-Cache圧縮：3-bit
// PolarQuant = 3.125 bits/dim" (steps 1-3, no QJL).
//
// Head dims 64 and 256 (head_dim 128 runs on the tensor-core kernels of
// tq_encode_tc.cu).  One CTA of 8 warps handles tiles of 32 vectors (4 per warp):
//   phase 1, one warp per vector: coalesced load, ||x|| by warp reduction,
//     sign flip + Walsh-Hadamard butterflies (register stages for the lane's
//     own coordinates j = lane + 32 r, shuffle stages across lanes), scale by
//     1 / (||x|| sqrt(d)), bucketize against the 7 boundaries, residual and
//     its norm gamma (K).  Codes are staged in shared memory in slot order.
//   phase 2 (K only): the JL projection Z = R S^T of the tile as an fp32
//     contraction from shared memory, each lane owning the JL rows whose sign
//     bits form one packed word, so one ballot yields each stored word.
//   phase 3: the staged codes are packed into the nibble words of the layout
//     and stored with coalesced 4-byte stores.
#include "tq_internal.h"

namespace tqi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;

template <int DT>
__device__ __forceinline__ float load_x(const void* p, int64_t i) {
    if constexpr (DT == TQ_F32) return __ldg(static_cast<const float*>(p) + i);
    else if constexpr (DT == TQ_BF16)
        return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    else return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Pack 8 byte-sized values (< 16) held in two words into 8 nibbles.
__device__ __forceinline__ uint32_t nibbles8(uint32_t lo4, uint32_t hi4) {
    uint32_t a = (lo4 | (lo4 >> 4)) & 0x00FF00FFu;
    a = (a | (a >> 8)) & 0x0000FFFFu;
    uint32_t b = (hi4 | (hi4 >> 4)) & 0x00FF00FFu;
    b = (b | (b >> 8)) & 0x0000FFFFu;
    return a | (b << 16);
}

// Shared-memory index of coordinate j's staged code: slots of 32 positions
// per 128-coordinate slice (16 positions per slot at d = 64).
template <int D>
__device__ __forceinline__ int stage_at(int j) {
    if constexpr (D == 64) return slot_of(j) * 16 + slot_pos(j);
    else return (j >> 7) * 128 + slot_of(j) * 32 + slot_pos(j);
}

// Code word w (0 .. 3D/32 - 1) of one token, from its codes staged in slot
// order (one byte per code).
template <int D>
__device__ __forceinline__ uint32_t code_word(const uint8_t* sc, int w) {
    if constexpr (D == 64) {
        if (w < 4) {                      // word t: codes 0..7 of slot t, bits 0 and 1 of codes 12..15
            const uint32_t* sw = reinterpret_cast<const uint32_t*>(sc + 16 * w);
            const uint32_t tl = nibbles8(sw[3], 0u);
            return nibbles8(sw[0], sw[1]) | ((tl & 0x1111u) << 3) | (((tl >> 1) & 0x1111u) << 19);
        }
        uint32_t r = 0;                   // halfwords of slots 2(w-4), 2(w-4)+1: codes 8..11, bit 2 of 12..15
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t* sw = reinterpret_cast<const uint32_t*>(sc + 16 * (2 * (w - 4) + hh));
            const uint32_t half = nibbles8(sw[2], 0u) | (((nibbles8(sw[3], 0u) >> 2) & 0x1111u) << 3);
            r |= half << (16 * hh);
        }
        return r;
    } else {
        const int s = w / 12, t = (w % 12) / 3, g = w % 3;
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(sc + s * 128 + t * 32);
        const uint32_t main = nibbles8(sw[2 * g], sw[2 * g + 1]);
        const uint32_t tail = nibbles8(sw[6], sw[7]);
        return main | (((tail >> g) & 0x11111111u) << 3);
    }
}

template <int D, bool IS_K, int TV>
struct EncSmem {
    static constexpr int R = D / 32;
    static constexpr int JC = (D == 128) ? 128 : 64;           // JL columns resident at once
    static constexpr size_t s_bytes = IS_K ? (size_t)JC * D * 4 : 0;
    static constexpr size_t r_bytes = IS_K ? (size_t)TV * D * 4 : 0;
    static constexpr size_t code_bytes = (size_t)TV * D;
    static constexpr size_t total = s_bytes + r_bytes + code_bytes;
};

// TV vectors per tile (32 for bulk encodes, 8 when there are too few tiles to
// fill the GPU, e.g. appending one token per head).
template <int D, bool IS_K, int DT, int TV>
__global__ void __launch_bounds__(kThreads) tq_encode_kernel(const EncArgs a) {
    using SM = EncSmem<D, IS_K, TV>;
    constexpr int kTileV = TV;
    constexpr int kVecPerWarp = TV / 8;
    constexpr int R = SM::R;
    constexpr int JC = SM::JC;
    extern __shared__ __align__(16) unsigned char smem[];
    float* sS = reinterpret_cast<float*>(smem);                        // [JC][R][32]
    float* sR = reinterpret_cast<float*>(smem + SM::s_bytes);          // [kTileV][D]
    uint8_t* sCode = smem + SM::s_bytes + SM::r_bytes;                 // [kTileV][D], slot order
    __shared__ float sC[8];

    pdl_trigger();                 // a chained kernel may start (it waits for this one's writes)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + kTileV - 1) / kTileV;
    const int64_t bb = block_bytes(D, IS_K);
    const float sqrt_d = sqrtf((float)D);

    if (threadIdx.x < 8) sC[threadIdx.x] = a.cb.c[threadIdx.x];
    float dsg[R];
#pragma unroll
    for (int r = 0; r < R; ++r) dsg[r] = __ldg(a.dsign + lane + 32 * r);
    if constexpr (IS_K && D == 128) {
        for (int i = threadIdx.x; i < JC * D / 4; i += kThreads)
            reinterpret_cast<float4*>(sS)[i] = __ldg(reinterpret_cast<const float4*>(a.sthr) + i);
    }
    __syncthreads();

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        // ---------------- phase 1: one warp per vector, the warp's vectors
        // processed together so their shuffle chains overlap
        float x[kVecPerWarp][R], ss[kVecPerWarp];
        int64_t tt[kVecPerWarp], bh[kVecPerWarp];
        bool valid[kVecPerWarp];
#pragma unroll
        for (int vv = 0; vv < kVecPerWarp; ++vv) {
            const int64_t gv = tile * kTileV + warp * kVecPerWarp + vv;
            valid[vv] = gv < N;
            ss[vv] = 0.f;
            tt[vv] = valid[vv] ? gv % a.Tnew : 0;
            bh[vv] = valid[vv] ? gv / a.Tnew : 0;
            const int64_t h = bh[vv] % a.Hkv, b = bh[vv] / a.Hkv;
            const int64_t base = b * a.sb + h * a.sh + tt[vv] * a.st;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                x[vv][r] = valid[vv] ? load_x<DT>(a.x, base + lane + 32 * r) : 0.f;
                ss[vv] = fmaf(x[vv][r], x[vv][r], ss[vv]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int vv = 0; vv < kVecPerWarp; ++vv) ss[vv] += __shfl_xor_sync(kFull, ss[vv], o);
        // sign flip, then butterflies over lane bits (coordinate bits 0..4)
#pragma unroll
        for (int vv = 0; vv < kVecPerWarp; ++vv)
#pragma unroll
            for (int r = 0; r < R; ++r) x[vv][r] *= dsg[r];
#pragma unroll
        for (int hb = 1; hb < 32; hb <<= 1) {
#pragma unroll
            for (int vv = 0; vv < kVecPerWarp; ++vv)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float p = __shfl_xor_sync(kFull, x[vv][r], hb);
                    x[vv][r] = (lane & hb) ? (p - x[vv][r]) : (x[vv][r] + p);
                }
        }
        // butterflies over register bits (coordinate bits 5..)
#pragma unroll
        for (int hb = 1; hb < R; hb <<= 1)
#pragma unroll
            for (int vv = 0; vv < kVecPerWarp; ++vv)
#pragma unroll
                for (int r = 0; r < R; ++r)
                    if ((r & hb) == 0) {
                        const float u = x[vv][r], w = x[vv][r | hb];
                        x[vv][r] = u + w;
                        x[vv][r | hb] = u - w;
                    }
        float g2[kVecPerWarp];
#pragma unroll
        for (int vv = 0; vv < kVecPerWarp; ++vv) {
            const int v = warp * kVecPerWarp + vv;
            const float n = sqrtf(ss[vv]);
            const float nsd = n * sqrt_d;
            g2[vv] = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int j = lane + 32 * r;
                const float y = (n > 0.f) ? __fdiv_rn(x[vv][r], nsd) : 0.f;
                int code = 0;
#pragma unroll
                for (int i = 0; i < 7; ++i) code += (y >= a.cb.b[i]) ? 1 : 0;
                const float res = (n > 0.f) ? (y - sC[code]) : 0.f;
                g2[vv] = fmaf(res, res, g2[vv]);
                if constexpr (IS_K) sR[v * D + j] = res;
                sCode[v * D + stage_at<D>(j)] = (uint8_t)code;
            }
        }
        if constexpr (IS_K) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int vv = 0; vv < kVecPerWarp; ++vv) g2[vv] += __shfl_xor_sync(kFull, g2[vv], o);
        }
#pragma unroll
        for (int vv = 0; vv < kVecPerWarp; ++vv) {
            if (valid[vv] && lane == 0) {
                const int64_t t = a.t0 + tt[vv];
                const int64_t pb = cache_block(a.table, a.pool, a.NB, bh[vv], t >> 6, a.err);
                uint8_t* blk = a.cache + pb * bb;
                const int tau = (int)(t & 63);
                const int64_t norm_off = kBlockT * code_bytes(D) + (IS_K ? kBlockT * sign_bytes(D) : 0);
                if (pb >= 0) {
                    reinterpret_cast<__half*>(blk + norm_off)[tau] = __float2half_rn(sqrtf(ss[vv]));
                    if constexpr (IS_K)
                        reinterpret_cast<__half*>(blk + norm_off + 2 * kBlockT)[tau] = __float2half_rn(sqrtf(g2[vv]));
                }
            }
        }
        __syncthreads();

        // ---------------- phase 2 (K): z = S r for the tile, signs by ballot
        if constexpr (IS_K) {
            float z[kVecPerWarp][R];
#pragma unroll
            for (int vv = 0; vv < kVecPerWarp; ++vv)
#pragma unroll
                for (int r = 0; r < R; ++r) z[vv][r] = 0.f;
            for (int j0 = 0; j0 < D; j0 += JC) {
                if constexpr (D != 128) {
                    __syncthreads();
                    const float4* src = reinterpret_cast<const float4*>(a.sthr + (size_t)j0 * D);
                    for (int i = threadIdx.x; i < JC * D / 4; i += kThreads)
                        reinterpret_cast<float4*>(sS)[i] = __ldg(src + i);
                    __syncthreads();
                }
#pragma unroll 2
                for (int jj = 0; jj < JC; jj += 4) {
                    float4 rv[kVecPerWarp];
#pragma unroll
                    for (int vv = 0; vv < kVecPerWarp; ++vv)
                        rv[vv] = *reinterpret_cast<const float4*>(sR + (warp * kVecPerWarp + vv) * D + j0 + jj);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const float s = sS[((jj + q) * R + r) * 32 + lane];
#pragma unroll
                            for (int vv = 0; vv < kVecPerWarp; ++vv) {
                                const float rq = (q == 0) ? rv[vv].x : (q == 1) ? rv[vv].y : (q == 2) ? rv[vv].z : rv[vv].w;
                                z[vv][r] = fmaf(rq, s, z[vv][r]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int vv = 0; vv < kVecPerWarp; ++vv) {
                const int64_t gv = tile * kTileV + warp * kVecPerWarp + vv;
                uint32_t mine = 0;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint32_t w = __ballot_sync(kFull, z[vv][r] >= 0.f);
                    if (lane == r) mine = w;
                }
                if (gv < N && lane < R) {
                    const int64_t tt = gv % a.Tnew, bh = gv / a.Tnew, t = a.t0 + tt;
                    const int64_t pb = cache_block(a.table, a.pool, a.NB, bh, t >> 6, a.err);
                    uint32_t* sw = reinterpret_cast<uint32_t*>(a.cache + pb * bb + kBlockT * code_bytes(D) +
                                                               (t & 63) * sign_bytes(D));
                    if (pb >= 0) sw[lane] = mine;
                }
            }
        }

        // ---------------- phase 3: pack staged codes into the layout's words
        constexpr int W = 3 * D / 32;
#pragma unroll
        for (int vv = 0; vv < kVecPerWarp; ++vv) {
            const int v = warp * kVecPerWarp + vv;
            const int64_t gv = tile * kTileV + v;
            if (gv < N && lane < W) {
                const uint32_t word = code_word<D>(sCode + v * D, lane);
                const int64_t tt = gv % a.Tnew, bh = gv / a.Tnew, tok = a.t0 + tt;
                const int64_t pb = cache_block(a.table, a.pool, a.NB, bh, tok >> 6, a.err);
                if (pb >= 0) reinterpret_cast<uint32_t*>(a.cache + pb * bb + (tok & 63) * code_bytes(D))[lane] = word;
            }
        }
        __syncthreads();
    }
    pdl_wait();                    // when chained: complete only after the previous kernel
}

// ---------------------------------------------------------------- small batches (K)
// Appends of a few vectors per head: one warp per vector and four warps per
// CTA, so a 32-vector append runs on 8 SMs at once instead of one.  The JL
// rows are split over gridDim.y CTAs (kSmallRowGroups groups of 32 rows each),
// each staging only its rows of S (64 KB at d = 256) and writing only their
// sign words; every CTA repeats steps 1-4 for its vectors and the row-chunk-0
// CTA stores the codes and norms.  Each z_i accumulates over the columns in
// the same order as the tiled kernel, so both give bit-identical sign words.
constexpr int kSmallWarps = 4;
constexpr int kSmallRowGroups = 2;

template <int D, int DT>
__global__ void __launch_bounds__(kSmallWarps * 32) tq_encode_k_small_kernel(const EncArgs a) {
    constexpr int R = D / 32;
    constexpr int RG = kSmallRowGroups;             // row groups of 32 JL rows per CTA
    extern __shared__ __align__(16) float sS[];     // [D][RG][32]
    __shared__ __align__(16) float sr[kSmallWarps][D];
    __shared__ __align__(16) uint8_t scode[kSmallWarps][D];
    __shared__ float sC[8];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg0 = blockIdx.y * RG;                // first row group of this CTA
    if (threadIdx.x < 8) sC[threadIdx.x] = a.cb.c[threadIdx.x];
    {
        // this CTA's rows of the lane-ordered JL matrix: RG*32 floats per column,
        // all copies in flight at once (they overlap the vector's load and rotation)
        const float4* src = reinterpret_cast<const float4*>(a.sthr);
        for (int i = threadIdx.x; i < D * RG * 8; i += kSmallWarps * 32) {
            const int j = i / (RG * 8), c = i % (RG * 8);
            cp_async16(reinterpret_cast<float4*>(sS) + i, src + ((size_t)j * R + rg0) * 8 + c);
        }
    }
    __syncthreads();                                 // sC
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t gv0 = (int64_t)blockIdx.x * kSmallWarps + warp;
    const bool valid = gv0 < N;
    const int64_t gv = valid ? gv0 : N - 1;
    const int64_t tt = gv % a.Tnew, bh = gv / a.Tnew;
    const int64_t t = a.t0 + tt;
    const int64_t pb = valid ? cache_block(a.table, a.pool, a.NB, bh, t >> 6, a.err) : 0;
    uint8_t* blk = a.cache + (pb >= 0 ? pb : 0) * block_bytes(D, true);
    const bool wr = valid && pb >= 0;                 // this warp stores its vector
    const int64_t h = bh % a.Hkv, b = bh / a.Hkv;
    const int64_t base = b * a.sb + h * a.sh + tt * a.st;
    float x[R];
    float ss = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        x[r] = load_x<DT>(a.x, base + lane + 32 * r);
        ss = fmaf(x[r], x[r], ss);
        x[r] *= __ldg(a.dsign + lane + 32 * r);
    }
    ss = warp_sum(ss);
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
    const float n = sqrtf(ss);
    const float nsd = n * sqrtf((float)D);
    float g2 = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int j = lane + 32 * r;
        const float y = (n > 0.f) ? __fdiv_rn(x[r], nsd) : 0.f;
        int code = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) code += (y >= a.cb.b[i]) ? 1 : 0;
        const float res = (n > 0.f) ? (y - sC[code]) : 0.f;
        g2 = fmaf(res, res, g2);
        sr[warp][j] = res;
        scode[warp][stage_at<D>(j)] = (uint8_t)code;
    }
    g2 = warp_sum(g2);
    cp_async_wait_all();
    __syncthreads();                                 // this CTA's rows of S are staged
    const bool writer = wr && blockIdx.y == 0;
    if (writer && lane == 0) {
        const int64_t norm_off = kBlockT * code_bytes(D) + kBlockT * sign_bytes(D);
        reinterpret_cast<__half*>(blk + norm_off)[t & 63] = __float2half_rn(n);
        reinterpret_cast<__half*>(blk + norm_off + 2 * kBlockT)[t & 63] = __float2half_rn(sqrtf(g2));
    }
    __syncwarp();
    float z[RG];
#pragma unroll
    for (int k = 0; k < RG; ++k) z[k] = 0.f;
#pragma unroll 4
    for (int j = 0; j < D; ++j) {
        const float rj = sr[warp][j];
#pragma unroll
        for (int k = 0; k < RG; ++k) z[k] = fmaf(rj, sS[(j * RG + k) * 32 + lane], z[k]);
    }
    if (!valid) {
        pdl_wait();
        return;
    }
    uint32_t mine = 0;
#pragma unroll
    for (int k = 0; k < RG; ++k) {
        const uint32_t word = __ballot_sync(kFull, z[k] >= 0.f);
        if (lane == k) mine = word;
    }
    if (wr && lane < RG)
        reinterpret_cast<uint32_t*>(blk + kBlockT * code_bytes(D) + (t & 63) * sign_bytes(D))[rg0 + lane] = mine;
    constexpr int W = 3 * D / 32;
    if (wr && blockIdx.y == 0 && lane < W)
        reinterpret_cast<uint32_t*>(blk + (t & 63) * code_bytes(D))[lane] = code_word<D>(scode[warp], lane);
    pdl_wait();
}

template <int D, bool IS_K, int DT, int TV>
cudaError_t launch_enc_tv(const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    using SM = EncSmem<D, IS_K, TV>;
    auto kern = tq_encode_kernel<D, IS_K, DT, TV>;
    cudaError_t e = set_smem_once<tq_encode_kernel<D, IS_K, DT, TV>>((int)SM::total);
    if (e != cudaSuccess) return e;
    const int64_t N = a.B * a.Hkv * a.Tnew;
    const int64_t ntiles = (N + TV - 1) / TV;
    // K kernels stage S once per CTA, so they run persistent (two CTAs per SM);
    // V kernels are small and take as many CTAs as fit.
    const int64_t cap = (int64_t)num_sms * (IS_K ? 2 : 8);
    const int grid = (int)(ntiles < cap ? ntiles : cap);
    if (grid <= 0) return cudaSuccess;
    if (pdl) return launch_pdl(kern, dim3(grid), dim3(kThreads), SM::total, s, a);
    kern<<<grid, kThreads, SM::total, s>>>(a);
    return cudaGetLastError();
}

template <int D, bool IS_K, int DT>
cudaError_t launch_enc_t(const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    const int64_t N = a.B * a.Hkv * a.Tnew;
    if constexpr (IS_K) {
        if (N <= (int64_t)4 * num_sms) {        // appends: one warp per vector
            const dim3 grid((unsigned)((N + kSmallWarps - 1) / kSmallWarps), D / 32 / kSmallRowGroups);
            const size_t smem = (size_t)D * kSmallRowGroups * 32 * sizeof(float);
            auto kern = tq_encode_k_small_kernel<D, DT>;
            cudaError_t e = set_smem_once<tq_encode_k_small_kernel<D, DT>>((int)smem);
            if (e != cudaSuccess) return e;
            if (pdl) return launch_pdl(kern, grid, dim3(kSmallWarps * 32), smem, s, a);
            kern<<<grid, kSmallWarps * 32, smem, s>>>(a);
            return cudaGetLastError();
        }
    }
    if (N < (int64_t)32 * num_sms) return launch_enc_tv<D, IS_K, DT, 8>(a, num_sms, pdl, s);
    return launch_enc_tv<D, IS_K, DT, 32>(a, num_sms, pdl, s);
}

template <int D, bool IS_K>
cudaError_t launch_enc_dt(tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    switch (dt) {
        case TQ_F32: return launch_enc_t<D, IS_K, TQ_F32>(a, num_sms, pdl, s);
        case TQ_BF16: return launch_enc_t<D, IS_K, TQ_BF16>(a, num_sms, pdl, s);
        case TQ_F16: return launch_enc_t<D, IS_K, TQ_F16>(a, num_sms, pdl, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_encode(int d, bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s) {
    if (d == 128) {
        const cudaError_t e = launch_encode128_rot(is_k, dt, a, num_sms, pdl, s);
        return e == cudaErrorNotSupported ? launch_encode128(is_k, dt, a, num_sms, pdl, s) : e;
    }
    if (d == 64) {
        const cudaError_t e = launch_encode64_rot(is_k, dt, a, num_sms, pdl, s);
        if (e != cudaErrorNotSupported) return e;
        return is_k ? launch_enc_dt<64, true>(dt, a, num_sms, pdl, s) : launch_enc_dt<64, false>(dt, a, num_sms, pdl, s);
    }
    if (d == 256)
        return is_k ? launch_enc_dt<256, true>(dt, a, num_sms, pdl, s) : launch_enc_dt<256, false>(dt, a, num_sms, pdl, s);
    return cudaErrorInvalidValue;
}

}  // namespace tqi
