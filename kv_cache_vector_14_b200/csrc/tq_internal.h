// Internal declarations shared by the libtq translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <vector>

#define TQ_API __attribute__((visibility("default")))
#include "tq.h"

namespace tqi {

constexpr int kBlockT = 64;      // tokens per cache block
constexpr int kMaxSplits = 2048; // split-K partials per query head (combine keeps their weights in smem)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kDefaultWaitLimit = 1 << 20;   // poll count of a bounded mbarrier wait
constexpr uint64_t kWaitNs = 1000000000ull;   // and its time bound (1 s)

#ifdef __CUDACC__
// global nanosecond timer of the GPU
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// 16-byte copy global -> shared that does not pass through registers
// (cp.async, cache-global); many of them are in flight at once and one
// cp_async_wait_all() waits for all of this thread's.  Both addresses 16-byte
// aligned.
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst_smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
#endif

// Codebook passed by value to every kernel (it lands in the constant bank).
struct Codebook {
    float c[8];         // centroids, ascending (fp16-exact values)
    float b[7];         // decision boundaries (midpoints)
    uint32_t lut_lo[2]; // low bytes of the fp16 bit patterns of c[0..7]
    uint32_t lut_hi[2]; // high bytes of the fp16 bit patterns of c[0..7]
    uint32_t pow2[32];  // 1 << k: shifts done as integer multiplies (FMA pipe, not ALU)
    // The centroids as exact integers c 2^14 = 256 hi + lo (signed byte limbs),
    // when every one is an integer of at most 15 bits (int8 key operands):
    // byte k of lut8_lo / lut8_hi is the lo / hi limb of c[k].
    uint32_t lut8_lo[2];
    uint32_t lut8_hi[2];
    int k8;             // 1: the limbs above are exact
};

// Host-side generation of the constants (tq_params.cpp).
bool make_params(int d, uint64_t seed, int8_t* D, float* S, float* c8, float* b7);
uint16_t double_to_half_bits(double x);
double half_bits_to_double(uint16_t h);

// Byte sizes of the block fields.
__host__ __device__ inline int64_t code_bytes(int d) { return 3LL * d / 8; }          // per token
__host__ __device__ inline int64_t sign_bytes(int d) { return (int64_t)d / 8; }       // per token
__host__ __device__ inline int64_t block_bytes(int d, bool is_k) {
    return kBlockT * code_bytes(d) + (is_k ? kBlockT * sign_bytes(d) + 4 * kBlockT : 2 * kBlockT);
}

// Slot order of coordinate j inside a token record: slot t (0..3) of slice
// j >> 7 owns 32 coordinates (16 at d = 64, one slice); position i inside the
// slot.
__host__ __device__ inline int slot_of(int j) { return (j >> 1) & 3; }
__host__ __device__ inline int slot_pos(int j) {
    int jj = j & 127;
    return ((jj >> 4) << 2) | (((jj >> 3) & 1) << 1) | (jj & 1);
}
__host__ __device__ inline int slot_coord(int s, int t, int i) {
    return 128 * s + 16 * (i >> 2) + 2 * t + (i & 1) + 8 * ((i >> 1) & 1);
}

// Tensor-core K encode (d = 128): operands of 128 rows x 128 fp16 columns in
// the 128-byte-swizzled K-major shared-memory layout (8-row groups of 1024
// bytes; 16-byte chunk c of row r stored at chunk c ^ (r & 7); columns 64..127
// in a second 16 KB half).
constexpr int kTcRows = 128;
__host__ __device__ inline uint32_t sw128_k_offset(int row, int k) {
    return (uint32_t)((k >> 6) * (kTcRows * 128) + (row >> 3) * 1024 + (row & 7) * 128 +
                      ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}
// JL row whose projection lands in column n of the product: bit n % 32 of
// stored sign word n / 32 (d = 128: word t = slot t, bit q -> position 2q,
// bit 16 + q -> position 2q + 1).
__host__ __device__ inline int qjl_row_of_column(int n) {
    const int b = n & 31;
    return slot_coord(0, n >> 5, b < 16 ? 2 * b : 2 * (b - 16) + 1);
}
// JL row whose sign is bit l of stored sign word r.  d >= 128: word 4s+t is
// slot t of slice s, bit q -> position 2q, bit 16+q -> position 2q+1.  d = 64:
// word r holds the 16-bit sign halfwords of slots 2r (bits 0-15) and 2r+1,
// bit i of a halfword -> position i.
__host__ __device__ inline int sign_row(int d, int r, int l) {
    if (d == 64) return slot_coord(0, 2 * r + (l >> 4), l & 15);
    return slot_coord(r >> 2, r & 3, l < 16 ? 2 * l : 2 * (l - 16) + 1);
}
__host__ __device__ inline bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }

// Division by a fixed divisor d >= 1 for dividends below 2^31:
// q = umulhi(n, m) >> s with m = ceil(2^(31 + ceil(log2 d)) / d); m = 0 marks d = 1.
struct FastDiv {
    uint32_t m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
    if (d <= 1) return {0u, 0u};
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    const uint64_t p = 31 + l;
    return {(uint32_t)(((1ull << p) + d - 1) / d), (uint32_t)(p - 32)};
}
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fdiv(uint32_t n, FastDiv f) { return f.m ? (__umulhi(n, f.m) >> f.s) : n; }
#endif

struct EncArgs {
    const void* x;
    int64_t sb, sh, st;
    int64_t B, Hkv, Tnew, t0;
    int64_t NB;               // blocks per sequence (Tcap / 64)
    uint8_t* cache;
    const int32_t* table;     // paged cache: [B*Hkv][NB] pool blocks, or null
    int64_t pool;             // pool blocks of a paged cache
    const float* dsign;       // [d] +-1
    const float* sthr;        // [d][d/32][32] JL matrix, encode lane order
    const uint8_t* bimg;      // JL matrix as tensor-core operand (hi, lo fp16 limbs; d = 128: K index =
                              // coordinate; d = 64: K index in slot order), rows in sign-word order
    int* err;                 // device check word
    int vec16;                // every input row starts on a 16-byte boundary
    int wait_x;               // launched as a programmatic dependent of a kernel that may write the
                              // input or the cache: wait for it (griddepcontrol.wait) before the first
                              // input load (tensor-core encodes)
    uint32_t dneg[4];         // bit i of word i / 32: d_i < 0 (head_dim up to 128)
    FastDiv fdT, fdH;         // division by Tnew and by Hkv (vector counts below 2^31)
    Codebook cb;
};

struct DecArgs {
    const float* qp;          // [B*Hq][d] rotated queries q' = H D q
    const float* up;          // [B*Hq][d] sqrt(pi/2)/m * S q'
    const uint8_t* kc;
    const uint8_t* vc;
    const int32_t* ktable;    // paged caches: block tables, or null
    const int32_t* vtable;
    int64_t kpool, vpool;
    int64_t NB;               // blocks per sequence
    const int32_t* seq_lens;  // device or null
    int64_t T;                // used when seq_lens is null
    int64_t Tcap;
    int64_t B, Hq, Hkv;
    int nsplit;               // partial slots per query head
    int64_t split_tokens;     // tokens per split, multiple of 64 (uniform split grid)
    // Stream-K grid (sk_ctas > 0; equal-length sequences only): the units
    // (batch, kv head, query-head group) laid end to end, sk_nck chunks each
    // (sk_total in all), and CTA c takes chunks [c sk_total / sk_ctas,
    // (c + 1) sk_total / sk_ctas), at most two units' worth.
    int sk_ctas;
    int64_t sk_nck, sk_total;
    float scale_log2;         // softmax scale * log2(e)
    float* part_ml;           // [B*Hq][nsplit][2] (running max in log2 units, sum)
    float* part_acc;          // [B*Hq][nsplit][d] rotated-domain accumulators
    int* err;                 // device check word
    int64_t fresh_lo, fresh_hi;   // tokens written by a chained encode: read only after pdl_wait
    int first_wait;           // try count of each warp's first ring wait (diagnostics; normally the full bound)
    Codebook cb;
};

#ifdef __CUDACC__
// Block index of logical block lb of sequence bh (= b * Hkv + h): bh * NB + lb
// for a contiguous cache, the block table's entry for a paged one.  An entry
// outside the pool sets the check word and gives -1.
__device__ __forceinline__ int64_t cache_block(const int32_t* table, int64_t pool, int64_t NB, int64_t bh,
                                               int64_t lb, int* err) {
    if (!table) return bh * NB + lb;
    const int32_t p = __ldg(table + bh * NB + lb);
    if (p < 0 || (int64_t)p >= pool) {
        atomicExch(err, 1);
        return -1;
    }
    return p;
}

// Input offset (elements) and cache block of vector gv (b, h, token order) of an
// encode; blk is null when a paged cache's table entry lies outside its pool.
__device__ __forceinline__ void encode_locate(const EncArgs& a, uint32_t gv, int64_t bb, int64_t& xoff, uint8_t*& blk,
                                              int& tau) {
    const uint32_t bh = fdiv(gv, a.fdT);
    const uint32_t tt = gv - bh * (uint32_t)a.Tnew;
    const uint32_t b = fdiv(bh, a.fdH);
    const uint32_t hh = bh - b * (uint32_t)a.Hkv;
    xoff = (int64_t)b * a.sb + (int64_t)hh * a.sh + (int64_t)tt * a.st;
    const int64_t t = a.t0 + tt;
    tau = (int)(t & 63);
    const int64_t pb = cache_block(a.table, a.pool, a.NB, bh, t >> 6, a.err);
    blk = pb >= 0 ? a.cache + pb * bb : nullptr;                   // null: nothing is written
}
#endif

// Programmatic dependent launch: a kernel launched with launch_pdl may start
// while the previous kernel on the stream is still running; it must execute
// pdl_wait() before reading anything that kernel writes.  pdl_trigger() lets
// the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Raise a kernel's dynamic shared-memory limit once per device and process,
// so repeated launches (and launches under stream capture) make no attribute
// calls.
template <auto Kern>
cudaError_t set_smem_once(int bytes) {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // the largest carveout too, as set_carveout_once below gives the step's other kernels
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Ask once per device and process for the largest shared-memory carveout.  The
// kernels of one decode step (appends, prologue, split-K, combine) then find the
// SMs configured alike, so a programmatic dependent's CTAs start without an SM
// being reconfigured, and a kernel with little shared memory fits as many CTAs
// per SM as its registers allow.
template <auto Kern>
cudaError_t set_carveout_once() {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Kernel launchers (tq_encode.cu, tq_decode.cu); return a CUDA error code.
cudaError_t launch_encode(int d, bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl,
                          cudaStream_t s);
cudaError_t launch_encode128(bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s);
// Bulk d = 128 encode of contiguous bf16 / fp16 input with the rotation on the
// tensor cores; cudaErrorNotSupported when the call does not qualify.
cudaError_t launch_encode128_rot(bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s);
cudaError_t launch_encode64_rot(bool is_k, tq_dtype dt, const EncArgs& a, int num_sms, bool pdl, cudaStream_t s);
// pdl: launched as a programmatic dependent of the previous kernel (fused
// append-and-attend step); the kernels then complete only after it.
cudaError_t launch_prologue(int d, const void* q, tq_dtype dt, int64_t BHq, const float* dsign,
                            const float* st, float* qp, float* up, bool pdl, cudaStream_t s);
// Chunked prefill (head_dim 128): rows (b, i, head) of Lq queries per sequence,
// query i over tokens [0, T0 + i]; partials as one split of a.part_ml/part_acc.
cudaError_t launch_prefill(int d, int G, const DecArgs& a, int64_t Lq, int64_t T0, cudaStream_t s);
// head_dim 128: the tcgen05 form (tq_prefill_tc.cu)
// d = 128 chunked prefill on tcgen05, one CTA per SM over the flattened tiles; the
// partials go to nsplit slots per row (*nsplit_out, at most split_cap).
int prefill_tc_split_cap(int num_sms, int64_t rows);
cudaError_t launch_prefill_tc(int G, const DecArgs& a, int64_t Lq, int64_t T0, int num_sms, int split_cap,
                              int* nsplit_out, cudaStream_t s);
// qjl = false: PolarQuant-only K cache (V layout), scores without the QJL term.
cudaError_t launch_decode(int d, int G, bool use_mma, bool qjl, const DecArgs& a, cudaStream_t s);
cudaError_t launch_combine(int d, int64_t BHq, int nsplit, const float* part_ml,
                           const float* part_acc, const float* dsign, float* out, cudaStream_t s);
bool mma_supported(int d, int G);
int decode_ctas_per_sm(bool use_mma);
int decode_chunk_tokens(int d, bool use_mma);   // split ranges are multiples of this
int decode_warps(bool use_mma, int G);   // warps sharing one split
int decode_head_groups(bool use_mma, int G);   // CTAs per (split, kv head, batch)

}  // namespace tqi

struct tq_handle {
    int d = 0;
    uint64_t seed = 0;
    int device = -1;
    int num_sms = 0;
    std::vector<int8_t> hD;
    std::vector<float> hS;    // [m][d]
    float hc[8] = {};
    float hb[7] = {};
    float* dsign = nullptr;   // [d]
    float* dST = nullptr;     // [d][m] transposed S (query prologue)
    float* dSThr = nullptr;   // [d][d/32][32] encode lane order
    uint8_t* dSB = nullptr;   // d = 128: JL operand image for the tensor-core encode (64 KB)
    uint32_t dneg[8] = {};    // bit i of word i / 32: d_i < 0
    int* derr = nullptr;
    tqi::Codebook cb{};
    cudaEvent_t ev_start = nullptr;   // optional timing of the split-K kernel
    cudaEvent_t ev_stop = nullptr;
    int decode_path = 0;              // diagnostics: 0 auto, 1 SIMT, 2 tensor-core uniform splits, 3 tensor-core stream-K
    int first_wait = -1;              // diagnostics: try count of the decode's first ring wait (< 0: full bound)
};
