/*
 * tq.h -- C ABI of libtq: TurboQuant KV-cache compression and decode attention
 * over the compressed cache, for NVIDIA B200 (sm_100a).
 *
 * The method (page "Apple Silicon向けSwiftLM、TurboQuant KVキャッシュ圧縮とSSD
 * Expert Streamingを実装", ai-heartland.com):
 *   K cache, section "K-Cache圧縮：3-bit PolarQuant + 1-bit QJL = 4.25 bits/dim":
 *     1. L2-norm extraction and normalisation, x_hat = x / ||x||;
 *     2. a fast Walsh-Hadamard rotation that spreads outliers (applied here
 *        after a fixed random sign diagonal D: y = H D x_hat);
 *     3. a 3-bit non-linear Lloyd-Max codebook per coordinate;
 *     4. the residual of step 3;
 *     5. a Johnson-Lindenstrauss (QJL) projection of the residual, keeping one
 *        sign bit per projection.
 *   V cache, section "V-Cache圧縮：3-bit PolarQuant = 3.125 bits/dim":
 *     steps 1-3 only; V is not used for scoring, so it carries no QJL bit.
 *   Attention, section on the hybrid V2+V3 design: dequantisation is fused
 *     into the attention kernel, which reads the packed cache directly.
 *
 * Conventions.  d = head_dim (64, 128 or 256); m = d JL rows; tokens per cache
 * block = 64.  All data buffers (inputs, caches, outputs, workspace) are
 * device memory owned by the caller; the library owns only the constants
 * created by tq_init.  Hot calls (encode, attend) allocate nothing, do not
 * synchronise and copy nothing to the host; they enqueue kernels on the
 * caller's stream and return.  Errors in the arguments are detected on the
 * host before anything is launched and leave all buffers untouched.
 * Asynchronous device faults surface at the caller's next synchronisation.
 * A handle is read-only after tq_init, so concurrent calls on different
 * streams are safe; calls whose outputs overlap race.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifndef TQ_API
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_handle tq_handle;

/* Status codes.  TQ_ERR_CUDA: a CUDA runtime call or a launch failed.
 * TQ_ERR_WORKSPACE: the workspace passed is smaller than required.
 * TQ_ERR_DEVICE_CHECK: a kernel recorded a failed device-side check (a bounded
 * wait that ran out); reported by tq_device_status. */
typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,
    TQ_ERR_UNSUPPORTED = 2,
    TQ_ERR_CUDA = 3,
    TQ_ERR_WORKSPACE = 4,
    TQ_ERR_DEVICE_CHECK = 5
} tq_status;

/* Element type of K/V inputs and of queries. */
typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* A compressed cache: caller-owned device buffer of tq_cache_bytes() bytes,
 * 16-byte aligned, laid out as [B][Hkv][Tcap/64] blocks (Tcap a multiple of 64).
 * Paged form (block_table != NULL): base is a pool of pool_blocks blocks of
 * tq_block_bytes(d, is_k) bytes, and block_table (device int32
 * [B*Hkv][Tcap/64], row b*Hkv + h) gives the pool block that holds tokens
 * [64 lb, 64 lb + 64) of (batch b, kv head h).  Blocks of different sequences
 * may be anywhere in the pool; a block must not be shared by two live
 * (sequence, logical block) pairs that are written.  A table entry outside
 * [0, pool_blocks) is a device-side check failure (reported by
 * tq_device_status): nothing is written through it and reads go to block 0.
 * With block_table == NULL pool_blocks is ignored.
 * K block (64 tokens): codes 64 x 3d/8 B | signs 64 x d/8 B | ||k|| fp16 x 64 |
 *                      gamma = ||residual|| fp16 x 64
 * V block (64 tokens): codes 64 x 3d/8 B | ||v|| fp16 x 64
 * Per token the 3-bit codes are 3d/32 little-endian uint32 words.  Slice s
 * (128 coordinates) and slot t (0..3) own words 12s+3t+{0,1,2} (Wa, Wb, Wc)
 * holding slot codes i = 0..31, where slot code i is coordinate
 *     j = 128 s + 16 (i >> 2) + 2 t + (i & 1) + 8 ((i >> 1) & 1).
 * Nibble k of Wa: bits 0-2 = code(i = k), bit 3 = bit 0 of code(24 + k);
 * Wb: code(8 + k) and bit 1 of code(24 + k); Wc: code(16 + k) and bit 2 of
 * code(24 + k).  Signs are d/32 words per token; word 4s+t holds the sign of
 * JL row i = 2q at bit q and of row 2q+1 at bit 16+q (q = 0..15), rows mapped
 * to indices exactly as coordinates above.  d = 64 is one slice of 16 codes
 * per slot (i = 0..15, s = 0): word t (t = 0..3) holds code(k) in bits 0-2 of
 * nibble k (k = 0..7); halfword t of bytes 16..23 holds code(8 + k) in bits
 * 0-2 of nibble k (k = 0..3); bits 0, 1, 2 of code(12 + k) are bit 3 of
 * nibble k of word t, of nibble 4 + k of word t and of nibble k of halfword t.
 * Its signs are 4 halfwords per token: bit i of halfword t is the sign of the
 * JL row of slot position i.  A sign bit is 1 when the projection is >= 0.  Storage: (3d + m + 32)/d bits/dim for K (4.25 at
 * d = 128) and (3d + 16)/d for V (3.125 at d = 128). */
typedef struct {
    void* base;
    int64_t B;
    int64_t Hkv;
    int64_t Tcap;
    const int32_t* block_table;   /* NULL: contiguous cache */
    int64_t pool_blocks;
} tq_cache;

/* ---- constants -------------------------------------------------------- */

/* Compute the method's constants on the host, with no device involved:
 * D (d signs, +-1), S (m x d fp32, row-major, iid N(0,1)), the 8 codebook
 * centroids (ascending) and the 7 decision boundaries (midpoints).
 * Readings: counter-based SplitMix64 stream `seed`; D_j = -1 iff the top bit of
 * draw j is set; S from Box-Muller on draws d+2p, d+2p+1 (cosine output to
 * element 2p, sine output to 2p+1), rounded to fp32; centroids = the 8-level
 * Lloyd-Max quantiser of N(0,1) (K flow step 3), scaled by 1/sqrt(d), rounded
 * to fp16.  Any output pointer may be NULL.  Errors: INVALID_ARG (d not 64, 128
 * or 256). */
TQ_API tq_status tq_params_host(int head_dim, uint64_t seed, int8_t* D, float* S, float* centroids8,
                         float* bounds7);

/* Create a handle on the current CUDA device: computes the constants as
 * tq_params_host does and uploads them (the only allocating call).
 * Errors: INVALID_ARG (bad d or NULL out), CUDA. */
TQ_API tq_status tq_init(int head_dim, uint64_t seed, tq_handle** out);

/* Free the handle's device constants.  NULL is accepted. */
TQ_API tq_status tq_destroy(tq_handle* h);

/* Copy the handle's constants to host arrays (any may be NULL); synchronous. */
TQ_API tq_status tq_get_params(const tq_handle* h, int8_t* D, float* S, float* centroids8,
                        float* bounds7);

TQ_API int tq_head_dim(const tq_handle* h);

/* ---- sizes ------------------------------------------------------------ */

/* Bytes of one 64-token block; 0 for an unsupported d. */
TQ_API size_t tq_block_bytes(int head_dim, int is_k);

/* Bytes of a cache [B][Hkv][Tcap/64 blocks]; 0 if Tcap is not a positive
 * multiple of 64 or d is unsupported. */
TQ_API size_t tq_cache_bytes(int head_dim, int is_k, int64_t B, int64_t Hkv, int64_t Tcap);

/* ---- encode (K flow steps 1-5 / V steps 1-3) --------------------------- */

/* Encode Tnew new vectors per (batch, kv head) into token positions
 * [t0, t0 + Tnew) of the cache.  x is a device tensor of `dtype` with element
 * strides (sb, sh, st) for (batch, head, token) and a contiguous last
 * dimension of d elements: vector (b, h, t) starts at x + b*sb + h*sh + t*st.
 * Each vector is normalised (n = ||x||, stored as fp16), rotated, quantised
 * to 3-bit codes against the boundaries (a coordinate equal to a boundary
 * takes the upper cell), and for K the residual's norm gamma (fp16) and the
 * sign bits of S * residual are stored.  A zero vector stores code 4, gamma 0,
 * all signs 1.  Tokens outside [t0, t0+Tnew) are not touched.
 * Stream order holds as for any launch.  A bulk encode of 16-bit input (at
 * d = 64 and 128, at least 16384 contiguous vectors) starts its set-up while
 * the previous kernel on the stream finishes, and it waits for that kernel
 * before it reads x or writes the cache.
 * Errors: INVALID_ARG (NULL pointers, B/Hkv mismatch with the cache, Tnew < 0,
 * t0 < 0, t0 + Tnew > Tcap, misaligned x or cache), CUDA. */
TQ_API tq_status tq_encode_k(const tq_handle* h, const void* x, tq_dtype dtype, int64_t B, int64_t Hkv,
                      int64_t Tnew, int64_t sb, int64_t sh, int64_t st, const tq_cache* kc,
                      int64_t t0, void* stream);
TQ_API tq_status tq_encode_v(const tq_handle* h, const void* x, tq_dtype dtype, int64_t B, int64_t Hkv,
                      int64_t Tnew, int64_t sb, int64_t sh, int64_t st, const tq_cache* vc,
                      int64_t t0, void* stream);

/* ---- decode attention --------------------------------------------------- */

/* Workspace bytes tq_attend_decode needs for these sizes on this handle's
 * device (query rotation, per-split softmax partials).  0 on bad arguments. */
TQ_API size_t tq_attend_workspace_bytes(const tq_handle* h, int64_t B, int64_t Hq, int64_t Hkv,
                                 int64_t Tmax);

/* Decode attention over the compressed cache: the page's hybrid V2+V3 section
 * (dequantisation fused into the attention kernel, which reads the packed
 * cache directly), with scores from its K section (3-bit codes plus the 1-bit
 * QJL residual correction) and values from its V section.
 * One decode step of attention for B x Hq queries (q [B][Hq][d] contiguous,
 * `qdtype`) over the compressed caches kc (K) and vc (V).  Query head h uses
 * kv head h / (Hq/Hkv).  Sequence b attends over tokens [0, seq_lens[b]) when
 * seq_lens (device int32[B]) is not NULL, else over [0, T).  Computes, per
 * query head, q' = H D q, u = S q' and
 *   s_t = scale * n_t * (<q', c[idx_t]> + gamma_t * sqrt(pi/2)/m * <u, 2 sigma_t - 1>),
 *   out = D H sum_t softmax(s)_t * nv_t * c[idxv_t],
 * with n_t, gamma_t, nv_t the stored fp16 values, in fp32 with split-K
 * (flash-decoding) partials in `ws` merged by a final kernel.  out is fp32
 * [B][Hq][d]; an empty sequence gives zeros.  Supported: d in {64, 128, 256},
 * any Hq/Hkv (kv heads with more than 8 query heads are served in groups of
 * up to 8), B <= 65535, Hkv * ceil(Hq/Hkv / 8) <= 65535, B * Hq < 2^31.  ws must be 256-byte
 * aligned with at least
 * tq_attend_workspace_bytes(h, B, Hq, Hkv, T or max seq_len) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
TQ_API tq_status tq_attend_decode(const tq_handle* h, const void* q, tq_dtype qdtype, int64_t B,
                           int64_t Hq, const tq_cache* kc, const tq_cache* vc,
                           const int32_t* seq_lens, int64_t T, float scale, float* out, void* ws,
                           size_t ws_bytes, void* stream);

/* ---- PolarQuant-only K (no QJL bit) --------------------------------------- */

/* Attention over a PolarQuant-only K cache: K stored like V, with 3-bit codes
 * and the fp16 norm but no QJL sign bits and no gamma (3.125 bits/dim at
 * d = 128 instead of 4.25).  Encode such a K cache with tq_encode_v into a
 * V-layout buffer (tq_cache_bytes(d, 0, ...)).  Scores drop the QJL term:
 *   s_t = scale * n_t * <q', c[idx_t]>,
 * the rest as tq_attend_decode (same arguments, workspace and errors).  The
 * page weighs the two K flows against each other: its K section adds the
 * 1-bit QJL residual to correct the inner-product bias of the 3-bit codes,
 * and its hybrid V2+V3 section trades that accuracy against the faster
 * PolarQuant-only path. */
TQ_API tq_status tq_attend_decode_polar(const tq_handle* h, const void* q, tq_dtype qdtype, int64_t B,
                                        int64_t Hq, const tq_cache* kc, const tq_cache* vc,
                                        const int32_t* seq_lens, int64_t T, float scale, float* out, void* ws,
                                        size_t ws_bytes, void* stream);

/* ---- chunked prefill ------------------------------------------------------ */

/* Workspace bytes tq_attend_prefill needs (rotated queries and the softmax
 * partials of B * Lq * Hq query rows; at head_dim 128 a row tile's tokens may
 * be spread over several CTAs, each writing one partial, up to a bound that
 * depends on the row count and the device's SM count).  0 on bad arguments. */
TQ_API size_t tq_prefill_workspace_bytes(const tq_handle* h, int64_t B, int64_t Lq, int64_t Hq);

/* Attention for a chunk of Lq new queries per sequence (q [B][Lq][Hq][d]
 * contiguous, `qdtype`) over the compressed caches, causal: query i of the
 * chunk attends over tokens [0, T0 + i] of its sequence, so the chunk's own K
 * and V must already be encoded at positions T0 .. T0 + Lq - 1.  Scores and
 * output as tq_attend_decode (the same estimator, in the page's K section and
 * hybrid V2+V3 section); out is fp32 [B][Lq][Hq][d].  With many queries per
 * kv head the score and value contractions are dense and run on tensor cores:
 * at d = 128 on tcgen05 with each 64-token block dequantised once per 128
 * query rows (q' and u' as fp16 hi and lo limbs), the row tiles' token ranges
 * spread evenly over one CTA per SM; at d = 64 and 256 on mma.sync tiles with
 * the keys dequantised once per 16 query rows and the QJL term on 16-bit
 * fixed-point u' (at d = 256 two CTAs share each 64 query rows, each
 * accumulating half of the value coordinates).  Supported: d in {64, 128,
 * 256}, any Hq/Hkv, B <= 65535, Lq Hq / Hkv <= 2^27, T0 + Lq <= Tcap;
 * contiguous or paged caches.  Errors: INVALID_ARG, UNSUPPORTED (grid or size
 * limits), WORKSPACE, CUDA. */
TQ_API tq_status tq_attend_prefill(const tq_handle* h, const void* q, tq_dtype qdtype, int64_t B, int64_t Lq,
                                   int64_t Hq, const tq_cache* kc, const tq_cache* vc, int64_t T0, float scale,
                                   float* out, void* ws, size_t ws_bytes, void* stream);

/* ---- fused append-and-attend step ---------------------------------------- */

/* One decode step of a serving loop: encode Tnew new K and V vectors per
 * (batch, kv head) into token positions [t0, t0 + Tnew) of kc and vc, then
 * attend for B x Hq queries over tokens [0, t0 + Tnew) of every sequence.
 * The page's decode loop appends each generated token's K/V to the
 * compressed cache and attends over it (page "Apple Silicon向けSwiftLM ...",
 * K/V sections and the hybrid V2+V3 section); this call does both in one
 * launch chain.  Results (cache bytes and out) are identical to
 * tq_encode_k + tq_encode_v + tq_attend_decode with T = t0 + Tnew.
 * k_new and v_new share `kv_dtype` and the element strides (sb, sh, st) as in
 * tq_encode_k; B and Hkv are the caches'.  q, out, ws and scale as in
 * tq_attend_decode (ws sized by tq_attend_workspace_bytes(h, B, Hq, Hkv,
 * t0 + Tnew)).  The kernels are chained with programmatic dependent launch:
 * the query prologue runs alongside the encodes and the attention kernel
 * sets up while they run, reading the cache only after they complete; every
 * kernel completes only after the one before it, so the next work on the
 * stream sees the finished step.
 * Errors: those of tq_encode_k and tq_attend_decode (checked before any
 * launch). */
TQ_API tq_status tq_append_attend(const tq_handle* h, const void* k_new, const void* v_new, tq_dtype kv_dtype,
                                  int64_t Tnew, int64_t sb, int64_t sh, int64_t st, const tq_cache* kc,
                                  const tq_cache* vc, int64_t t0, const void* q, tq_dtype q_dtype, int64_t Hq,
                                  float scale, float* out, void* ws, size_t ws_bytes, void* stream);

/* ---- decode attention without device allocation ------------------------- */

/* Size of the scratch array inside the library used by tq_attend_decode_static. */
#define TQ_STATIC_SCRATCH_BYTES (8u << 20)

/* The method's pages have no counterpart to this call; it exists for callers.
 * Same computation, arguments and results as tq_attend_decode, but with no
 * workspace argument: the scratch (rotated queries, split-K partials) is a
 * fixed TQ_STATIC_SCRATCH_BYTES (8 MiB) array inside the library, which every
 * GPU that loads the library keeps until the process exits.  It is for callers
 * that cannot allocate device memory when they run a decode step: a plugin or
 * custom operator handed only input and output pointers by a host framework
 * that owns the allocator, a serving loop that fixes its memory budget at
 * start-up and must not grow it or pay an allocation's implicit
 * synchronisation per token, or a deployment that forbids dynamic device
 * allocation after initialisation.  Nothing here calls cudaMalloc or cudaFree.
 * The first call on each device resolves the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  Sizes that need more scratch than
 * the array holds (tq_attend_workspace_bytes(...) above 8 MiB) are rejected
 * with TQ_ERR_WORKSPACE before anything is launched.  All calls on a device
 * share the one array and it keeps the last call's contents (every byte a call
 * reads is written by that call first, so nothing needs clearing); calls that
 * overlap on the GPU -- on different streams, or from different threads --
 * race on it and must be serialised by the caller.
 * Errors: those of tq_attend_decode; CUDA if the address cannot be resolved. */
TQ_API tq_status tq_attend_decode_static(const tq_handle* h, const void* q, tq_dtype qdtype, int64_t B,
                                         int64_t Hq, const tq_cache* kc, const tq_cache* vc,
                                         const int32_t* seq_lens, int64_t T, float scale, float* out,
                                         void* stream);

/* ---- diagnostics -------------------------------------------------------- */

/* Synchronise `stream`, then report and clear the handle's device check word:
 * TQ_ERR_DEVICE_CHECK if a kernel gave up a bounded wait since the last call. */
TQ_API tq_status tq_device_status(const tq_handle* h, void* stream);

/* Diagnostics: when ev_start/ev_stop (cudaEvent_t, created by the caller) are
 * not NULL, each later tq_attend_decode records ev_start just before its
 * split-K attention kernel and ev_stop just after it, on the call's stream, so
 * the caller can time that kernel alone.  Pass NULLs to stop.  Not thread-safe
 * with concurrent tq_attend_decode calls on the same handle. */
TQ_API tq_status tq_set_decode_events(tq_handle* h, void* ev_start, void* ev_stop);

/* Diagnostics: the number of times each warp of the split-K attention kernel
 * polls the mbarrier of its first staged chunk before giving up (every wait in
 * the kernels is bounded; normally 2^20 polls).  A give-up sets the handle's
 * check word, waits with the full bound for the warp's copies still in flight,
 * and leaves that warp's tokens out of the result (the outputs of such a call
 * are not the attention; tq_device_status reports TQ_ERR_DEVICE_CHECK).  0
 * makes every first wait give up at once, which lets a test exercise this path
 * without a fault; a negative value restores the full bound.  Not thread-safe
 * with concurrent calls on the same handle.  Errors: INVALID_ARG (NULL h). */
TQ_API tq_status tq_set_wait_limit(tq_handle* h, int first_wait);

/* Diagnostics: choose the decode kernel of later tq_attend_decode calls on this
 * handle: 0 = automatic (tensor-core kernel where supported, with the work
 * partition its cost model prefers), 1 = the SIMT kernel, 2 = the tensor-core
 * kernel on the uniform split grid only, 3 = the tensor-core kernel on the
 * stream-K grid wherever that fits (sequences of one length, no more
 * (batch, kv head, head group) units than CTA slots, partial slots within the
 * workspace bound).  Paths 0, 2 and 3 give the same outputs up to the fp32
 * order of the softmax merge.  Changes the workspace size
 * tq_attend_workspace_bytes reports (path 1).  Errors: INVALID_ARG (NULL h,
 * path outside 0..3). */
TQ_API tq_status tq_set_decode_path(tq_handle* h, int path);

/* Diagnostics, host only (no device or handle needed): the work partition the
 * tensor-core decode takes for a call of these sizes (head_dim, B sequences,
 * Hq / Hkv heads, T tokens) on a GPU with num_sms SMs, automatic path.
 * equal_len != 0: every sequence has T tokens (a call without seq_lens; only
 * then is the stream-K grid considered), else T is the cache capacity.
 * Outputs: *nsplit partial slots per query head; *split_tokens tokens per
 * split of the uniform grid; *streamk_ctas the CTAs of the stream-K grid (0:
 * the uniform grid is used) and *streamk_chunks the chunks of one (batch, kv
 * head, query-head group) unit that it divides; *chunk_tokens tokens per chunk.
 * Errors: INVALID_ARG (head_dim not 64/128/256, sizes as tq_attend_decode
 * rejects them, num_sms < 1, a NULL output). */
TQ_API tq_status tq_decode_plan(int num_sms, int head_dim, int64_t B, int64_t Hq, int64_t Hkv, int64_t T,
                                int equal_len, int* nsplit, int64_t* split_tokens, int64_t* streamk_ctas,
                                int64_t* streamk_chunks, int* chunk_tokens);

/* Name of the kernel path tq_attend_decode uses for these sizes on this handle
 * ("mma" or "simt"); static string. */
TQ_API const char* tq_attend_path(const tq_handle* h, int64_t Hq, int64_t Hkv);

TQ_API const char* tq_status_string(tq_status s);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
