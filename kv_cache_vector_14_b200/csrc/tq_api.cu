// C ABI of libtq (declared in include/tq.h): argument validation, the handle
// with its device constants, and the launch sequences of encode and decode.
#include <cmath>
#include <cstring>
#include <new>

#include "tq_internal.h"

using namespace tqi;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t dtype_size(tq_dtype dt) { return dt == TQ_F32 ? 4 : 2; }
bool dtype_ok(int dt) { return dt == TQ_F32 || dt == TQ_BF16 || dt == TQ_F16; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split count for decode.  Work is `pairs` sequences of nchunk chunks; a CTA
// handles `per` consecutive chunks spread over its warps.  Its warps share one
// SM and interleave, so its time follows the SM's work, per / warps chunk-steps
// (at least one: a warp's own chunk is the shortest time), and the kernel's
// time is waves * that.  The
// count maximising ideal / actual time wins (ties: fewer partials).  The loop
// bound is also the workspace's upper bound (split_upper_bound).
int64_t split_loop_bound(int64_t cap, int64_t pairs, int64_t nchunk) {
    int64_t bound = 16 * cap / pairs + 1;
    if (bound > kMaxSplits) bound = kMaxSplits;
    return bound < nchunk ? bound : nchunk;
}

// A CTA also pays a fixed cost (constants, barrier set-up, the merge of its
// warps, the partial it writes), about kSetup chunk-steps per warp.
constexpr double kSetup = 2.0;
// chunk-steps of a CTA with `chunks` chunks over `warps` warps (see above)
double chunk_steps(int64_t chunks, int warps) {
    const double t = (double)chunks / warps;
    return t > 1.0 ? t : 1.0;
}

int choose_nsplit(int64_t cap, int warps, int64_t pairs, int64_t nchunk, double* steps = nullptr) {
    const int64_t hi = split_loop_bound(cap, pairs, nchunk);
    const double ideal = (double)pairs * nchunk / ((double)cap * warps);
    int64_t best = 1;
    double best_eff = -1.0;
    for (int64_t ns = 1; ns <= hi; ++ns) {
        const int64_t per = (nchunk + ns - 1) / ns;
        const int64_t used = (nchunk + per - 1) / per;
        if (used != ns) continue;
        const int64_t waves = (pairs * used + cap - 1) / cap;
        const double t = (double)waves * (chunk_steps(per, warps) + kSetup);
        const double eff = ideal / t;
        if (eff > best_eff + 1e-12) { best_eff = eff; best = ns; if (steps) *steps = t; }
    }
    return (int)best;
}

// Stream-K plan for sequences of one length: nC CTAs take equal shares of the
// units' chunks laid end to end (units x nck in all), and each warp a
// contiguous run of its CTA's share.  With nC >= units a share spans at most
// two units, so at most one warp per CTA crosses into the next unit (it pays
// a tenth of a chunk-step or so to switch).  Returns the modelled chunk-steps of the
// slowest CTA (plus the fixed cost) and the partial slots a unit needs (the
// CTAs that overlap it), or -1 when the shape does not fit.
double streamk_plan(int64_t cap, int warps, int64_t units, int64_t nck, int64_t* nC_out, int* slots_out) {
    const int64_t N = units * nck;
    const int64_t nC = cap < N ? cap : N;
    if (nC < units || nC <= 0) return -1.0;
    double worst = 0.0;
    for (int64_t c = 0; c < nC; ++c) {
        const int64_t lo = c * N / nC, hi = (c + 1) * N / nC;
        const int64_t u0 = lo / nck, u1 = (hi - 1) / nck;
        if (hi <= lo || u1 - u0 > 1) return -1.0;
        const double t = chunk_steps(hi - lo, warps) + (u1 != u0 ? 0.1 : 0.0);
        worst = t > worst ? t : worst;
    }
    int64_t slots = 0;
    for (int64_t u = 0; u < units; ++u) {
        const int64_t cf = ((u * nck + 1) * nC - 1) / N, cl = ((u * nck + nck) * nC - 1) / N;
        slots = cl - cf + 1 > slots ? cl - cf + 1 : slots;
    }
    *nC_out = nC;
    *slots_out = (int)slots;
    // a stream-K CTA's set-up is longer (its share's bounds and the slots of two
    // units): ~0.6 chunk-steps more, measured on the GQA, long-context and
    // append-and-attend workloads against their uniform grids
    return worst + kSetup + 0.6;
}

struct DecodePlan {
    int G = 0;
    bool use_mma = false;
    int nsplit = 0;
    int64_t split_tokens = 0;
    int64_t sk_ctas = 0, sk_nck = 0;     // stream-K grid (sk_ctas > 0)
    size_t off_qp = 0, off_up = 0, off_ml = 0, off_acc = 0, bytes = 0;
};

void layout_ws(int d, size_t BHq, int nsplit, DecodePlan* p) {
    size_t off = 0;
    p->off_qp = off; off = round_up(off + BHq * d * 4, 256);
    p->off_up = off; off = round_up(off + BHq * d * 4, 256);
    p->off_ml = off; off = round_up(off + BHq * nsplit * 2 * 4, 256);
    p->off_acc = off; off = round_up(off + BHq * nsplit * d * 4, 256);
    p->bytes = off;
}

// upper_bound: the plan whose workspace bounds every call up to Tmax tokens.
// equal_len: every sequence has Tmax tokens (no per-sequence lengths), which
// lets the tensor-core kernel take the stream-K grid when it models faster.
// The plan for head_dim d on a GPU of num_sms SMs; decode_path as tq_set_decode_path.
bool make_plan_core(int d, int num_sms, int decode_path, int64_t B, int64_t Hq, int64_t Hkv, int64_t Tmax,
                    DecodePlan* p, bool upper_bound, bool equal_len) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Tmax < 0 || Hq % Hkv || num_sms < 1) return false;
    p->G = (int)(Hq / Hkv);
    p->use_mma = decode_path != 1 && mma_supported(d, p->G);
    const int64_t pairs = B * Hkv > 0 ? B * Hkv * decode_head_groups(p->use_mma, p->G) : 1;
    const int64_t cap = (int64_t)num_sms * decode_ctas_per_sm(p->use_mma);
    const int chunk = decode_chunk_tokens(d, p->use_mma);
    const int64_t nchunk = Tmax > 0 ? (Tmax + chunk - 1) / chunk : 1;
    const int warps = decode_warps(p->use_mma, p->G);
    double t_split = 0.0;
    p->nsplit = upper_bound ? (int)split_loop_bound(cap, pairs, nchunk)
                            : choose_nsplit(cap, warps, pairs, nchunk, &t_split);
    p->split_tokens = ((nchunk + p->nsplit - 1) / p->nsplit) * chunk;
    p->sk_ctas = p->sk_nck = 0;
    if (!upper_bound && equal_len && p->use_mma && Tmax > 0 && B * Hkv > 0) {
        int64_t nC = 0;
        int slots = 0;
        const double t_sk = streamk_plan(cap, warps, pairs, nchunk, &nC, &slots);
        // the workspace of any call was sized by the split count bound
        const bool faster = decode_path == 3 || (decode_path == 0 && t_sk < t_split);
        if (t_sk > 0.0 && faster && slots <= split_loop_bound(cap, pairs, nchunk)) {
            p->nsplit = slots;
            p->sk_ctas = nC;
            p->sk_nck = nchunk;
        }
    }
    layout_ws(d, (size_t)(B * Hq), p->nsplit, p);
    return true;
}

bool make_plan(const tq_handle* h, int64_t B, int64_t Hq, int64_t Hkv, int64_t Tmax, DecodePlan* p,
               bool upper_bound, bool equal_len = false) {
    return h && make_plan_core(h->d, h->num_sms, h->decode_path, B, Hq, Hkv, Tmax, p, upper_bound, equal_len);
}

tq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

bool cache_ok(const tq_handle* h, const tq_cache* c) {
    return c && c->base && aligned(c->base, 16) && c->B >= 0 && c->Hkv > 0 && c->Tcap > 0 &&
           c->Tcap % kBlockT == 0 && h &&
           (!c->block_table || (aligned(c->block_table, 4) && c->pool_blocks > 0 && c->pool_blocks < (1LL << 31)));
}

tq_status prepare_encode(const tq_handle* h, const void* x, tq_dtype dt, int64_t B, int64_t Hkv, int64_t Tnew,
                         int64_t sb, int64_t sh, int64_t st, const tq_cache* c, int64_t t0, EncArgs* a,
                         bool* empty) {
    *empty = false;
    if (!h || !dtype_ok(dt) || !cache_ok(h, c)) return TQ_ERR_INVALID_ARG;
    if (B != c->B || Hkv != c->Hkv || Tnew < 0 || t0 < 0 || t0 + Tnew > c->Tcap) return TQ_ERR_INVALID_ARG;
    if (B == 0 || Tnew == 0) {
        *empty = true;
        return TQ_OK;
    }
    if (!x || !aligned(x, dtype_size(dt)) || sb < 0 || sh < 0 || st < 0) return TQ_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev != h->device) return TQ_ERR_INVALID_ARG;
    if (B * Hkv * Tnew >= (int64_t)1 << 31) return TQ_ERR_UNSUPPORTED;      // vector indices are 32-bit
    *a = EncArgs{};
    a->x = x; a->sb = sb; a->sh = sh; a->st = st;
    a->B = B; a->Hkv = Hkv; a->Tnew = Tnew; a->t0 = t0;
    a->NB = c->Tcap / kBlockT;
    a->cache = static_cast<uint8_t*>(c->base);
    a->table = c->block_table;
    a->pool = c->pool_blocks;
    a->dsign = h->dsign; a->sthr = h->dSThr; a->bimg = h->dSB; a->err = h->derr; a->cb = h->cb;
    for (int i = 0; i < 4; ++i) a->dneg[i] = h->dneg[i];
    const int64_t es = (int64_t)dtype_size(dt);
    a->vec16 = (aligned(x, 16) && (sb * es) % 16 == 0 && (sh * es) % 16 == 0 && (st * es) % 16 == 0) ? 1 : 0;
    a->fdT = make_fastdiv((uint32_t)Tnew);
    a->fdH = make_fastdiv((uint32_t)Hkv);
    return TQ_OK;
}

tq_status encode_common(const tq_handle* h, const void* x, tq_dtype dt, int64_t B, int64_t Hkv, int64_t Tnew,
                        int64_t sb, int64_t sh, int64_t st, const tq_cache* c, int64_t t0, void* stream, bool is_k) {
    EncArgs a;
    bool empty;
    const tq_status r = prepare_encode(h, x, dt, B, Hkv, Tnew, sb, sh, st, c, t0, &a, &empty);
    if (r != TQ_OK || empty) return r;
    return cuda_status(launch_encode(h->d, is_k, dt, a, h->num_sms, false, static_cast<cudaStream_t>(stream)));
}

// Checks of an attention call and its kernel arguments; *G receives the group size.
tq_status prepare_attend(const tq_handle* h, const void* q, tq_dtype qdt, int64_t B, int64_t Hq, const tq_cache* kc,
                         const tq_cache* vc, const int32_t* seq_lens, int64_t T, float scale, float* out, void* ws,
                         size_t ws_bytes, DecodePlan* p, DecArgs* a) {
    if (!h || !dtype_ok(qdt) || !cache_ok(h, kc) || !cache_ok(h, vc)) return TQ_ERR_INVALID_ARG;
    if (B < 0 || Hq <= 0 || kc->B != B || vc->B != B || kc->Hkv != vc->Hkv || kc->Tcap != vc->Tcap)
        return TQ_ERR_INVALID_ARG;
    const int64_t Hkv = kc->Hkv;
    if (Hq % Hkv) return TQ_ERR_INVALID_ARG;
    const int64_t G = Hq / Hkv;
    // grid limits: y = kv heads x query-head groups, z = batch; one combine CTA per query head
    if (B > 65535 || Hkv * ((G + 7) / 8) > 65535 || B * Hq >= ((int64_t)1 << 31)) return TQ_ERR_UNSUPPORTED;
    if (!seq_lens && (T < 0 || T > kc->Tcap)) return TQ_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
    if (B == 0) return TQ_OK;
    if (!q || !out || !ws || !aligned(q, dtype_size(qdt)) || !aligned(out, 16) || !aligned(ws, 256))
        return TQ_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev != h->device) return TQ_ERR_INVALID_ARG;
    const int64_t Tmax = seq_lens ? kc->Tcap : T;
    if (!make_plan(h, B, Hq, Hkv, Tmax, p, false, seq_lens == nullptr)) return TQ_ERR_INVALID_ARG;
    if (ws_bytes < p->bytes) return TQ_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    *a = DecArgs{};
    a->qp = reinterpret_cast<float*>(w + p->off_qp);
    a->up = reinterpret_cast<float*>(w + p->off_up);
    a->kc = static_cast<const uint8_t*>(kc->base);
    a->vc = static_cast<const uint8_t*>(vc->base);
    a->ktable = kc->block_table;
    a->vtable = vc->block_table;
    a->kpool = kc->pool_blocks;
    a->vpool = vc->pool_blocks;
    a->NB = kc->Tcap / kBlockT;
    a->seq_lens = seq_lens;
    a->T = T;
    a->Tcap = kc->Tcap;
    a->B = B; a->Hq = Hq; a->Hkv = Hkv;
    a->nsplit = p->nsplit;
    a->split_tokens = p->split_tokens;
    a->sk_ctas = (int)p->sk_ctas;
    a->sk_nck = p->sk_nck;
    a->sk_total = p->sk_nck * B * Hkv * decode_head_groups(p->use_mma, p->G);
    a->scale_log2 = scale * kLog2e;
    a->part_ml = reinterpret_cast<float*>(w + p->off_ml);
    a->part_acc = reinterpret_cast<float*>(w + p->off_acc);
    a->err = h->derr;
    a->first_wait = h->first_wait >= 0 ? h->first_wait : kDefaultWaitLimit;
    a->cb = h->cb;
    return TQ_OK;
}

// Prologue, split-K attention, combine.  chained: the prologue is a
// programmatic dependent of the kernel before it (the fused step's encodes).
cudaError_t launch_attend(const tq_handle* h, const void* q, tq_dtype qdt, const DecodePlan& p, const DecArgs& a,
                          float* out, bool chained, cudaStream_t s, bool qjl = true) {
    const int64_t BHq = a.B * a.Hq;
    cudaError_t e = launch_prologue(h->d, q, qdt, BHq, h->dsign, h->dST, const_cast<float*>(a.qp),
                                    const_cast<float*>(a.up), chained, s);
    if (e == cudaSuccess && h->ev_start) e = cudaEventRecord(h->ev_start, s);
    if (e == cudaSuccess) e = launch_decode(h->d, p.G, p.use_mma, qjl, a, s);
    if (e == cudaSuccess && h->ev_stop) e = cudaEventRecord(h->ev_stop, s);
    if (e == cudaSuccess) e = launch_combine(h->d, BHq, p.nsplit, a.part_ml, a.part_acc, h->dsign, out, s);
    return e;
}

}  // namespace

extern "C" {

const char* tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "ok";
        case TQ_ERR_INVALID_ARG: return "invalid argument";
        case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case TQ_ERR_CUDA: return "CUDA error";
        case TQ_ERR_WORKSPACE: return "workspace too small";
        case TQ_ERR_DEVICE_CHECK: return "device-side check failed";
    }
    return "unknown status";
}

tq_status tq_params_host(int head_dim, uint64_t seed, int8_t* D, float* S, float* c8, float* b7) {
    return make_params(head_dim, seed, D, S, c8, b7) ? TQ_OK : TQ_ERR_INVALID_ARG;
}

size_t tq_block_bytes(int head_dim, int is_k) {
    if (!head_dim_ok(head_dim)) return 0;
    return (size_t)block_bytes(head_dim, is_k != 0);
}

size_t tq_cache_bytes(int head_dim, int is_k, int64_t B, int64_t Hkv, int64_t Tcap) {
    if (!head_dim_ok(head_dim) || B < 0 || Hkv < 0 || Tcap <= 0 || Tcap % kBlockT) return 0;
    return (size_t)(B * Hkv * (Tcap / kBlockT)) * (size_t)block_bytes(head_dim, is_k != 0);
}

tq_status tq_init(int head_dim, uint64_t seed, tq_handle** out) {
    if (!out || !head_dim_ok(head_dim)) return TQ_ERR_INVALID_ARG;
    *out = nullptr;
    tq_handle* h = new (std::nothrow) tq_handle();
    if (!h) return TQ_ERR_CUDA;
    const int d = head_dim;
    h->d = d;
    h->seed = seed;
    h->hD.resize(d);
    h->hS.resize((size_t)d * d);
    make_params(d, seed, h->hD.data(), h->hS.data(), h->hc, h->hb);
    for (int k = 0; k < 8; ++k) h->cb.c[k] = h->hc[k];
    for (int k = 0; k < 7; ++k) h->cb.b[k] = h->hb[k];
    uint32_t lo[2] = {0, 0}, hi[2] = {0, 0};
    for (int k = 0; k < 8; ++k) {
        const uint16_t bits = double_to_half_bits((double)h->hc[k]);
        lo[k >> 2] |= (uint32_t)(bits & 0xFF) << (8 * (k & 3));
        hi[k >> 2] |= (uint32_t)(bits >> 8) << (8 * (k & 3));
    }
    h->cb.lut_lo[0] = lo[0]; h->cb.lut_lo[1] = lo[1];
    h->cb.lut_hi[0] = hi[0]; h->cb.lut_hi[1] = hi[1];
    for (int k = 0; k < 32; ++k) h->cb.pow2[k] = 1u << k;
    // integer byte limbs of c 2^14 (exact when each fp16 centroid is a multiple of 2^-14)
    h->cb.k8 = 1;
    uint32_t l8[2] = {0, 0}, h8[2] = {0, 0};
    for (int k = 0; k < 8; ++k) {
        const double ci = half_bits_to_double(double_to_half_bits((double)h->hc[k])) * 16384.0;
        const long long v = std::llround(ci);
        if ((double)v != ci || v > 32767 || v < -32768) h->cb.k8 = 0;
        const int lo8 = (int)(((v + 128) & 255) - 128), hi8 = (int)((v - lo8) / 256);
        if (hi8 < -128 || hi8 > 127) h->cb.k8 = 0;
        l8[k >> 2] |= (uint32_t)(uint8_t)(int8_t)lo8 << (8 * (k & 3));
        h8[k >> 2] |= (uint32_t)(uint8_t)(int8_t)hi8 << (8 * (k & 3));
    }
    h->cb.lut8_lo[0] = l8[0]; h->cb.lut8_lo[1] = l8[1];
    h->cb.lut8_hi[0] = h8[0]; h->cb.lut8_hi[1] = h8[1];

    std::vector<float> sign(d), st((size_t)d * d), sthr((size_t)d * d);
    for (int j = 0; j < d; ++j) sign[j] = (float)h->hD[j];
    for (int j = 0; j < d; ++j)
        if (h->hD[j] < 0) h->dneg[j >> 5] |= 1u << (j & 31);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) st[(size_t)j * d + i] = h->hS[(size_t)i * d + j];
    const int R = d / 32;
    for (int j = 0; j < d; ++j)
        for (int r = 0; r < R; ++r)
            for (int l = 0; l < 32; ++l) {
                const int row = sign_row(d, r, l);
                sthr[((size_t)j * R + r) * 32 + l] = h->hS[(size_t)row * d + j];
            }
    // d = 128: the JL matrix as the B operand of the tensor-core encode, rows
    // permuted into sign-word order, fp16 hi and lo limbs of each fp32 entry
    std::vector<uint16_t> simg;
    if (d == 64) {
        // d = 64: rows in sign-word order (word r, bit l), the K index in the slot order of
        // the bulk encode's rotated tile (16 t + p is coordinate slot_coord(0, t, p))
        simg.assign((size_t)2 * 64 * d, 0);
        for (int nr = 0; nr < d; ++nr) {
            const int row = sign_row(d, nr >> 5, nr & 31);
            for (int k = 0; k < d; ++k) {
                const double sv = (double)h->hS[(size_t)row * d + slot_coord(0, k >> 4, k & 15)];
                const uint16_t hi = double_to_half_bits(sv);
                const uint16_t lo = double_to_half_bits(sv - half_bits_to_double(hi));
                const size_t at = sw128_k_offset(nr, k) / 2;
                simg[at] = hi;
                simg[(size_t)64 * d + at] = lo;
            }
        }
    }
    if (d == 128) {
        simg.assign((size_t)2 * kTcRows * d, 0);
        for (int n = 0; n < d; ++n) {
            const int row = qjl_row_of_column(n);
            for (int k = 0; k < d; ++k) {
                const double sv = (double)h->hS[(size_t)row * d + k];
                const uint16_t hi = double_to_half_bits(sv);
                const uint16_t lo = double_to_half_bits(sv - half_bits_to_double(hi));
                const size_t at = sw128_k_offset(n, k) / 2;
                simg[at] = hi;
                simg[(size_t)kTcRows * d + at] = lo;
            }
        }
    }
    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
    if (e == cudaSuccess) e = cudaMalloc(&h->dsign, sizeof(float) * d);
    if (e == cudaSuccess) e = cudaMalloc(&h->dST, sizeof(float) * d * d);
    if (e == cudaSuccess) e = cudaMalloc(&h->dSThr, sizeof(float) * d * d);
    if (e == cudaSuccess) e = cudaMalloc(&h->derr, sizeof(int));
    if (e == cudaSuccess && !simg.empty()) e = cudaMalloc(&h->dSB, simg.size() * sizeof(uint16_t));
    if (e == cudaSuccess && !simg.empty())
        e = cudaMemcpy(h->dSB, simg.data(), simg.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->dsign, sign.data(), sizeof(float) * d, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->dST, st.data(), sizeof(float) * d * d, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->dSThr, sthr.data(), sizeof(float) * d * d, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(h->derr, 0, sizeof(int));
    if (e != cudaSuccess) {
        tq_destroy(h);
        return TQ_ERR_CUDA;
    }
    *out = h;
    return TQ_OK;
}

tq_status tq_destroy(tq_handle* h) {
    if (!h) return TQ_OK;
    cudaFree(h->dsign);
    cudaFree(h->dST);
    cudaFree(h->dSThr);
    cudaFree(h->dSB);
    cudaFree(h->derr);
    delete h;
    return TQ_OK;
}

tq_status tq_get_params(const tq_handle* h, int8_t* D, float* S, float* c8, float* b7) {
    if (!h) return TQ_ERR_INVALID_ARG;
    const int d = h->d;
    if (D) std::memcpy(D, h->hD.data(), d);
    if (S) std::memcpy(S, h->hS.data(), sizeof(float) * d * d);
    if (c8) std::memcpy(c8, h->hc, sizeof(h->hc));
    if (b7) std::memcpy(b7, h->hb, sizeof(h->hb));
    return TQ_OK;
}

int tq_head_dim(const tq_handle* h) { return h ? h->d : 0; }

tq_status tq_encode_k(const tq_handle* h, const void* x, tq_dtype dt, int64_t B, int64_t Hkv, int64_t Tnew,
                      int64_t sb, int64_t sh, int64_t st, const tq_cache* kc, int64_t t0, void* stream) {
    return encode_common(h, x, dt, B, Hkv, Tnew, sb, sh, st, kc, t0, stream, true);
}

tq_status tq_encode_v(const tq_handle* h, const void* x, tq_dtype dt, int64_t B, int64_t Hkv, int64_t Tnew,
                      int64_t sb, int64_t sh, int64_t st, const tq_cache* vc, int64_t t0, void* stream) {
    return encode_common(h, x, dt, B, Hkv, Tnew, sb, sh, st, vc, t0, stream, false);
}

tq_status tq_decode_plan(int num_sms, int head_dim, int64_t B, int64_t Hq, int64_t Hkv, int64_t T, int equal_len,
                         int* nsplit, int64_t* split_tokens, int64_t* streamk_ctas, int64_t* streamk_chunks,
                         int* chunk_tokens) {
    if (!nsplit || !split_tokens || !streamk_ctas || !streamk_chunks || !chunk_tokens) return TQ_ERR_INVALID_ARG;
    if (!head_dim_ok(head_dim) || T < 0) return TQ_ERR_INVALID_ARG;
    DecodePlan p;
    if (!make_plan_core(head_dim, num_sms, 0, B, Hq, Hkv, T, &p, false, equal_len != 0)) return TQ_ERR_INVALID_ARG;
    *nsplit = p.nsplit;
    *split_tokens = p.split_tokens;
    *streamk_ctas = p.sk_ctas;
    *streamk_chunks = p.sk_nck;
    *chunk_tokens = decode_chunk_tokens(head_dim, p.use_mma);
    return TQ_OK;
}

size_t tq_attend_workspace_bytes(const tq_handle* h, int64_t B, int64_t Hq, int64_t Hkv, int64_t Tmax) {
    DecodePlan p;
    if (!make_plan(h, B, Hq, Hkv, Tmax, &p, true)) return 0;
    return p.bytes;
}

// Partials per row of a prefill call: the d = 128 kernel spreads row tiles over the SMs
// and merges up to prefill_tc_split_cap partials per row; the others write one.
static int prefill_splits(const tq_handle* h, int64_t rows) {
    return h->d == 128 ? prefill_tc_split_cap(h->num_sms, rows) : 1;
}

size_t tq_prefill_workspace_bytes(const tq_handle* h, int64_t B, int64_t Lq, int64_t Hq) {
    if (!h || B < 0 || Lq < 0 || Hq <= 0) return 0;
    DecodePlan p;
    const int64_t rows = B * Lq * Hq;
    layout_ws(h->d, (size_t)rows, prefill_splits(h, rows), &p);
    return p.bytes;
}

tq_status tq_attend_prefill(const tq_handle* h, const void* q, tq_dtype qdt, int64_t B, int64_t Lq, int64_t Hq,
                            const tq_cache* kc, const tq_cache* vc, int64_t T0, float scale, float* out, void* ws,
                            size_t ws_bytes, void* stream) {
    if (!h || !dtype_ok(qdt) || !cache_ok(h, kc) || !cache_ok(h, vc)) return TQ_ERR_INVALID_ARG;
    if (B < 0 || Lq < 0 || Hq <= 0 || T0 < 0 || kc->B != B || vc->B != B || kc->Hkv != vc->Hkv ||
        kc->Tcap != vc->Tcap || T0 + Lq > kc->Tcap || !std::isfinite(scale))
        return TQ_ERR_INVALID_ARG;
    const int64_t Hkv = kc->Hkv;
    if (Hq % Hkv) return TQ_ERR_INVALID_ARG;
    const int G = (int)(Hq / Hkv);
    if (B > 65535 || Hkv > 65535) return TQ_ERR_UNSUPPORTED;          // grid limits
    if ((Lq * G + 63) / 64 * 2 >= ((int64_t)1 << 31)) return TQ_ERR_UNSUPPORTED;
    if (Lq * G > ((int64_t)1 << 27)) return TQ_ERR_UNSUPPORTED;        // row tiles per sequence (host plan)
    if (B == 0 || Lq == 0) return TQ_OK;
    if (!q || !out || !ws || !aligned(q, dtype_size(qdt)) || !aligned(out, 16) || !aligned(ws, 256))
        return TQ_ERR_INVALID_ARG;
    if (B * Lq * Hq >= ((int64_t)1 << 31)) return TQ_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev != h->device) return TQ_ERR_INVALID_ARG;
    const int64_t rows = B * Lq * Hq;
    const int cap = prefill_splits(h, rows);
    DecodePlan p;
    layout_ws(h->d, (size_t)rows, cap, &p);
    if (ws_bytes < p.bytes) return TQ_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    DecArgs a{};
    a.qp = reinterpret_cast<float*>(w + p.off_qp);
    a.up = reinterpret_cast<float*>(w + p.off_up);
    a.kc = static_cast<const uint8_t*>(kc->base);
    a.vc = static_cast<const uint8_t*>(vc->base);
    a.ktable = kc->block_table;
    a.vtable = vc->block_table;
    a.kpool = kc->pool_blocks;
    a.vpool = vc->pool_blocks;
    a.NB = kc->Tcap / kBlockT;
    a.Tcap = kc->Tcap;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv;
    a.nsplit = 1;
    a.scale_log2 = scale * kLog2e;
    a.part_ml = reinterpret_cast<float*>(w + p.off_ml);
    a.part_acc = reinterpret_cast<float*>(w + p.off_acc);
    a.err = h->derr;
    a.first_wait = kDefaultWaitLimit;
    a.cb = h->cb;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_prologue(h->d, q, qdt, rows, h->dsign, h->dST, const_cast<float*>(a.qp),
                                    const_cast<float*>(a.up), false, s);
    int nsplit = 1;
    if (e == cudaSuccess)
        e = h->d == 128 ? launch_prefill_tc(G, a, Lq, T0, h->num_sms, cap, &nsplit, s)
                        : launch_prefill(h->d, G, a, Lq, T0, s);
    if (e == cudaSuccess) e = launch_combine(h->d, rows, nsplit, a.part_ml, a.part_acc, h->dsign, out, s);
    return cuda_status(e);
}

const char* tq_attend_path(const tq_handle* h, int64_t Hq, int64_t Hkv) {
    if (!h || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return "invalid";
    return (h->decode_path != 1 && mma_supported(h->d, (int)(Hq / Hkv))) ? "mma" : "simt";
}

tq_status tq_attend_decode(const tq_handle* h, const void* q, tq_dtype qdt, int64_t B, int64_t Hq,
                           const tq_cache* kc, const tq_cache* vc, const int32_t* seq_lens, int64_t T,
                           float scale, float* out, void* ws, size_t ws_bytes, void* stream) {
    DecodePlan p;
    DecArgs a;
    const tq_status r = prepare_attend(h, q, qdt, B, Hq, kc, vc, seq_lens, T, scale, out, ws, ws_bytes, &p, &a);
    if (r != TQ_OK || B == 0) return r;
    return cuda_status(launch_attend(h, q, qdt, p, a, out, false, static_cast<cudaStream_t>(stream)));
}

tq_status tq_attend_decode_polar(const tq_handle* h, const void* q, tq_dtype qdt, int64_t B, int64_t Hq,
                                 const tq_cache* kc, const tq_cache* vc, const int32_t* seq_lens, int64_t T,
                                 float scale, float* out, void* ws, size_t ws_bytes, void* stream) {
    DecodePlan p;
    DecArgs a;
    const tq_status r = prepare_attend(h, q, qdt, B, Hq, kc, vc, seq_lens, T, scale, out, ws, ws_bytes, &p, &a);
    if (r != TQ_OK || B == 0) return r;
    return cuda_status(launch_attend(h, q, qdt, p, a, out, false, static_cast<cudaStream_t>(stream), false));
}

tq_status tq_append_attend(const tq_handle* h, const void* k_new, const void* v_new, tq_dtype kv_dtype,
                           int64_t Tnew, int64_t sb, int64_t sh, int64_t st, const tq_cache* kc,
                           const tq_cache* vc, int64_t t0, const void* q, tq_dtype q_dtype, int64_t Hq,
                           float scale, float* out, void* ws, size_t ws_bytes, void* stream) {
    if (!kc || !vc) return TQ_ERR_INVALID_ARG;
    const int64_t B = kc->B, Hkv = kc->Hkv;
    EncArgs ek, ev;
    bool empty_k, empty_v;
    tq_status r = prepare_encode(h, k_new, kv_dtype, B, Hkv, Tnew, sb, sh, st, kc, t0, &ek, &empty_k);
    if (r == TQ_OK) r = prepare_encode(h, v_new, kv_dtype, B, Hkv, Tnew, sb, sh, st, vc, t0, &ev, &empty_v);
    if (r != TQ_OK) return r;
    DecodePlan p;
    DecArgs a;
    r = prepare_attend(h, q, q_dtype, B, Hq, kc, vc, nullptr, t0 + Tnew, scale, out, ws, ws_bytes, &p, &a);
    if (r != TQ_OK || B == 0) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    const bool chained = !empty_k;
    if (chained) {
        // K encode as a plain launch, V encode and the prologue as its
        // programmatic dependents (each completes only after its predecessor);
        // the split-K kernel sets up while they run and reads the cache and
        // the query operands after it waits.
        e = launch_encode(h->d, true, kv_dtype, ek, h->num_sms, false, s);
        if (e == cudaSuccess) e = launch_encode(h->d, false, kv_dtype, ev, h->num_sms, true, s);
        a.fresh_lo = t0;
        a.fresh_hi = t0 + Tnew;
    }
    if (e == cudaSuccess) e = launch_attend(h, q, q_dtype, p, a, out, chained, s);
    return cuda_status(e);
}

tq_status tq_set_decode_events(tq_handle* h, void* ev_start, void* ev_stop) {
    if (!h || (ev_start == nullptr) != (ev_stop == nullptr)) return TQ_ERR_INVALID_ARG;
    h->ev_start = static_cast<cudaEvent_t>(ev_start);
    h->ev_stop = static_cast<cudaEvent_t>(ev_stop);
    return TQ_OK;
}

tq_status tq_set_wait_limit(tq_handle* h, int first_wait) {
    if (!h) return TQ_ERR_INVALID_ARG;
    h->first_wait = first_wait < 0 ? -1 : first_wait;
    return TQ_OK;
}

tq_status tq_set_decode_path(tq_handle* h, int path) {
    if (!h || path < 0 || path > 3) return TQ_ERR_INVALID_ARG;
    h->decode_path = path;
    return TQ_OK;
}

tq_status tq_device_status(const tq_handle* h, void* stream) {
    if (!h) return TQ_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TQ_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, h->derr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ERR_CUDA;
    if (v != 0) {
        if (cudaMemset(h->derr, 0, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
        return TQ_ERR_DEVICE_CHECK;
    }
    return TQ_OK;
}

}  // extern "C"
