// tq_attend_decode_static: decode attention whose scratch memory (rotated
// queries and split-K softmax partials) lives in a fixed array inside the
// library instead of a caller-provided workspace, so that nothing has to be
// allocated on the device at call time.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds TQ_STATIC_SCRATCH_BYTES of it until the process exits.  Host
// code cannot use the variable's name as a device pointer (on the host it
// names a stand-in object), so the first call on each device asks the runtime
// for the array's device address with that device current and caches it.
#include <mutex>

#include "tq_internal.h"

namespace {

static __device__ __align__(256) unsigned char tq_static_scratch[TQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of tq_static_scratch on the current device (resolved once).
tq_status static_scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, tq_static_scratch);
        if (e != cudaSuccess || p == nullptr) return TQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_attend_decode_static(const tq_handle* h, const void* q, tq_dtype qdtype, int64_t B,
                                             int64_t Hq, const tq_cache* kc, const tq_cache* vc,
                                             const int32_t* seq_lens, int64_t T, float scale, float* out,
                                             void* stream) {
    if (!h) return TQ_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const tq_status st = static_scratch_address(&scratch);
    if (st != TQ_OK) return st;
    // Everything the decode writes into its scratch (rotated queries, every
    // split's partial) is written before it is read, so the array needs no
    // clearing between calls.  Sizes whose scratch exceeds the array get
    // TQ_ERR_WORKSPACE from the size check in tq_attend_decode.
    return tq_attend_decode(h, q, qdtype, B, Hq, kc, vc, seq_lens, T, scale, out, scratch,
                            (size_t)TQ_STATIC_SCRATCH_BYTES, stream);
}
