// rq_noalloc.cu -- qjl_score for callers that cannot allocate device memory.
//
// qjl_score needs a scratch buffer (the rotated / projected queries) that its
// caller normally allocates.  Some callers cannot do that: a serving engine
// that reserved all of its HBM for the KV cache at start-up and forbids any
// later device allocation, or a host that reaches this library through a
// plain-C plugin interface that hands over device pointers but no allocator.
// qjl_score_noalloc runs the same kernels with that scratch taken from a
// fixed array that lives in this library's own device image instead.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "rq.h"
#include "rq_kernels.h"

namespace {

// The scratch every qjl_score_noalloc call on a device uses.  It is part of
// the library's device image: every GPU that loads librq holds these bytes
// until the process exits.  In host code `g_score_scratch` is only a
// host-side stand-in for the symbol, never a device address; the address the
// kernels get comes from cudaGetSymbolAddress below.
constexpr size_t kScratchBytes = (size_t)8 << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_score_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, looked up once through the runtime (the
// library links only against cudart).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

// Device address of the scratch array on the current device, looked up with
// that device current and remembered together with the context it belongs
// to; nullptr on failure.  A device reset (or any teardown and re-creation of
// the primary context) reloads the library's module, possibly at another
// address: the context check sees the new context and looks the address up
// again instead of handing out a stale pointer.
void *scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return nullptr;
    // The context current on this thread; null when the runtime has not made
    // the device's primary context current here yet (the lookup below does).
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || !p) return nullptr;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" rq_status qjl_score_noalloc(const void *q, int64_t G, int n_q, int d, int m, const void *proj,
                                       rq_dtype proj_dtype, const uint8_t *signs, const uint16_t *sk_norms,
                                       int64_t T_len, const void *codes, const uint16_t *norms, int bits,
                                       rq_layout layout, int use_signs, uint64_t sign_seed,
                                       const float *centroids, float *scores, rq_stream_t stream)
{
    const size_t need = qjl_score_workspace_bytes(G, n_q, d, m);
    if (need > kScratchBytes) return RQ_ESIZE;
    void *ws = scratch_for_current_device();
    if (!ws) return RQ_ECUDA;
    // Nothing in the scratch has to start at zero: the score prologue writes
    // every byte the main kernel reads before it reads it.
    return qjl_score(q, G, n_q, d, m, proj, proj_dtype, signs, sk_norms, T_len, codes, norms, bits, layout,
                     use_signs, sign_seed, centroids, scores, ws, kScratchBytes, stream);
}
