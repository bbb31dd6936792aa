// noalloc.cu -- tri_mul_forward_noalloc: the update for callers that cannot allocate
// device memory.
//
// tri_mul_forward needs a workspace (a, b, x and a few small per-batch vectors) that the
// caller allocates and binds. Some callers cannot do that: a plug-in running inside a host
// framework that owns the device allocator and offers the plug-in no way to request memory,
// or a code path that must not risk an allocation failing (or waiting on the allocator) in
// the middle of its work. For them this entry point keeps the intermediates in a fixed array
// that is part of the library itself. The kernels, their launches and every argument check
// are exactly those of tri_mul_forward; only the place the intermediates live differs.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "trimul.h"

namespace trimul {
trimul_status_t set_last_error(trimul_status_t st, const char *msg);
trimul_status_t forward_buffers(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L,
                                trimul_direction_t dir, trimul_pair_t *out, bool residual, void *ws_ptr,
                                size_t ws_bytes, bool timing, void *stream, bool check_only, const int *given_ext);
}

// The library's own scratch for the intermediates. Every GPU that loads the library holds
// these TRIMUL_NOALLOC_SCRATCH_BYTES bytes of device memory until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TRIMUL_NOALLOC_SCRATCH_BYTES];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchEntry {
    unsigned long long ctx_id;    // driver id of the context the address belongs to (never 0 when set)
    void *ptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[64];

// The driver's id of the calling thread's current context (unique for the life of the process,
// so a context destroyed and created again gets a new one), or 0 when there is none yet or the
// driver entry points are unavailable.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(fn);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Device address of g_noalloc_scratch in the current device's context. In host code the
// array's name is only a host-side stand-in, so the address is looked up with the device
// current (cudaGetSymbolAddress) the first time a context uses it and cached under that
// context's id; a device reset or a new context gets a fresh lookup. Without a context id the
// lookup is repeated on every call.
trimul_status_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return trimul::set_last_error(TRIMUL_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return trimul::set_last_error(TRIMUL_ERR_UNSUPPORTED_DEVICE, "device index out of range");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long id = current_context_id();
    if (id != 0 && g_scratch[dev].ctx_id == id) {
        *out = g_scratch[dev].ptr;
        return TRIMUL_OK;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
        return trimul::set_last_error(TRIMUL_ERR_CUDA, "cudaGetSymbolAddress of the no-allocation scratch failed");
    const unsigned long long id_now = id != 0 ? id : current_context_id();   // the lookup made a context current
    g_scratch[dev].ctx_id = id_now;
    g_scratch[dev].ptr = p;
    *out = p;
    return TRIMUL_OK;
}
}  // namespace

extern "C" trimul_status_t tri_mul_forward_noalloc(const trimul_pair_t *z, const void *mask,
                                                   const trimul_layer_t *layer, trimul_direction_t direction,
                                                   trimul_pair_t *out, void *stream) {
    // every argument rule first, with nothing touched on the device
    trimul_status_t st = trimul::forward_buffers(z, mask, layer, direction, out, false, nullptr,
                                                 (size_t)TRIMUL_NOALLOC_SCRATCH_BYTES, false, stream, true, nullptr);
    if (st == TRIMUL_ERR_WORKSPACE)
        return trimul::set_last_error(TRIMUL_ERR_WORKSPACE,
                                      "problem needs more intermediate memory than the built-in "
                                      "TRIMUL_NOALLOC_SCRATCH_BYTES; use tri_mul_forward with a workspace");
    if (st != TRIMUL_OK) return st;
    void *base = nullptr;
    st = scratch_address(&base);
    if (st != TRIMUL_OK) return st;
    // Nothing in the array has to start at zero: a call writes every intermediate it reads
    // (the channel sums that must start at zero live in the layer handle).
    return trimul::forward_buffers(z, mask, layer, direction, out, false, base,
                                   (size_t)TRIMUL_NOALLOC_SCRATCH_BYTES, false, stream, false, nullptr);
}
