// noalloc.cu -- tri_mul_forward_noalloc: the update for callers that cannot allocate
// device memory.
//
// tri_mul_forward needs a workspace (a, b and x) that the caller allocates and binds.
// Some callers cannot do that: a plug-in running inside a host framework that owns the
// device allocator and offers the plug-in no way to request memory, or a code path that
// must not risk an allocation failing (or waiting on the allocator) in the middle of its
// work. For them this entry point keeps a, b and x in a fixed array that is part of the
// library itself. The three kernels and their launches are exactly those of
// tri_mul_forward; only the place the intermediates live differs.
#include <cuda_runtime.h>

#include <mutex>

#include "trimul.h"

namespace trimul {
trimul_status_t set_last_error(trimul_status_t st, const char *msg);
}

// The library's own scratch for a, b and x. Every GPU that loads the library holds
// these TRIMUL_NOALLOC_SCRATCH_BYTES bytes of device memory until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TRIMUL_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mu;
void *g_scratch_ptr[64];
bool g_scratch_ready[64];

// Device address of g_noalloc_scratch on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device, with
// that device current, and cached.
trimul_status_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return trimul::set_last_error(TRIMUL_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return trimul::set_last_error(TRIMUL_ERR_UNSUPPORTED_DEVICE, "device index out of range");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ready[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return trimul::set_last_error(TRIMUL_ERR_CUDA, "cudaGetSymbolAddress of the no-allocation scratch failed");
        g_scratch_ptr[dev] = p;
        g_scratch_ready[dev] = true;
    }
    *out = g_scratch_ptr[dev];
    return TRIMUL_OK;
}
}  // namespace

extern "C" trimul_status_t tri_mul_forward_noalloc(const trimul_pair_t *z, const void *mask,
                                                   const trimul_layer_t *layer, trimul_direction_t direction,
                                                   trimul_pair_t *out, void *stream) {
    if (!z || !layer || !out) return trimul::set_last_error(TRIMUL_ERR_INVALID_ARG, "NULL argument");
    if (z->dtype != TRIMUL_F32 && z->dtype != TRIMUL_BF16)
        return trimul::set_last_error(TRIMUL_ERR_INVALID_ARG, "z must be F32 or BF16");
    if (direction != TRIMUL_OUTGOING && direction != TRIMUL_INCOMING)
        return trimul::set_last_error(TRIMUL_ERR_INVALID_ARG, "unknown direction");
    // a, b and x: three planes, the same layout tri_mul_forward uses in a bound workspace
    // (which also holds the mask extents after them; this path skips no tiles and needs none)
    const size_t ws = tri_mul_workspace_bytes(layer, z->B, z->N, z->dtype);
    if (ws == 0) return trimul::set_last_error(TRIMUL_ERR_INVALID_ARG, "invalid layer or size");
    const size_t need = ws - (((size_t)z->B * 2 * sizeof(int) + 255) & ~size_t(255));
    if (need > (size_t)TRIMUL_NOALLOC_SCRATCH_BYTES)
        return trimul::set_last_error(TRIMUL_ERR_WORKSPACE,
                                      "problem needs more intermediate memory than the built-in "
                                      "TRIMUL_NOALLOC_SCRATCH_BYTES; use tri_mul_forward with a workspace");
    void *base = nullptr;
    trimul_status_t st = scratch_address(&base);
    if (st != TRIMUL_OK) return st;
    const size_t plane = need / 3;
    unsigned char *p = static_cast<unsigned char *>(base);
    void *a = p, *b = p + plane, *x = p + 2 * plane;
    // Nothing in the scratch has to start at zero: every call writes all of a, b and x
    // before reading them.
    const bool tc = z->dtype == TRIMUL_BF16;
    const float x_scale = tc ? tri_mul_contract_scale(z->N) : 1.0f;
    st = tri_mul_project(z, mask, layer, a, b, stream);
    if (st != TRIMUL_OK) return st;
    // for the sizes tri_mul_project accepts (N % 8 == 0, c_h % 32 == 0) a plane is exactly
    // B * c_h * N * N elements, so c_h follows from its size
    const int64_t c_h = (int64_t)(plane / ((size_t)z->B * z->N * z->N * (tc ? 2 : 4)));
    st = tri_mul_contract(a, b, x, z->B, c_h, z->N, tc ? TRIMUL_F16 : TRIMUL_F32, direction, x_scale, stream);
    if (st != TRIMUL_OK) return st;
    return tri_mul_output_gate(z, mask, x, x_scale, layer, out, stream);
}
