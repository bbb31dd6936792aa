// extents.cu -- the extents of a pair mask, for skipping wholly masked tiles.
//
// For batch element b: R_b = 1 + the largest row index i with a nonzero m[b, i, j] for some j,
// C_b = 1 + the largest column index j with a nonzero m[b, i, j] for some i (both 0 when every
// pair of b is masked). Every pair with i >= R_b or j >= C_b is masked, whatever the mask's
// pattern; for the left-aligned padding masks of the pages ("RFProteina architecture",
// section "Kernel support": masks are left-aligned, so a per-row valid count bounds the work)
// R_b = C_b = the valid length. The kernels use them to leave out tiles that are masked in
// full and the k-range beyond them; the results do not change.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

// One thread per 8 consecutive mask entries (16 bytes of bf16; N is a multiple of 8, so the
// 8 entries lie in one row). Warp maxima go to ext with atomicMax; ext is zeroed before.
__global__ void __launch_bounds__(256) mask_extents_kernel(const uint16_t *mask, long long NN, int N,
                                                           uint64_t rowdiv, int *ext) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.y;
    const uint16_t *m = mask + (long long)b * NN;
    int rmax = 0, cmax = 0;
    const long long step = (long long)gridDim.x * blockDim.x * 8;
    for (long long e = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8; e < NN; e += step) {
        const uint4 w = *reinterpret_cast<const uint4 *>(m + e);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        int last = -1;                                   // last nonzero entry among the 8
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (ws[k] & 0x7FFFu) last = 2 * k;           // +-0 counts as zero
            if (ws[k] & 0x7FFF0000u) last = 2 * k + 1;
        }
        if (last >= 0) {
            const int i = (int)div_by_magic((uint32_t)(e >> 3), rowdiv);
            const int j = (int)(e - (long long)i * N) + last;
            rmax = max(rmax, i + 1);
            cmax = max(cmax, j + 1);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        rmax = max(rmax, __shfl_xor_sync(0xffffffffu, rmax, o));
        cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    }
    if ((threadIdx.x & 31) == 0 && (rmax | cmax)) {
        atomicMax(ext + 2 * b, rmax);
        atomicMax(ext + 2 * b + 1, cmax);
    }
}

cudaError_t mask_extents_launch(const uint16_t *mask, int B, int N, uint64_t rowdiv, int *ext, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(ext, 0, sizeof(int) * 2 * (size_t)B, stream);
    if (e != cudaSuccess) return e;
    const long long NN = (long long)N * N;
    long long blocks = (NN / 8 + 255) / 256;
    if (blocks > 64) blocks = 64;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, (unsigned)B);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, mask_extents_kernel, mask, NN, N, rowdiv, ext);
}

}  // namespace trimul
