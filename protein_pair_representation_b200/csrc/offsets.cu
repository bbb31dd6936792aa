// offsets.cu -- the per-batch-element offset of the stored contraction result.
//
// The output LayerNorm normalizes x_ij over its c_h channels. When the gated projections a
// and b have a large common mode (for example positive projection biases), every channel of
// x_ij carries a large part L * mean(a_c) * mean(b_c), nearly the same for all pairs and
// channels, so |mean_c x| is many times std_c x, and rounding x itself to fp16 (11 significant
// bits) costs far more than the 2e-2 RMS budget once the LayerNorm divides by std_c x. The
// LayerNorm ignores a constant added to every channel of a pair, so the update stores x - o_b
// instead, with one offset per batch element,
//     o_b = L (1 / c_h) sum_c mean(a_c) mean(b_c)
// the channel mean of the common mode: mean(.) over a sample of b's unmasked pairs (K1 sums
// the first pairs of each tile) and L = (unmasked pairs) / (rows whose first pair is unmasked),
// the number of valid k of a padding mask's valid pairs, also for a shard of rows. The output
// kernel needs no correction: any o_b gives the same function, a good one only makes the stored
// value small. In the scaled units x is stored in, q = x_scale * o_b, rounded to an fp16 value
// so that a pair whose x is 0 in every channel is stored as exactly -q in every channel (and
// normalizes to exactly 0).
//
// The projection kernel gathers the sums (fixed point) and counts with integer atomics, so
// they, and with them every stored value, do not depend on the order the tiles finish in. This
// kernel turns them into q and zeroes them for the next forward.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

__global__ void __launch_bounds__(256) xoffsets_kernel(unsigned long long *acc, int c_h, float x_scale, float *q) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ double part[256];
    const int b = blockIdx.x;
    unsigned long long *ab = acc + (size_t)b * kAccStride;
    const double ns = (double)(long long)ab[kAccSampled];
    const double na = (double)(long long)ab[kAccAll];
    const double nr = (double)(long long)ab[kAccRows];
    const double unit = 1.0 / (double)kAccScale;
    double sum = 0.0;
    for (int c = threadIdx.x; c < c_h; c += blockDim.x)
        sum += ((double)(long long)ab[c] * unit) * ((double)(long long)ab[c_h + c] * unit);
    part[threadIdx.x] = sum;
    __syncthreads();                              // every sum has been read: clear them
    for (int c = threadIdx.x; c < kAccStride; c += blockDim.x) ab[c] = 0ull;
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {  // fixed-order tree: the same value every run
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const double L = nr > 0.0 ? na / nr : 0.0;
    const double o = ns > 0.0 ? part[0] / ((double)c_h * ns * ns) * L : 0.0;
    const float v = fminf(fmaxf((float)(o * (double)x_scale), -65504.f), 65504.f);
    const float vq = __half2float(__float2half_rn(v));
    for (int c = threadIdx.x; c < c_h; c += blockDim.x) q[(size_t)b * c_h + c] = vq;
}

cudaError_t xoffsets_launch(unsigned long long *acc, int B, int c_h, float x_scale, float *q, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)B);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xoffsets_kernel, acc, c_h, x_scale, q);
}

}  // namespace trimul
