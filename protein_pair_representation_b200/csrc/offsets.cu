// offsets.cu -- the per-(batch, channel) offset of the stored contraction result.
//
// The output LayerNorm normalizes x_ij over its c_h channels. When the gated projections a
// and b have a large common mode (for example positive projection biases), every channel of
// x_ij carries a large part L * mean(a_c) * mean(b_c) that is nearly the same for all pairs,
// so |mean_c x| is many times std_c x, and rounding x itself to fp16 (11 significant bits)
// costs far more than the 2e-2 RMS budget once the LayerNorm divides by std_c x. The update
// therefore stores x - o[b][c] instead, with o the common-mode estimate
//     o[b][c] = Sa Sb / P^1.5,   Sa = sum over the pairs of b of a_c, Sb likewise, P = #unmasked
// (for a padding mask of valid length L: P = L^2 and o = L mean(a_c) mean(b_c)), and the output
// kernel adds it back exactly: any o leaves the result unchanged, a good one only makes the
// stored value small. In the scaled units x is stored in, q = x_scale * o; the output kernel
// also needs Q[b][n] = sum_c q[b][c] W_o'[n][c], the offsets' share of the x-GEMM.
//
// The projection kernel gathers Sa, Sb (fixed point) and P with integer atomics, so the sums,
// and with them every stored value, do not depend on the order the tiles finish in. This
// kernel turns them into q and Q and zeroes them for the next forward.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

__global__ void __launch_bounds__(256) xoffsets_kernel(unsigned long long *acc, int c_h, int c_z, float x_scale,
                                                       const uint16_t *wo, float *q, float *Q) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ float qs[];                 // [c_h]
    const int b = blockIdx.x;
    unsigned long long *ab = acc + (size_t)b * (2 * c_h + 1);
    const double P = (double)(long long)ab[2 * c_h];
    const double inv = P > 0.0 ? 1.0 / (P * sqrt(P)) : 0.0;
    const double unit = 1.0 / (double)kAccScale;
    for (int c = threadIdx.x; c < c_h; c += blockDim.x) {
        const double sa = (double)(long long)ab[c] * unit;
        const double sb = (double)(long long)ab[c_h + c] * unit;
        const float v = fminf(fmaxf((float)(sa * sb * inv * (double)x_scale), -65504.f), 65504.f);
        // an fp16 value: a pair whose x is exactly 0 in every channel (a valid pair none of whose
        // k is valid) is then stored as exactly -q and read back as exactly 0, so its output
        // LayerNorm sees no rounding residue to amplify
        const float vq = __half2float(__float2half_rn(v));
        qs[c] = vq;
        q[(size_t)b * c_h + c] = vq;
    }
    __syncthreads();                              // every sum has been read: clear them
    for (int c = threadIdx.x; c < 2 * c_h + 1; c += blockDim.x) ab[c] = 0ull;
    for (int n = threadIdx.x; n < c_z; n += blockDim.x) {
        const uint16_t *w = wo + (size_t)n * c_h;
        float s = 0.f;
        for (int c = 0; c < c_h; ++c) s = fmaf(qs[c], __half2float(__ushort_as_half(w[c])), s);
        Q[(size_t)b * c_z + n] = s;
    }
}

cudaError_t xoffsets_launch(unsigned long long *acc, int B, int c_h, int c_z, float x_scale, const uint16_t *wo,
                            float *q, float *Q, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)B);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (size_t)c_h * sizeof(float);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xoffsets_kernel, acc, c_h, c_z, x_scale, wo, q, Q);
}

}  // namespace trimul
