// fold.cu -- layer-creation kernels: fold LayerNorm gamma/beta into projection weights.
//
// For a linear layer y = LN(x) W^T + bias with LN(x) = (x - mean) rstd gamma + beta:
//   LN(x) W^T + bias = rstd (x . W' - mean sum_k W'_k) + (sum_k beta_k W_k + bias)
// with W' = W * gamma (per input column). The tensor-core kernels multiply raw inputs by
// W' (bf16) and apply the two per-row constants in their epilogue ("RFProteina
// architecture", section "Triangle multiplication on SM90": the LayerNorms are folded
// into the projection weights). The row sum is taken over the bf16-rounded W' that the
// tensor cores see, so the correction matches the product exactly.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

__device__ __forceinline__ float load_as_f32(const void *p, int idx, int is_bf16) {
    if (is_bf16) return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t *>(p)[idx]) << 16);
    return reinterpret_cast<const float *>(p)[idx];
}

// One block per source row r.
__global__ void fold_kernel(FoldArgs a) {
    const int r = blockIdx.x;
    const int tid = threadIdx.x;
    int dst_row = r;
    if (a.row_mode == 1) {
        const int g = a.operand * a.gpo + r / a.cpg;
        const int rr = r % a.cpg;
        dst_row = g * a.ncol + (rr / 16) * 32 + a.kind * 16 + (rr % 16);
    } else if (a.row_mode == 2) {
        // one block of rows per operand: [gate rows of all channels, projection rows of all channels]
        dst_row = a.operand * 2 * a.R + a.kind * a.R + r;
    }
    double sum_w = 0.0, shift = 0.0;
    for (int k = tid; k < a.K; k += blockDim.x) {
        const float w = load_as_f32(a.w, r * a.K + k, a.src_bf16);
        const float g = a.gamma ? load_as_f32(a.gamma, k, a.src_bf16) : 1.0f;
        const float bt = a.beta ? load_as_f32(a.beta, k, a.src_bf16) : 0.0f;
        float wq;
        const float sc = a.scale == 0.f ? 1.f : a.scale;
        if (a.dst_f16) {
            const __half h = __float2half_rn(w * g * sc);
            a.dst[(size_t)dst_row * a.K + k] = __half_as_ushort(h);
            wq = __half2float(h);
        } else {
            const __nv_bfloat16 h = __float2bfloat16_rn(w * g * sc);
            a.dst[(size_t)dst_row * a.K + k] = __bfloat16_as_ushort(h);
            wq = __bfloat162float(h);
        }
        sum_w += (double)wq;
        shift += (double)bt * (double)w;
    }
    __shared__ double red[2][32];
    for (int o = 16; o > 0; o >>= 1) {
        sum_w += __shfl_xor_sync(0xffffffffu, sum_w, o);
        shift += __shfl_xor_sync(0xffffffffu, shift, o);
    }
    if ((tid & 31) == 0) {
        red[0][tid >> 5] = sum_w;
        red[1][tid >> 5] = shift;
    }
    __syncthreads();
    if (tid == 0) {
        double s0 = 0.0, s1 = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            s0 += red[0][w];
            s1 += red[1][w];
        }
        const double bias = a.bias ? (double)load_as_f32(a.bias, r, a.src_bf16) : 0.0;
        const double sc = a.scale == 0.f ? 1.0 : (double)a.scale;
        a.sum_out[(size_t)r * a.out_stride] = (float)s0;          // already the sum of the scaled row
        a.shift_out[(size_t)r * a.out_stride] = (float)((s1 + bias) * sc);
    }
}

cudaError_t fold_launch(const FoldArgs &a, cudaStream_t stream) {
    fold_kernel<<<a.R, 128, 0, stream>>>(a);
    return cudaGetLastError();
}

__global__ void to_f32_kernel(const void *src, int src_bf16, float *dst, int R, int K, int transpose) {
    const long long n = (long long)R * K;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i / K), k = (int)(i % K);
        const float v = load_as_f32(src, (int)i, src_bf16);
        if (transpose) dst[(long long)k * R + r] = v;
        else dst[i] = v;
    }
}

cudaError_t to_f32_launch(const void *src, int src_bf16, float *dst, int R, int K, int transpose,
                          cudaStream_t stream) {
    const long long n = (long long)R * K;
    const int blocks = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    to_f32_kernel<<<blocks > 0 ? blocks : 1, 256, 0, stream>>>(src, src_bf16, dst, R, K, transpose);
    return cudaGetLastError();
}

}  // namespace trimul
