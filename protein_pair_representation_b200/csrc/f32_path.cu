// f32_path.cu -- the fp32 path (CUDA cores, fp32 FMA, no TF32).
//
// Same three steps as the tensor-core path, written for exactness rather than
// speed: the LayerNorms are applied explicitly (two-pass mean / variance), the
// gates use the accurate expf, and every dot product accumulates in fp32. This is
// the strict-FP32 mode the pages validate against ("RFProteina architecture",
// section "Measured results": parity measured with TF32 disabled).
#include "kernels.h"

namespace trimul {

namespace f32 {
constexpr int TP = 32;        // pairs per block
constexpr int THREADS = 256;

__device__ __forceinline__ float sigmoid_acc(float v) { return 1.0f / (1.0f + expf(-v)); }

__device__ __forceinline__ float warp_sum(float v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// LayerNorm of `rows` rows of `C` floats in shared memory (row stride `ld`), in place,
// one warp per row.
__device__ void layernorm_rows(float *buf, int rows, int C, int ld, const float *gamma, const float *beta,
                               float eps) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < rows; r += THREADS / 32) {
        float *x = buf + r * ld;
        float s = 0.f;
        for (int c = lane; c < C; c += 32) s += x[c];
        const float mean = warp_sum(s) / (float)C;
        float v = 0.f;
        for (int c = lane; c < C; c += 32) {
            const float d = x[c] - mean;
            v = fmaf(d, d, v);
        }
        const float rstd = 1.0f / sqrtf(warp_sum(v) / (float)C + eps);
        for (int c = lane; c < C; c += 32) {
            const float g = gamma ? gamma[c] : 1.f, bb = beta ? beta[c] : 0.f;
            x[c] = (x[c] - mean) * rstd * g + bb;
        }
    }
}
}  // namespace f32

__global__ void __launch_bounds__(f32::THREADS) f32_project_kernel(const float *z, const float *mask, F32Weights w,
                                                                   int c_z, int c_h, long long NN, float eps,
                                                                   float *a, float *b) {
    using namespace f32;
    extern __shared__ float zs[];  // [TP][c_z + 1]
    const int ld = c_z + 1;
    const long long tiles_per_batch = NN / TP;
    const int bb = (int)(blockIdx.x / tiles_per_batch);
    const long long p0 = (blockIdx.x % tiles_per_batch) * TP;
    const float *zt = z + ((long long)bb * NN + p0) * c_z;
    for (int i = threadIdx.x; i < TP * c_z; i += THREADS) zs[(i / c_z) * ld + (i % c_z)] = zt[i];
    __syncthreads();
    layernorm_rows(zs, TP, c_z, ld, w.ln_in_g, w.ln_in_b, eps);
    __syncthreads();

    const int pl = threadIdx.x & 31;        // pair within tile
    const int cg = threadIdx.x >> 5;        // channel phase
    const float m = mask ? mask[(long long)bb * NN + p0 + pl] : 1.f;
    const float *zr = zs + pl * ld;
    for (int c = cg; c < c_h; c += THREADS / 32) {
        const float *wag = w.w_ag + (long long)c * c_z, *wap = w.w_ap + (long long)c * c_z;
        const float *wbg = w.w_bg + (long long)c * c_z, *wbp = w.w_bp + (long long)c * c_z;
        float ag = 0.f, ap = 0.f, bg = 0.f, bp = 0.f;
        for (int k = 0; k < c_z; ++k) {
            const float zk = zr[k];
            ag = fmaf(zk, __ldg(wag + k), ag);
            ap = fmaf(zk, __ldg(wap + k), ap);
            bg = fmaf(zk, __ldg(wbg + k), bg);
            bp = fmaf(zk, __ldg(wbp + k), bp);
        }
        if (w.b_ag) ag += w.b_ag[c];
        if (w.b_ap) ap += w.b_ap[c];
        if (w.b_bg) bg += w.b_bg[c];
        if (w.b_bp) bp += w.b_bp[c];
        const long long o = ((long long)bb * c_h + c) * NN + p0 + pl;
        a[o] = m * sigmoid_acc(ag) * ap;
        b[o] = m * sigmoid_acc(bg) * bp;
    }
}

__global__ void __launch_bounds__(256) f32_contract_kernel(const float *a, const float *b, float *x, int N,
                                                           int incoming, float x_scale) {
    __shared__ float As[16][64 + 4];
    __shared__ float Bs[16][64 + 4];
    const int c = blockIdx.z;
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    const long long plane = (long long)N * N;
    const float *A = a + c * plane, *B = b + c * plane;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < N; k0 += 16) {
        for (int e = tid; e < 16 * 64; e += 256) {
            int kk, ii;
            if (!incoming) { ii = e / 16; kk = e % 16; }   // read along k (contiguous)
            else { kk = e / 64; ii = e % 64; }             // read along i / j (contiguous)
            const int k = k0 + kk, i = i0 + ii, j = j0 + ii;
            float va = 0.f, vb = 0.f;
            if (k < N && i < N) va = incoming ? A[(long long)k * N + i] : A[(long long)i * N + k];
            if (k < N && j < N) vb = incoming ? B[(long long)k * N + j] : B[(long long)j * N + k];
            As[kk][ii] = va;
            Bs[kk][ii] = vb;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float ra[4], rb[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ra[u] = As[kk][ty * 4 + u];
                rb[u] = Bs[kk][tx * 4 + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(ra[u], rb[v], acc[u][v]);
        }
        __syncthreads();
    }
    for (int u = 0; u < 4; ++u)
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + ty * 4 + u, j = j0 + tx * 4 + v;
            if (i < N && j < N) x[c * plane + (long long)i * N + j] = acc[u][v] * x_scale;
        }
}

__global__ void __launch_bounds__(f32::THREADS) f32_output_kernel(const float *z, const float *mask, const float *x,
                                                                  F32Weights w, int c_z, int c_h, long long NN,
                                                                  float eps, float eps_x, int residual, float *out) {
    using namespace f32;
    extern __shared__ float sm[];
    const int ldz = c_z + 1, ldx = c_h + 1;
    float *zs = sm;                 // [TP][c_z + 1]
    float *xs = sm + TP * ldz;      // [TP][c_h + 1]
    const long long tiles_per_batch = NN / TP;
    const int bb = (int)(blockIdx.x / tiles_per_batch);
    const long long p0 = (blockIdx.x % tiles_per_batch) * TP;
    const float *zt = z + ((long long)bb * NN + p0) * c_z;
    for (int i = threadIdx.x; i < TP * c_z; i += THREADS) zs[(i / c_z) * ldz + (i % c_z)] = zt[i];
    for (int i = threadIdx.x; i < TP * c_h; i += THREADS) {
        const int c = i / TP, pl = i % TP;
        xs[pl * ldx + c] = x[((long long)bb * c_h + c) * NN + p0 + pl];
    }
    __syncthreads();
    layernorm_rows(zs, TP, c_z, ldz, w.ln_in_g, w.ln_in_b, eps);
    layernorm_rows(xs, TP, c_h, ldx, w.ln_out_g, w.ln_out_b, eps_x);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PPW = TP / (THREADS / 32);   // pairs per warp = 4
    for (int n = lane; n < c_z; n += 32) {
        float g[PPW] = {}, o[PPW] = {};
        for (int k = 0; k < c_z; ++k) {
            const float wv = __ldg(w.w_gT + (long long)k * c_z + n);
#pragma unroll
            for (int q = 0; q < PPW; ++q) g[q] = fmaf(zs[(warp * PPW + q) * ldz + k], wv, g[q]);
        }
        for (int c = 0; c < c_h; ++c) {
            const float wv = __ldg(w.w_oT + (long long)c * c_z + n);
#pragma unroll
            for (int q = 0; q < PPW; ++q) o[q] = fmaf(xs[(warp * PPW + q) * ldx + c], wv, o[q]);
        }
        const float bg = w.b_g ? w.b_g[n] : 0.f, bo = w.b_o ? w.b_o[n] : 0.f;
#pragma unroll
        for (int q = 0; q < PPW; ++q) {
            const long long pi = p0 + warp * PPW + q;
            const float m = mask ? mask[(long long)bb * NN + pi] : 1.f;
            const long long oi = ((long long)bb * NN + pi) * c_z + n;
            const float u = m * sigmoid_acc(g[q] + bg) * (o[q] + bo);
            out[oi] = residual ? __fadd_rn(z[oi], u) : u;   // no FMA contraction: z + (rounded update)
        }
    }
}

cudaError_t f32_project_launch(const float *z, const float *mask, const F32Weights &w, int c_z, int c_h, int B,
                               int N, float eps, float *a, float *b, cudaStream_t stream) {
    const long long NN = (long long)N * N;
    const size_t smem = (size_t)f32::TP * (c_z + 1) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(f32_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const long long blocks = (long long)B * (NN / f32::TP);
    f32_project_kernel<<<(unsigned)blocks, f32::THREADS, smem, stream>>>(z, mask, w, c_z, c_h, NN, eps, a, b);
    return cudaGetLastError();
}

cudaError_t f32_contract_launch(const float *a, const float *b, float *x, int BC, int N, bool incoming,
                                float x_scale, cudaStream_t stream) {
    dim3 grid((N + 63) / 64, (N + 63) / 64, BC);
    f32_contract_kernel<<<grid, 256, 0, stream>>>(a, b, x, N, incoming ? 1 : 0, x_scale);
    return cudaGetLastError();
}

cudaError_t f32_output_launch(const float *z, const float *mask, const float *x, const F32Weights &w, int c_z,
                              int c_h, int B, int N, float eps, float eps_x, bool residual, float *out,
                              cudaStream_t stream) {
    const long long NN = (long long)N * N;
    const size_t smem = (size_t)f32::TP * ((c_z + 1) + (c_h + 1)) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(f32_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const long long blocks = (long long)B * (NN / f32::TP);
    f32_output_kernel<<<(unsigned)blocks, f32::THREADS, smem, stream>>>(z, mask, x, w, c_z, c_h, NN, eps, eps_x,
                                                                        residual ? 1 : 0, out);
    return cudaGetLastError();
}

}  // namespace trimul
