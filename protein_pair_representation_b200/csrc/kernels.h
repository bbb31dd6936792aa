// kernels.h -- launch interface between the host-side C ABI and the CUDA kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace trimul {

constexpr int kHidden = 128;  // c_h of the tensor-core path

// ---- bf16 tensor-core path ---------------------------------------------------------

struct K1Args {
    CUtensorMap tm_z;      // z: c_z = 128: {64 ch, N*N, 2 halves, B}, box {64, 64, 2, 1}; c_z = 384:
                           // [B][N*N][c_z], box {64, 128, 1}; bf16, 128B swizzle
    CUtensorMap tm_w;      // packed weights [4*c_h][c_z] bf16, box {64, NCOL}, 128B swizzle
    CUtensorMap tm_a;      // a [B][c_h][N*N] f16; c_z = 128: box {64, 128, 1} 128B swizzle,
                           // c_z = 384: box {128, channels per warpgroup, 1} no swizzle
    CUtensorMap tm_b;      // b, same as tm_a
    const uint16_t *mask;  // [B][N*N] bf16 bits, or nullptr
    const float4 *vec;     // [2][c_h] {sum W'_gate, shift_gate, sum W'_proj, shift_proj}
    int B, N;
    long long NN;
    int tiles_per_batch;   // ceil(NN / k1_tile_pairs(c_z))
    float eps;
    const int *ext;        // mask extents [B][2] {R_b, C_b} (tiles wholly beyond them skipped), or nullptr
    uint64_t rowdiv;       // multiplier dividing by N / 8 (div_by_magic)
    unsigned long long *acc;   // per batch element kAccStride entries (below): sums and counts added
                               // with integer atomics (order-independent); nullptr: not gathered
};

// The channel sums behind the offset of the stored x (K1Args::acc), per batch element:
// [c_h sums of a | c_h sums of b | sampled | all | rows], the sums in fixed point (x kAccScale)
// over a sample of the pairs, then the counts of unmasked pairs in the sample, of all unmasked
// pairs, and of rows whose first pair is unmasked. The stride is fixed by c_h = kHidden.
constexpr float kAccScale = 256.0f;
constexpr int kAccSampled = 2 * kHidden, kAccAll = 2 * kHidden + 1, kAccRows = 2 * kHidden + 2;
constexpr int kAccStride = 2 * kHidden + 3;

struct K2Args {
    CUtensorMap tm_a, tm_b, tm_x;
    int BC, N;
    int m_tiles, n_tiles, k_chunks;
    bool incoming;
    bool f16;              // operands and result in fp16 (else bf16)
    float x_scale;         // result = x_scale * sum_k ...
    const int *ext;        // mask extents [B][2] {R_b, C_b}, or nullptr: the sum runs over k < C_b
                           // (outgoing) or k < R_b (incoming); output tiles at rows >= R_b or
                           // columns >= C_b are not written (the output kernel never reads them)
    int C;                 // channels per batch element (bc / C = batch element)
    const float *xoff;     // offset q subtracted after the scaling, before the rounding:
                           // x = round(x_scale * sum - xoff[bc * xoff_stride])
    int xoff_stride;       // 1, or 0 with xoff pointing at a single zero
};

// The contraction for one shard of a row-sharded update. The N x N planes of a and b are
// split by rows over G shards, shard g holding rows [row0[g], row0[g + 1]) of every plane
// ([B*c_h][rows][N], its own buffer: a local copy or another GPU's memory); this shard's
// output rows are x[., i0 + i, .] for i < R (base.m_tiles covers R, base.tm_x is [B*c_h][R][N]).
//   outgoing: x_ij = sum_k a_ik b_jk   A = this shard's a rows (base.tm_a), B rows j from their shards
//   incoming: x_ij = sum_k a_ki b_kj   A columns i and B rows k, both from the shard holding row k
// Every shard boundary is a multiple of 128 rows, so a 128-row box never spans two shards.
constexpr int kMaxShards = 8;
struct K2ShardArgs {
    K2Args base;
    CUtensorMap tm_sa[kMaxShards];   // incoming: shard g's a, {N, R_g, B*c_h}, box {64, 64, 1}
    CUtensorMap tm_sb[kMaxShards];   // shard g's b: outgoing box {64, 128, 1}, incoming box {64, 64, 1}
    int row0[kMaxShards + 1];
    int G;
    int i0;                          // first global row of this shard's output
};

struct K3Args {
    CUtensorMap tm_x;      // x [B][c_h][N*N] f16, box {64, 64, 1}, 128B swizzle (MN-major A)
    CUtensorMap tm_z;      // z [B][N*N][c_z] bf16, box {64, 128, 1}, 128B swizzle
    CUtensorMap tm_wo;     // folded W_o [c_z][c_h] f16, box {64, 128}
    CUtensorMap tm_wg;     // folded W_g [c_z][c_z] bf16, box {64, 128}
    CUtensorMap tm_out;    // out [B][N*N][c_z] f32 (box {32,128,1}) or bf16 (box {64,128,1})
    const uint16_t *mask;
    const float4 *vec;     // [c_z] {sum W_o', shift_o, sum W_g', shift_g}
    int B, N;
    long long NN;
    int tiles_per_batch;
    float eps;             // input LayerNorm
    float eps_x;           // output LayerNorm on the stored (scaled) x: eps * x_scale^2
    const uint16_t *zres;  // residual: z (bf16, [B][N*N][c_z]) added to the output; null = none
    const int *ext;        // mask extents (as K1Args); ignored with a residual (masked pairs then copy z)
    uint64_t rowdiv;
};

// Launch with programmatic stream serialization: the kernel may begin while the previous
// kernel of the stream finishes; every kernel launched this way calls pdl_wait() before it
// touches memory the previous kernel may write or read.
template <typename Kernel, typename Args>
inline cudaError_t launch_pdl(Kernel kernel, int grid, int block, size_t smem, cudaStream_t stream,
                              const Args &args, int cluster = 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster > 1) {      // clusters of `cluster` consecutive CTAs (grid a multiple of it)
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, kernel, args);
}

// Kernel resource queries (dynamic shared memory bytes) and launches.
size_t k1_smem_bytes(int c_z);
int k1_groups(int c_z);
int k1_ncol(int c_z);
int k1_channels_per_warpgroup(int c_z);
cudaError_t k1_launch(int c_z, const K1Args &args, int grid, cudaStream_t stream);
int k1_row_mode(int c_z);
int k1_tile_pairs(int c_z);        // pairs per K1 tile (128; at c_z = 128 a CTA pair's, 64 from each CTA)

size_t k2_smem_bytes();
cudaError_t k2_launch(const K2Args &args, int grid, cudaStream_t stream);
cudaError_t k2_shard_launch(const K2ShardArgs &args, int grid, cudaStream_t stream);

// The fused pair transition (c = 128, hidden 256): out = z + m * (relu(z W1^T + b1) W2^T + b2).
struct PtArgs {
    CUtensorMap tm_z;      // z [B][N*N][128] bf16 viewed {64 ch, N*N, 2 halves, B}, box {64, 64, 2, 1}, 128B swizzle
    CUtensorMap tm_w1;     // W1 [256][128] bf16, box {64, 256}, 128B swizzle
    CUtensorMap tm_w2;     // W2 [128][256] f16, box {64, 128}, 128B swizzle
    CUtensorMap tm_out;    // out [B][N*N][128] f32 or bf16, box {128, 32, 1}, no swizzle
    const uint16_t *z;     // the same z, bf16 bits, for the residual
    const uint16_t *mask;  // [B][N*N] bf16 bits, or nullptr
    const float *b1;       // [256] fp32 (zeros when the layer has no bias)
    const float *b2;       // [128] fp32
    int B;
    long long NN;
    int tiles_per_batch;   // NN / 64
};
cudaError_t pt_launch(bool out_f32, const PtArgs &args, int grid, cudaStream_t stream);
cudaError_t bf16_to_f16_launch(const void *src, void *dst, long long n, cudaStream_t stream);
size_t pt_smem_bytes(bool out_f32);

// Mask extents {R_b, C_b} into ext[2B] (zeroed first), for a bf16 mask [B][N*N]; rowdiv
// divides by N / 8 (host_rowdiv).
cudaError_t mask_extents_launch(const uint16_t *mask, int B, int N, uint64_t rowdiv, int *ext, cudaStream_t stream);

// Multiplier for div_by_magic dividing by d >= 1, or 0 for d = 1: floor((2^64 - 1) / d) + 1,
// which is floor(2^64 / d) + 1 when d does not divide 2^64 and exactly 2^64 / d when it does
// (then the division is exact outright).
inline uint64_t host_rowdiv(uint64_t d) { return d <= 1 ? 0 : ~0ull / d + 1; }

size_t k3_smem_bytes(int c_z, bool out_f32);
int k3_groups(int c_z);
cudaError_t k3_launch(int c_z, bool out_f32, const K3Args &args, int grid, cudaStream_t stream);  // residual iff args.zres

// The offset of the stored x of each batch element from K1's sums, written to all c_h entries
// q[b][c]: x_scale * L * (1 / c_h) sum_c mean(a_c) mean(b_c), rounded to an fp16 value (the means
// over the sampled unmasked pairs, L = all / rows the estimated contraction length; 0 without
// sampled pairs); the sums are zeroed for the next forward. One CTA per batch element.
cudaError_t xoffsets_launch(unsigned long long *acc, int B, int c_h, float x_scale, float *q, cudaStream_t stream);

// ---- weight folding (layer creation) -----------------------------------------------

struct FoldArgs {
    const void *w;        // source [R][K]
    const void *gamma;    // [K] or nullptr (= 1)
    const void *beta;     // [K] or nullptr (= 0)
    const void *bias;     // [R] or nullptr (= 0)
    int src_bf16;         // storage type of w / gamma / beta / bias
    int R, K;
    uint16_t *dst;        // bf16 (or f16 when dst_f16) rows [*, K]
    int dst_f16;
    int row_mode;         // 0: dst row = r; 1: K1 interleaved layout (c_z = 384); 2: K1 blocked layout (c_z = 128)
    int operand;          // row_mode 1: 0 = a, 1 = b
    int kind;             // row_mode 1: 0 = gate, 1 = projection
    int ncol, cpg, gpo;   // row_mode 1: group width, channels per group, groups per operand
    float scale;          // multiplies the folded row, its sum and its shift (1 = none; powers of two are exact)
    float *sum_out;       // element r * stride: sum_k bf16(W[r,k] * gamma[k])
    float *shift_out;     // element r * stride: sum_k beta[k] W[r,k] + bias[r]
    int out_stride;       // in floats
};
cudaError_t fold_launch(const FoldArgs &a, cudaStream_t stream);

// Convert n values (bf16 or f32) to f32; optional transpose of an [R][K] matrix.
cudaError_t to_f32_launch(const void *src, int src_bf16, float *dst, int R, int K, int transpose,
                          cudaStream_t stream);

// ---- fp32 SIMT path ----------------------------------------------------------------

struct F32Weights {
    const float *ln_in_g, *ln_in_b;
    const float *w_ag, *b_ag, *w_ap, *b_ap, *w_bg, *b_bg, *w_bp, *b_bp;
    const float *w_gT, *b_g;      // W_g transposed: [c_z (in)][c_z (out)]
    const float *ln_out_g, *ln_out_b;
    const float *w_oT, *b_o;      // W_o transposed: [c_h (in)][c_z (out)]
};

cudaError_t f32_project_launch(const float *z, const float *mask, const F32Weights &w, int c_z,
                               int c_h, int B, int N, float eps, float *a, float *b,
                               cudaStream_t stream);
cudaError_t f32_contract_launch(const float *a, const float *b, float *x, int BC, int N,
                                bool incoming, float x_scale, cudaStream_t stream);
cudaError_t f32_output_launch(const float *z, const float *mask, const float *x,
                              const F32Weights &w, int c_z, int c_h, int B, int N, float eps,
                              float eps_x, bool residual, float *out, cudaStream_t stream);

}  // namespace trimul
