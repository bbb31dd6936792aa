// transition.cu -- the fused pair transition on tensor cores (sm_100a).
//
//   out_ij = z_ij + m_ij * (relu(z_ij . W1^T + b1) . W2^T + b2)
//
// for c = 128 and hidden width 2c = 256 ("RFProteina architecture", section "Kernel support":
// one launch runs both linears, the ReLU, the mask and the residual and keeps the hidden
// activation on chip; the released pair width takes an expansion of 2).
//
// Channel-lane accumulators over 64-pair tiles:
//   GEMM1  D1[h, p] = W1[h] . z_p           A = W1 (K-major, two M=128 halves), B = z tile (K-major)
//   WG0    H[h, p] = f16(relu(D1 + b1))     written to shared memory as GEMM2's MN-major B operand
//   GEMM2  D2[n, p] = W2[n] . H[:, p]       A = W2 in f16 (K-major, K = 256), B = H
// (f16 rather than bf16 for the on-chip activation: 11 significant bits instead of 8 at the
// same tensor-core rate; both operands of an MMA share the type, so W2 is kept in f16 too, an
// exact copy of the bf16 weights except below 2^-14 in magnitude, where the absolute error is
// under 2^-25.)
//   WG1    out[p, n] = z[p, n] + m_p (D2 + b2[n]), rows of 128 channels through TMA stores
// Warps: 0-7 the hidden activation (warpgroup k: hidden half k), 8-15 the output (warpgroup k:
// pairs [32k, 32k + 32), its own staging and store), 16 TMA producer, 17 TMEM and MMA issuer.
// TMEM: two buffers of [D1: 128 columns | D2: 64 columns]. H is single-buffered: the MMA thread
// issues GEMM1 of tile t+1 before GEMM2 of tile t, so the activation warpgroups work on the next
// tile while the output warpgroups write this one. A z tile is released as soon as GEMM1 has
// read it, so the input ring runs ahead of the whole pipeline. The output warpgroups take the
// residual from global memory (L2: GEMM1's copy has just brought it in), one tile ahead, as
// 16-byte row segments: thread = channel puts m_p (D2 + b2) in fp32 staging rows, then thread =
// row segment adds z and rounds in place.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

namespace pt {
constexpr int C = 128, HID = 256, TP = 64;                 // channels, hidden units, pairs per tile
constexpr int W1_BYTES = HID * C * 2;                      // 64 KB: 2 K-chunks of [256 rows][64]
constexpr int W2_BYTES = C * HID * 2;                      // 64 KB: 4 K-chunks of [128 rows][64]
constexpr int ZT_BYTES = TP * C * 2;                       // 16 KB: [2 halves][64 pairs][64 ch]
constexpr int H_BYTES = HID * TP * 2;                      // 32 KB: [256 rows][64 pairs]
constexpr int OUT_ROWS = 32;                               // pairs per output warpgroup
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 576;
constexpr int TMA_WARP = 16, MMA_WARP = 17;
constexpr int SMAX = 2;                                    // z tiles in flight (each freed by GEMM1)

struct Smem {
    uint64_t wbar;
    uint64_t zfull[SMAX], zempty[SMAX];
    uint64_t d1full[2], d1empty[2];
    uint64_t d2full[2], d2empty[2];
    uint64_t hfull, hempty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

template <bool OUT_F32>
struct Cfg {
    static constexpr int S = SMAX;
    static constexpr int STG_BYTES = OUT_ROWS * C * 4;     // per output warpgroup: [32 pairs][128] fp32
    static constexpr size_t SMEM = 1024 + W1_BYTES + W2_BYTES + S * ZT_BYTES + H_BYTES + 2 * STG_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory");
};
}  // namespace pt

template <bool OUT_F32>
__global__ void __launch_bounds__(pt::THREADS, 1) pair_transition_kernel(const __grid_constant__ PtArgs p) {
    using namespace pt;
    constexpr int S = Cfg<OUT_F32>::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *w1_s = base;
    uint8_t *w2_s = w1_s + W1_BYTES;
    uint8_t *zt = w2_s + W2_BYTES;                         // S z tiles
    uint8_t *h_s = zt + S * ZT_BYTES;                      // hidden activation (GEMM2's B)
    uint8_t *stg0 = h_s + H_BYTES;                         // output rows, one block per output warpgroup
    Smem &s = *reinterpret_cast<Smem *>(stg0 + 2 * Cfg<OUT_F32>::STG_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;
    const int num_tiles = p.B * p.tiles_per_batch;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        for (int i = 0; i < S; ++i) {
            mbar_init(&s.zfull[i], 1);
            mbar_init(&s.zempty[i], 1);                    // GEMM1's commit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.d1full[i], 1);
            mbar_init(&s.d1empty[i], 8);                   // activation warps
            mbar_init(&s.d2full[i], 1);
            mbar_init(&s.d2empty[i], 8);                   // output warps
        }
        mbar_init(&s.hfull, 8);                            // activation warps
        mbar_init(&s.hempty, 1);                           // GEMM2's commit
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(&s.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    pdl_launch_dependents();
    if (warp != TMA_WARP) pdl_wait();

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_z);
            mbar_arrive_expect_tx(&s.wbar, W1_BYTES + W2_BYTES);
            for (int kc = 0; kc < C / 64; ++kc) tma_load_2d(w1_s + kc * (HID * 128), &p.tm_w1, &s.wbar, kc * 64, 0);
            for (int kc = 0; kc < HID / 64; ++kc) tma_load_2d(w2_s + kc * (C * 128), &p.tm_w2, &s.wbar, kc * 64, 0);
            pdl_wait();
            int st = 0;
            uint32_t ph = 0;
            uint32_t filled = 0;
            TileWalk tw(blockIdx.x, p.tiles_per_batch);
            for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tw.advance(gridDim.x, p.tiles_per_batch)) {
                if (!mbar_wait(&s.zempty[st], ph ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                mbar_arrive_expect_tx(&s.zfull[st], ZT_BYTES);
                // both 64-channel halves of 64 pairs: [half][pair][64 channels]
                tma_load_4d(zt + st * ZT_BYTES, &p.tm_z, &s.zfull[st], 0, tw.t * TP, 0, tw.b);
                ++filled;
                if (++st == S) { st = 0; ph ^= 1; }
            }
            goto producer_done;
        producer_abort:
            for (uint32_t i = 0; i < (filled < (uint32_t)S ? filled : (uint32_t)S); ++i) {
                const uint32_t f = filled - 1 - i;
                mbar_drain(&s.zfull[f % S], (f / S) & 1);
            }
        producer_done:
            mbar_drain(&s.wbar, 0);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            const uint32_t idesc1 = idesc_f32acc(128, TP, false, false, false);   // W1 . z^T
            const uint32_t idesc2 = idesc_f32acc(128, TP, false, true, true);     // f16 W2 . f16 H (H MN-major)
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma);
            // GEMM1 of the CTA's tile j; false after an abort
            auto gemm1 = [&](int j) -> bool {
                const int st = j % S;
                const int u = j & 1;
                if (!mbar_wait(&s.zfull[st], (uint32_t)(j / S) & 1, abort_flag, kErrTimeoutMma)) return false;
                if (!mbar_wait(&s.d1empty[u], ((uint32_t)(j >> 1) & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
                tc_fence_after();
                const uint8_t *zb = zt + st * ZT_BYTES;
#pragma unroll
                for (int h = 0; h < 2; ++h) {                      // hidden units [128 h, 128 h + 128)
                    const uint32_t d = tmem_base + u * 192 + h * 64;
#pragma unroll
                    for (int kc = 0; kc < 2; ++kc)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = smem_desc_sw128(w1_s + kc * (HID * 128) + h * (128 * 128) + kk * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(zb + kc * (TP * 128) + kk * 32, 16, 1024);
                            tc_mma_bf16(d, ad, bd, idesc1, (kc | kk) != 0);
                        }
                }
                tc_commit(&s.d1full[u]);
                tc_commit(&s.zempty[st]);                            // GEMM1 has read the z tile
                return true;
            };
            // GEMM2 of the CTA's tile j (H of tile j in shared memory)
            auto gemm2 = [&](int j) -> bool {
                const int u = j & 1;
                if (!mbar_wait(&s.hfull, (uint32_t)j & 1, abort_flag, kErrTimeoutMma)) return false;
                if (!mbar_wait(&s.d2empty[u], ((uint32_t)(j >> 1) & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
                tc_fence_after();
                const uint32_t d = tmem_base + u * 192 + 128;
#pragma unroll
                for (int kc = 0; kc < HID / 64; ++kc)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc_sw128(w2_s + kc * (C * 128) + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(h_s + kc * 8192 + kk * 2048, 8192, 1024);
                        tc_mma_bf16(d, ad, bd, idesc2, (kc | kk) != 0);
                    }
                tc_commit(&s.d2full[u]);
                tc_commit(&s.hempty);                                // GEMM2 has read H
                return true;
            };
            const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
            if (ok && my_tiles > 0) ok = gemm1(0);
            for (int j = 0; ok && j < my_tiles; ++j) {
                if (j + 1 < my_tiles && !gemm1(j + 1)) break;
                if (!gemm2(j)) break;
            }
            tc_commit(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else if (warp < 8) {
        // activation warpgroup hf: H[h, p] = f16(relu(D1[h, p] + b1[h])) for the hidden units
        // h = 128 hf + r of its half; thread = TMEM lane r
        const int hf = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t bar_id = 1 + hf;
        const float bh = p.b1[hf * 128 + r];
        const int row = hf * 128 + r;                          // K index of GEMM2 = hidden unit
        const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        for (int j = 0; j < my_tiles; ++j) {
            const int u = j & 1;
            if (!group_all(mbar_wait(&s.d1full[u], (uint32_t)(j >> 1) & 1, abort_flag, kErrTimeoutEpilogue), bar_id, 128)) break;
            // GEMM2 of the previous tile has read H
            if (!group_all(mbar_wait(&s.hempty, ((uint32_t)j & 1) ^ 1, abort_flag, kErrTimeoutEpilogue), bar_id, 128)) break;
            tc_fence_after();
            float v0[32], v1[32];                              // pairs 0-31 and 32-63
            tmem_ld32(tmem_base + u * 192 + hf * 64 + lane_off, v0);
            tmem_ld32(tmem_base + u * 192 + hf * 64 + lane_off + 32, v1);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.d1empty[u]);         // D1 read in full
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {                   // 8 pairs per 16-byte unit
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 8 * (uu & 3) + 2 * e;
                    const float a0 = uu < 4 ? v0[i] : v1[i], a1 = uu < 4 ? v0[i + 1] : v1[i + 1];
                    w[e] = pack_f16x2(fmaxf(a0 + bh, 0.f), fmaxf(a1 + bh, 0.f));
                }
                *reinterpret_cast<uint4 *>(h_s + sw128_offset(row, uu)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();                          // H is read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.hfull);
        }
    } else if (warp < 16) {
        // output warpgroup k: out[p, n] = z[p, n] + m_p (D2[n, p] + b2[n]) for the pairs
        // [32k, 32k + 32) of the tile. Phase 1, thread = output channel n: m_p (D2 + b2[n]) into
        // the fp32 staging rows. Phase 2, thread = 8-channel row segments (4 of the block's 512):
        // + z, rounded to the output type, in place.
        const int k = (warp - 8) >> 2;
        const int q = warp & 3;
        const int n = q * 32 + lane;
        const int tk = q * 32 + lane;                          // thread index within the warpgroup
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t bar_id = 3 + k;
        const bool leader = tk == 0;
        float *stg = reinterpret_cast<float *>(stg0 + k * Cfg<OUT_F32>::STG_BYTES);
        const float bias = p.b2[n];
        constexpr int SEGS = OUT_ROWS * C / 8 / 128;           // row segments per thread
        // segment r of this thread: pair tk / 16 + 8 r of the block, channels 8 (tk % 16) + 0..7
        const int seg_pair = tk >> 4, seg_ch = (tk & 15) * 8;
        auto load_residual = [&](const TileWalk &w, uint4 (&dst)[SEGS]) {
            const uint16_t *src = p.z + ((long long)w.b * p.NN + w.t * TP + k * OUT_ROWS + seg_pair) * C + seg_ch;
#pragma unroll
            for (int r = 0; r < SEGS; ++r) dst[r] = __ldg(reinterpret_cast<const uint4 *>(src + r * 8 * C));
        };
        int j = 0;
        TileWalk tw(blockIdx.x, p.tiles_per_batch);
        // one tile ahead: lane l of every warp holds the mask of pair 32k + l (bf16 bits), and
        // zn the residual segments
        uint32_t mbits = 0x3F80u;
        uint4 zn[SEGS];
        if (blockIdx.x < num_tiles) {
            if (p.mask) mbits = p.mask[(long long)tw.b * p.NN + tw.t * TP + k * OUT_ROWS + lane];
            load_residual(tw, zn);
        }
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tw.advance(gridDim.x, p.tiles_per_batch), ++j) {
            const int b = tw.b;
            const int u = j & 1;
            const float mreg = __uint_as_float(mbits << 16);
            uint4 zc[SEGS];
#pragma unroll
            for (int r = 0; r < SEGS; ++r) zc[r] = zn[r];
            uint32_t mbits_next = 0x3F80u;
            if (t + (int)gridDim.x < num_tiles) {
                TileWalk tn = tw;
                tn.advance(gridDim.x, p.tiles_per_batch);
                if (p.mask) mbits_next = p.mask[(long long)tn.b * p.NN + tn.t * TP + k * OUT_ROWS + lane];
                load_residual(tn, zn);
            }
            if (leader) tma_store_wait_read<0>();              // this warpgroup's previous store has read its rows
            if (!group_all(mbar_wait(&s.d2full[u], (uint32_t)(j >> 1) & 1, abort_flag, kErrTimeoutEpilogue), bar_id, 128)) break;
            tc_fence_after();
            float d[32];
            tmem_ld32(tmem_base + u * 192 + 128 + lane_off + k * OUT_ROWS, d);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.d2empty[u]);
#pragma unroll
            for (int pp = 0; pp < OUT_ROWS; ++pp) stg[pp * C + n] = __shfl_sync(0xffffffffu, mreg, pp) * (d[pp] + bias);
            named_bar_sync(bar_id, 128);
            float v[SEGS][8];
#pragma unroll
            for (int r = 0; r < SEGS; ++r) {
                const float4 *src = reinterpret_cast<const float4 *>(stg + (seg_pair + 8 * r) * C + seg_ch);
                const float4 lo = src[0], hi = src[1];
                const uint32_t zw[4] = {zc[r].x, zc[r].y, zc[r].z, zc[r].w};
                const float f[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[r][2 * e] = f[2 * e] + __uint_as_float(zw[e] << 16);
                    v[r][2 * e + 1] = f[2 * e + 1] + __uint_as_float(zw[e] & 0xFFFF0000u);
                }
            }
            if (OUT_F32) {
#pragma unroll
                for (int r = 0; r < SEGS; ++r) {               // the same addresses this thread read
                    float4 *dst = reinterpret_cast<float4 *>(stg + (seg_pair + 8 * r) * C + seg_ch);
                    dst[0] = make_float4(v[r][0], v[r][1], v[r][2], v[r][3]);
                    dst[1] = make_float4(v[r][4], v[r][5], v[r][6], v[r][7]);
                }
            } else {
                named_bar_sync(bar_id, 128);                   // every fp32 row is read before bf16 rows overwrite them
                uint16_t *ob = reinterpret_cast<uint16_t *>(stg);
#pragma unroll
                for (int r = 0; r < SEGS; ++r)
                    *reinterpret_cast<uint4 *>(ob + (seg_pair + 8 * r) * C + seg_ch) =
                        make_uint4(pack_bf16x2(v[r][0], v[r][1]), pack_bf16x2(v[r][2], v[r][3]),
                                   pack_bf16x2(v[r][4], v[r][5]), pack_bf16x2(v[r][6], v[r][7]));
            }
            fence_proxy_async_smem();
            named_bar_sync(bar_id, 128);
            if (leader) {
                tma_store_3d(&p.tm_out, stg, 0, tw.t * TP + k * OUT_ROWS, b);
                tma_store_commit();
            }
            mbits = mbits_next;
        }
        if (leader) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

__global__ void bf16_to_f16_kernel(const uint16_t *src, __half *dst, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        dst[i] = __float2half_rn(__uint_as_float((uint32_t)src[i] << 16));
}

cudaError_t bf16_to_f16_launch(const void *src, void *dst, long long n, cudaStream_t stream) {
    const long long blocks = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
    bf16_to_f16_kernel<<<(unsigned)(blocks > 0 ? blocks : 1), 256, 0, stream>>>(reinterpret_cast<const uint16_t *>(src),
                                                                                reinterpret_cast<__half *>(dst), n);
    return cudaGetLastError();
}

size_t pt_smem_bytes(bool out_f32) { return out_f32 ? pt::Cfg<true>::SMEM : pt::Cfg<false>::SMEM; }

template <bool F32>
static cudaError_t pt_launch_t(const PtArgs &args, int grid, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(pair_transition_kernel<F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)pt::Cfg<F32>::SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return launch_pdl(pair_transition_kernel<F32>, grid, pt::THREADS, pt::Cfg<F32>::SMEM, stream, args);
}

cudaError_t pt_launch(bool out_f32, const PtArgs &args, int grid, cudaStream_t stream) {
    return out_f32 ? pt_launch_t<true>(args, grid, stream) : pt_launch_t<false>(args, grid, stream);
}

}  // namespace trimul
