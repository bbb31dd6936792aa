// k1_project.cu -- K1, the input LayerNorm + gated projection on tensor cores (sm_100a).
//
// Computes, for every pair p = (b, i, j) and hidden channel c,
//   a[b, c, i, j] = m_p * sigmoid(zhat_p . W_ag[c] + b_ag[c]) * (zhat_p . W_ap[c] + b_ap[c])
// and b likewise (stored as fp16), with zhat_p = LayerNorm(z_p) ("RFProteina architecture", section
// "Dual-GEMM gates": the one-input gate that reads the normalized pair tensor,
// applies the mask and emits its output transposed for the contraction; section
// "Triangle multiplication on SM90": K1 with the input LayerNorm folded into its
// weights).
//
// LayerNorm folding: with W' = W * gamma (per input column, rounded to bf16),
//   zhat . W = rstd_p * (z_p . W' - mean_p * sum_k W'_k) + (sum_k beta_k W_k + bias)
// so the tensor cores multiply the raw bf16 z tile, and the epilogue applies the
// per-pair (mean, rstd) and the per-channel (sum W', shift) pair of constants.
//
// Two kernels. c_z = 128 (k1_project_cm_kernel, further below) puts one hidden channel
// on each TMEM lane. c_z = 384 (k1_project_kernel) puts one pair on each TMEM lane:
// 128 consecutive pairs of one batch element times NCOL = 128 packed weight rows, laid
// out in 32-row blocks of [16 gate rows, 16 projection rows] for 16 channels so one
// 32-column TMEM load gives a thread both factors of 16 outputs, with four column groups
// (two per operand) so each group's weights stay resident in shared memory. A CTA keeps
// one group for its whole life (the grid is a multiple of the group count).
//
// Warps: 0-7 epilogue (two warpgroups, half the columns each), 8-11 LayerNorm
// statistics (one thread per pair), 12 TMA producer, 13 TMEM allocator + MMA issuer.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

template <int CZ>
struct K1Cfg {
    static constexpr int C_H = kHidden;
    static constexpr int NCOL = (CZ == 128) ? 256 : 128;
    static constexpr int KC = CZ / 64;                 // 64-channel chunks of z per tile
    static constexpr int CPG = NCOL / 2;               // output channels per group
    static constexpr int G = 4 * C_H / NCOL;           // groups
    static constexpr int GPO = G / 2;                  // groups per operand
    static constexpr int NB = 512 / NCOL;              // TMEM accumulator buffers
    static constexpr int CH_WG = CPG / 2;              // channels per epilogue warpgroup
    static constexpr int BLK_WG = CH_WG / 16;          // 32-column blocks per warpgroup
    static constexpr int W_BYTES = NCOL * CZ * 2;
    static constexpr int CHUNK = 128 * 64 * 2;         // one z chunk: 128 pairs x 64 channels
    static constexpr int STG_BYTES = CH_WG * 128 * 2;  // per warpgroup: [channels][128 pairs] bf16
    static constexpr int SNB = 2;                      // stats ring depth
    static constexpr int FIXED = 1024 + W_BYTES + 2 * STG_BYTES + SNB * 128 * 16 + 1024;
    static constexpr int S = (232448 - FIXED) / CHUNK > 8 ? 8 : (232448 - FIXED) / CHUNK;
    static constexpr size_t SMEM = FIXED + (size_t)S * CHUNK;
    static constexpr int THREADS = 448;
    static constexpr int TMA_WARP = 12, MMA_WARP = 13;
};

struct K1Smem {
    uint64_t wbar;
    uint64_t full[8], empty[8];
    uint64_t tfull[4], tempty[4];
    uint64_t sfull[4], sempty[4];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// SKIP: the instance that leaves out wholly masked tiles (p.ext set); the other one carries
// none of that code.
template <int CZ, bool SKIP>
__global__ void __launch_bounds__(448, 1) k1_project_kernel(const __grid_constant__ K1Args p) {
    using C = K1Cfg<CZ>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *w_s = base;                                   // KC chunks of [NCOL][64] bf16
    uint8_t *chunks = w_s + C::W_BYTES;                    // S chunks of [128][64] bf16
    uint8_t *staging = chunks + C::S * C::CHUNK;           // 2 x [CH_WG][128] bf16
    float4 *stats = reinterpret_cast<float4 *>(staging + 2 * C::STG_BYTES);  // [SNB][128]
    K1Smem &s = *reinterpret_cast<K1Smem *>(stats + C::SNB * 128);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;

    const int group = blockIdx.x % C::G;
    const int cta_in_group = blockIdx.x / C::G;
    const int ctas_per_group = gridDim.x / C::G;
    const int num_ptiles = p.B * p.tiles_per_batch;
    const int operand = group / C::GPO;
    const int ch0 = (group % C::GPO) * C::CPG;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        for (int i = 0; i < C::S; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + 4);  // MMA commit + 4 stats warps
        }
        for (int i = 0; i < C::NB; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 8);
        }
        for (int i = 0; i < C::SNB; ++i) {
            mbar_init(&s.sfull[i], 4);
            mbar_init(&s.sempty[i], 8);
        }
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(&s.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    pdl_launch_dependents();
    if (warp != C::TMA_WARP) pdl_wait();       // the producer waits after its weight loads

    if (warp == C::TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_z);
            tma_prefetch_desc(&p.tm_w);
            // resident weights of this CTA's group
            mbar_arrive_expect_tx(&s.wbar, C::W_BYTES);
            for (int kc = 0; kc < C::KC; ++kc)
                tma_load_2d(w_s + kc * C::NCOL * 128, &p.tm_w, &s.wbar, kc * 64, group * C::NCOL);
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;
            TileWalk tw(cta_in_group, p.tiles_per_batch);
            for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
                const int b = tw.b;
                const int p0 = tw.t * 128;
                if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;   // nothing to load
                for (int kc = 0; kc < C::KC; ++kc) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                    mbar_arrive_expect_tx(&s.full[stage], C::CHUNK);
                    tma_load_3d(chunks + stage * C::CHUNK, &p.tm_z, &s.full[stage], kc * 64, p0, b);
                    ++filled;
                    if (++stage == C::S) { stage = 0; phase ^= 1; }
                }
            }
            goto producer_done;
        producer_abort:
            for (uint32_t i = 0; i < (filled < (uint32_t)C::S ? filled : (uint32_t)C::S); ++i) {
                uint32_t f = filled - 1 - i;
                mbar_drain(&s.full[f % C::S], (f / C::S) & 1);
            }
        producer_done:
            mbar_drain(&s.wbar, 0);
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(128, C::NCOL, false, false, false);
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma);
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            TileWalk tw(cta_in_group, p.tiles_per_batch);
            for (int pt = cta_in_group; ok && pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
                if (SKIP && tile_masked_out(p.ext, tw.b, tw.t * 128, p.N, p.NN, p.rowdiv)) continue;
                if (!mbar_wait(&s.tempty[abuf], aphase ^ 1, abort_flag, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + abuf * C::NCOL;
                for (int kc = 0; kc < C::KC; ++kc) {
                    if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t *za = chunks + stage * C::CHUNK;
                    const uint8_t *wb = w_s + kc * C::NCOL * 128;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        uint64_t ad = smem_desc_sw128(za + kk * 32, 16, 1024);
                        uint64_t bd = smem_desc_sw128(wb + kk * 32, 16, 1024);
                        tc_mma_bf16(d_tmem, ad, bd, idesc, (kc | kk) != 0);
                    }
                    tc_commit(&s.empty[stage]);
                    if (++stage == C::S) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(&s.tfull[abuf]);
                if (++abuf == C::NB) { abuf = 0; aphase ^= 1; }
            }
            tc_commit(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else if (warp >= 8) {
        // LayerNorm statistics: thread = pair row of the tile
        const int row = (warp - 8) * 32 + lane;
        int stage = 0;
        uint32_t phase = 0;
        int sbuf = 0;
        uint32_t sphase = 0;
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
            // shifted sums in packed pairs: s1 = sum(v - shift), s2 = sum((v - shift)^2), with
            // the row's first entry as the shift
            float shift = 0.f;
            float2 nsh = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
            bool ok = true;
            for (int kc = 0; kc < C::KC; ++kc) {
                if (!__all_sync(0xffffffffu, mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutEpilogue))) { ok = false; break; }
                const uint8_t *zc = chunks + stage * C::CHUNK;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(zc + sw128_offset(row, u));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                    if (kc == 0 && u == 0) {
                        shift = bf16_lo(w.x);
                        nsh = make_float2(-shift, -shift);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 d = f2_add(make_float2(bf16_lo(ws[e]), bf16_hi(ws[e])), nsh);
                        s1 = f2_add(s1, d);
                        s2 = f2_fma(d, d, s2);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.empty[stage]);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            const float inv_n = 1.0f / (float)CZ;
            const float dm = (s1.x + s1.y) * inv_n;
            const float var = fmaxf((s2.x + s2.y) * inv_n - dm * dm, 0.f);
            const float mean = shift + dm;
            const float rstd = rsqrtf(var + p.eps);
            const long long pi = (long long)p0 + row;
            float m = 1.f;
            if (p.mask) m = (pi < p.NN) ? __uint_as_float((uint32_t)p.mask[(long long)b * p.NN + pi] << 16) : 0.f;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sempty[sbuf], sphase ^ 1, abort_flag, kErrTimeoutEpilogue))) break;
            stats[sbuf * 128 + row] = make_float4(mean, rstd, m, 0.f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sfull[sbuf]);
            if (++sbuf == C::SNB) { sbuf = 0; sphase ^= 1; }
        }
    } else {
        // epilogue: warpgroup wg handles channels [ch0 + wg*CH_WG, +CH_WG)
        const int wg = warp >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;
        uint16_t *stg = reinterpret_cast<uint16_t *>(staging + wg * C::STG_BYTES);
        const bool leader = (threadIdx.x & 127) == 0;
        const CUtensorMap *tm_out = operand == 0 ? &p.tm_a : &p.tm_b;
        const float4 *vec = p.vec + operand * C::C_H + ch0 + wg * C::CH_WG;
        int abuf = 0;
        uint32_t aphase = 0;
        int sbuf = 0;
        uint32_t sphase = 0;
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) {
                // every pair of the tile is masked: a and b are 0 there (the contraction reads them)
                if (leader) tma_store_wait_read<0>();
                named_bar_sync(1 + wg, 128);
                for (int ch = 0; ch < C::CH_WG; ++ch) stg[ch * 128 + row] = 0;
                fence_proxy_async_smem();
                named_bar_sync(1 + wg, 128);
                if (leader) {
                    tma_store_3d(tm_out, stg, p0, ch0 + wg * C::CH_WG, b);
                    tma_store_commit();
                }
                continue;
            }
            if (!group_all(mbar_wait(&s.sfull[sbuf], sphase, abort_flag, kErrTimeoutEpilogue), 1 + wg, 128)) break;
            const float4 st = stats[sbuf * 128 + row];
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sempty[sbuf]);
            if (++sbuf == C::SNB) { sbuf = 0; sphase ^= 1; }
            const float mean = st.x, rstd = st.y, m = st.z;

            if (!group_all(mbar_wait(&s.tfull[abuf], aphase, abort_flag, kErrTimeoutEpilogue), 1 + wg, 128)) break;
            tc_fence_after();
            if (leader) tma_store_wait_read<0>();
            named_bar_sync(1 + wg, 128);
#pragma unroll 1
            for (int blk = 0; blk < C::BLK_WG; ++blk) {
                float v[32];
                tmem_ld32(tmem_base + abuf * C::NCOL + ((uint32_t)(q * 32) << 16) + (wg * C::BLK_WG + blk) * 32, v);
                tc_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 cv = __ldg(&vec[blk * 16 + e]);
                    const float g = fmaf(rstd, fmaf(-mean, cv.x, v[e]), cv.y);
                    const float pr = fmaf(rstd, fmaf(-mean, cv.z, v[16 + e]), cv.w);
                    const float out = sigmoid_tanh(g) * pr * m;
                    stg[(blk * 16 + e) * 128 + row] = __half_as_ushort(__float2half_rn(out));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.tempty[abuf]);
            if (++abuf == C::NB) { abuf = 0; aphase ^= 1; }
            fence_proxy_async_smem();
            named_bar_sync(1 + wg, 128);
            if (leader) {
                tma_store_3d(tm_out, stg, p0, ch0 + wg * C::CH_WG, b);
                tma_store_commit();
            }
        }
        if (leader) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ------------------------------------------------------------------------------------------
// K1 for c_z = 128: accumulators with one TMEM lane per hidden channel.
//
// D_gate[c, p] = W'_gate[c] . z_p and D_proj[c, p] = W'_proj[c] . z_p for the 128 channels
// of one operand (a or b) and 128 pairs: A = folded weights [128 channels x c_z], B = the z
// tile [128 pairs x c_z], both K-major. A thread of the epilogue owns one channel for the
// whole kernel, so that channel's four folding constants stay in registers; the per-pair
// LayerNorm statistics are read from shared memory (broadcast, four pairs per load); and
// consecutive pairs of one channel are consecutive columns, which pack directly into
// 16-byte rows of the channel-major output tile.
// The gate is evaluated in f16x2 (tanh.approx.f16x2 on g/2, the gate rows being folded
// with an extra factor 1/2), as are the products with the projection and the mask.
// Warps: 0-15 epilogue (two teams of two warpgroups that take alternate tiles; warpgroup
// s of a team: pairs [64s, 64s+64) of its tiles), 16-19 LayerNorm statistics, 20 TMA
// producer, 21 TMEM allocator + MMA issuer.
struct K1CmCfg {
    static constexpr int CZ = 128, C_H = kHidden, KC = CZ / 64;
    static constexpr int G = 2;                               // one group per operand
    static constexpr int W_CHUNK = 2 * C_H * 64 * 2;          // [gate 128 rows, proj 128 rows] x 64 k
    static constexpr int W_BYTES = KC * W_CHUNK;              // 64 KB
    static constexpr int CHUNK = 128 * 64 * 2;                // z chunk: 128 pairs x 64 channels
    static constexpr int WARP_STG = 32 * 32 * 2;              // per epilogue warp: [32 ch][32 pairs] f16
    static constexpr int STG_TOTAL = 16 * WARP_STG;           // 32 KB for the 16 epilogue warps
    static constexpr int SNB = 2;
    static constexpr int STATS_BYTES = SNB * 128 * (4 + 4 + 2);   // mean, rstd (f32), mask (f16) per pair
    static constexpr int FIXED = 1024 + W_BYTES + STG_TOTAL + STATS_BYTES + 1024;
    static constexpr int S = (232448 - FIXED) / CHUNK > 8 ? 8 : (232448 - FIXED) / CHUNK;
    static constexpr size_t SMEM = FIXED + (size_t)S * CHUNK;
    static constexpr int EPI_WARPS = 16;                      // four warpgroups, 32 pairs each
    static constexpr int STATS_WARP0 = 16, STATS_WARPS = 4;
    static constexpr int TMA_WARP = 20, MMA_WARP = 21;
    static constexpr int THREADS = 22 * 32;
};

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// tanh of two halves at once (hardware approximation).
__device__ __forceinline__ __half2 tanh_h2(__half2 x) {
    uint32_t t;
    asm("tanh.approx.f16x2 %0, %1;" : "=r"(t) : "r"(h2_as_u32(x)));
    return u32_as_h2(t);
}

template <bool SKIP>
__global__ void __launch_bounds__(K1CmCfg::THREADS, 1) k1_project_cm_kernel(const __grid_constant__ K1Args p) {
    using C = K1CmCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *w_s = base;                                  // KC chunks of [256 rows][64] bf16
    uint8_t *chunks = w_s + C::W_BYTES;                   // S chunks of [128 pairs][64] bf16
    uint8_t *staging = chunks + C::S * C::CHUNK;          // 16 x [32 ch][32 pairs] f16, 64B swizzle
    float *st_nmean = reinterpret_cast<float *>(staging + C::STG_TOTAL);     // [SNB][128] -mean
    float *st_rstd = st_nmean + C::SNB * 128;
    __half *st_hmask = reinterpret_cast<__half *>(st_rstd + C::SNB * 128);    // [SNB][128] mask / 2
    K1Smem &s = *reinterpret_cast<K1Smem *>(st_hmask + C::SNB * 128);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;

    const int operand = blockIdx.x % C::G;
    const int cta_in_group = blockIdx.x / C::G;
    const int ctas_per_group = gridDim.x / C::G;
    const int num_ptiles = p.B * p.tiles_per_batch;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        for (int i = 0; i < C::S; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + C::STATS_WARPS);  // MMA commit + stats warps
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], C::EPI_WARPS / 2);     // the team that drains buffer i
        }
        for (int i = 0; i < C::SNB; ++i) {
            mbar_init(&s.sfull[i], C::STATS_WARPS);
            mbar_init(&s.sempty[i], C::EPI_WARPS / 2);
        }
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(&s.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    pdl_launch_dependents();
    if (warp != C::TMA_WARP) pdl_wait();       // the producer waits after its weight loads

    if (warp == C::TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_z);
            tma_prefetch_desc(&p.tm_w);
            mbar_arrive_expect_tx(&s.wbar, C::W_BYTES);
            for (int kc = 0; kc < C::KC; ++kc)
                tma_load_2d(w_s + kc * C::W_CHUNK, &p.tm_w, &s.wbar, kc * 64, operand * 2 * C::C_H);
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;
            TileWalk tw(cta_in_group, p.tiles_per_batch);
            for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
                const int b = tw.b;
                const int p0 = tw.t * 128;
                if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;   // nothing to load
                for (int kc = 0; kc < C::KC; ++kc) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                    mbar_arrive_expect_tx(&s.full[stage], C::CHUNK);
                    tma_load_3d(chunks + stage * C::CHUNK, &p.tm_z, &s.full[stage], kc * 64, p0, b);
                    ++filled;
                    if (++stage == C::S) { stage = 0; phase ^= 1; }
                }
            }
            goto producer_done;
        producer_abort:
            for (uint32_t i = 0; i < (filled < (uint32_t)C::S ? filled : (uint32_t)C::S); ++i) {
                uint32_t f = filled - 1 - i;
                mbar_drain(&s.full[f % C::S], (f / C::S) & 1);
            }
        producer_done:
            mbar_drain(&s.wbar, 0);
        }
    } else if (warp == C::MMA_WARP) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(128, 128, false, false, false);
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t aphase[2] = {0, 0};           // tile j of this CTA uses TMEM buffer j % 2
            int j = 0;
            TileWalk tw(cta_in_group, p.tiles_per_batch);
            for (int pt = cta_in_group; ok && pt < num_ptiles;
                 pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch), ++j) {
                if (SKIP && tile_masked_out(p.ext, tw.b, tw.t * 128, p.N, p.NN, p.rowdiv)) continue;
                const int abuf = j & 1;
                if (!mbar_wait(&s.tempty[abuf], aphase[abuf] ^ 1, abort_flag, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint32_t d_gate = tmem_base + abuf * 256;
                const uint32_t d_proj = d_gate + 128;
                for (int kc = 0; kc < C::KC; ++kc) {
                    if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t *zc = chunks + stage * C::CHUNK;
                    const uint8_t *wg = w_s + kc * C::W_CHUNK;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = smem_desc_sw128(zc + kk * 32, 16, 1024);
                        const uint64_t ag = smem_desc_sw128(wg + kk * 32, 16, 1024);
                        const uint64_t ap = smem_desc_sw128(wg + C::C_H * 128 + kk * 32, 16, 1024);
                        tc_mma_bf16(d_gate, ag, bd, idesc, (kc | kk) != 0);
                        tc_mma_bf16(d_proj, ap, bd, idesc, (kc | kk) != 0);
                    }
                    tc_commit(&s.empty[stage]);
                    if (++stage == C::S) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(&s.tfull[abuf]);
                aphase[abuf] ^= 1;
            }
            tc_commit(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else if (warp >= C::STATS_WARP0) {
        // LayerNorm statistics: thread = pair row of the tile
        const int row = (warp - C::STATS_WARP0) * 32 + lane;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t sphase[2] = {0, 0};               // tile j of this CTA uses statistics buffer j % 2
        int j = -1;
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            ++j;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
            const int sbuf = j & 1;
            const long long pi = (long long)p0 + row;
            uint16_t mbits = 0x3F80u;   // bf16 1.0; the load is issued first so its latency overlaps
            if (p.mask) mbits = (pi < p.NN) ? p.mask[(long long)b * p.NN + pi] : (uint16_t)0;
            // shifted sums in packed pairs: s1 = sum(v - shift), s2 = sum((v - shift)^2), with
            // the row's first entry as the shift
            float shift = 0.f;
            float2 nsh = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
            bool ok = true;
            for (int kc = 0; kc < C::KC; ++kc) {
                if (!__all_sync(0xffffffffu, mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutEpilogue))) { ok = false; break; }
                const uint8_t *zc = chunks + stage * C::CHUNK;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(zc + sw128_offset(row, u));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                    if (kc == 0 && u == 0) {
                        shift = bf16_lo(w.x);
                        nsh = make_float2(-shift, -shift);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 d = f2_add(make_float2(bf16_lo(ws[e]), bf16_hi(ws[e])), nsh);
                        s1 = f2_add(s1, d);
                        s2 = f2_fma(d, d, s2);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.empty[stage]);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            const float inv_n = 1.0f / (float)C::CZ;
            const float dm = (s1.x + s1.y) * inv_n;
            const float var = fmaxf((s2.x + s2.y) * inv_n - dm * dm, 0.f);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sempty[sbuf], sphase[sbuf] ^ 1, abort_flag, kErrTimeoutEpilogue))) break;
            st_nmean[sbuf * 128 + row] = -(shift + dm);
            st_rstd[sbuf * 128 + row] = rsqrtf(var + p.eps);
            st_hmask[sbuf * 128 + row] = __float2half_rn(0.5f * __uint_as_float((uint32_t)mbits << 16));
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sfull[sbuf]);
            sphase[sbuf] ^= 1;
        }
    } else {
        // epilogue: two teams of eight warps take alternate tiles of this CTA's sequence (team k
        // drains TMEM buffer k and statistics buffer k), so that one team's waits and TMEM
        // loads overlap the other team's arithmetic. Thread = hidden channel c; warpgroup s of
        // a team owns the 64 pairs [64 s, 64 s + 64) of its tiles. Every warp runs on its own:
        // it waits on the barriers itself and stages each [32 channels][32 pairs] block of its
        // output in its own 2 KB of shared memory (64-byte rows, 64-byte swizzle) for a TMA
        // store.
        const int wg = warp >> 2;
        const int team = wg >> 1;
        const int q = warp & 3;
        const int c = q * 32 + lane;
        const int col0 = 64 * (wg & 1);
        uint8_t *stg = staging + warp * C::WARP_STG;
        const CUtensorMap *tm_out = operand == 0 ? &p.tm_a : &p.tm_b;
        // {sum W'_gate, shift_gate, sum W'_proj, shift_proj}; the gate entries are for g / 2
        const float4 cv = p.vec[operand * C::C_H + c];
        const float2 cg_sum = make_float2(cv.x, cv.x), cg_shift = make_float2(cv.y, cv.y);
        const float2 cp_sum = make_float2(cv.z, cv.z), cp_shift = make_float2(cv.w, cv.w);
        static_assert(C::SNB == 2, "one statistics buffer per epilogue team");
        const int abuf = team, sbuf = team;
        const uint32_t tbase = tmem_base + abuf * 256 + ((uint32_t)(q * 32) << 16);
        const float *snmean0 = st_nmean + sbuf * 128 + col0, *srstd0 = st_rstd + sbuf * 128 + col0;
        const __half *shmask0 = st_hmask + sbuf * 128 + col0;
        uint32_t phase = 0;
        const int first = cta_in_group + team * ctas_per_group;
        TileWalk tw(first, p.tiles_per_batch);
        for (int pt = first; pt < num_ptiles; pt += 2 * ctas_per_group, tw.advance(2 * ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) {
                // every pair of the tile is masked: a and b are 0 there (the contraction reads them)
#pragma unroll 1
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = col0 + 32 * blk;
                    if (lane == 0) tma_store_wait_read<0>();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4 *>(stg + sw64_offset(lane, u)) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && p0 + col < p.NN) {
                        tma_store_3d(tm_out, stg, p0 + col, q * 32, b);
                        tma_store_commit();
                    }
                }
                continue;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sfull[sbuf], phase, abort_flag, kErrTimeoutEpilogue) &&
                                             mbar_wait(&s.tfull[abuf], phase, abort_flag, kErrTimeoutEpilogue)))
                break;
            tc_fence_after();
#pragma unroll 1
            for (int blk = 0; blk < 2; ++blk) {         // two store blocks of 32 pairs
                const int col = col0 + 32 * blk;
                if (lane == 0) tma_store_wait_read<0>();   // this warp's previous store has read its block
                __syncwarp();
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {      // two halves of 16 pairs
                    float g[16], pr[16];
                    tmem_ld16(tbase + col + 16 * hh, g);
                    tmem_ld16(tbase + 128 + col + 16 * hh, pr);
                    tc_wait_ld();
                    if (blk == 1 && hh == 1) {
                        // the last TMEM load of the tile has landed: hand the buffer back to the
                        // MMA now, not after this warp's arithmetic and store
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&s.tempty[abuf]);
                    }
                    const int o = 32 * blk + 16 * hh;
                    uint32_t outw[8];
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        const float4 nm = *reinterpret_cast<const float4 *>(snmean0 + o + j);
                        const float4 rs = *reinterpret_cast<const float4 *>(srstd0 + o + j);
                        const uint2 mk = *reinterpret_cast<const uint2 *>(shmask0 + o + j);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            // two consecutive pairs of this channel in one packed lane pair
                            const float2 nm2 = h == 0 ? make_float2(nm.x, nm.y) : make_float2(nm.z, nm.w);
                            const float2 rs2 = h == 0 ? make_float2(rs.x, rs.y) : make_float2(rs.z, rs.w);
                            const float2 gv = f2_fma(rs2, f2_fma(nm2, cg_sum, make_float2(g[j + 2 * h], g[j + 2 * h + 1])), cg_shift);
                            const float2 pv = f2_fma(rs2, f2_fma(nm2, cp_sum, make_float2(pr[j + 2 * h], pr[j + 2 * h + 1])), cp_shift);
                            // mask * sigmoid(2 x) = (mask / 2) tanh(x) + mask / 2, x being the halved gate
                            const __half2 hm = u32_as_h2(h == 0 ? mk.x : mk.y);
                            const __half2 gm = __hfma2(tanh_h2(__floats2half2_rn(gv.x, gv.y)), hm, hm);
                            outw[j / 2 + h] = h2_as_u32(__hmul2(gm, __floats2half2_rn(pv.x, pv.y)));
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        *reinterpret_cast<uint4 *>(stg + sw64_offset(lane, 2 * hh + u)) =
                            make_uint4(outw[4 * u], outw[4 * u + 1], outw[4 * u + 2], outw[4 * u + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (blk == 1) mbar_arrive(&s.sempty[sbuf]);   // statistics read in full
                    if (p0 + col < p.NN) {              // blocks wholly past the last pair are not stored
                        tma_store_3d(tm_out, stg, p0 + col, q * 32, b);
                        tma_store_commit();
                    }
                }
            }
            phase ^= 1;
        }
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

int k1_ncol(int c_z) { return c_z == 128 ? 2 * K1CmCfg::C_H : K1Cfg<384>::NCOL; }
int k1_groups(int c_z) { return c_z == 128 ? K1CmCfg::G : K1Cfg<384>::G; }
int k1_channels_per_warpgroup(int c_z) { return c_z == 128 ? K1CmCfg::C_H : K1Cfg<384>::CH_WG; }
int k1_row_mode(int c_z) { return c_z == 128 ? 2 : 1; }
size_t k1_smem_bytes(int c_z) { return c_z == 128 ? K1CmCfg::SMEM : K1Cfg<384>::SMEM; }

template <int CZ, bool SKIP>
static cudaError_t k1_launch_t(const K1Args &args, int grid, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k1_project_kernel<CZ, SKIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1Cfg<CZ>::SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return launch_pdl(k1_project_kernel<CZ, SKIP>, grid, K1Cfg<CZ>::THREADS, K1Cfg<CZ>::SMEM, stream, args);
}

template <bool SKIP>
static cudaError_t k1_launch_cm(const K1Args &args, int grid, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k1_project_cm_kernel<SKIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1CmCfg::SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return launch_pdl(k1_project_cm_kernel<SKIP>, grid, K1CmCfg::THREADS, K1CmCfg::SMEM, stream, args);
}

cudaError_t k1_launch(int c_z, const K1Args &args, int grid, cudaStream_t stream) {
    const bool skip = args.ext != nullptr;
    if (c_z == 128) return skip ? k1_launch_cm<true>(args, grid, stream) : k1_launch_cm<false>(args, grid, stream);
    if (c_z == 384) return skip ? k1_launch_t<384, true>(args, grid, stream) : k1_launch_t<384, false>(args, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace trimul
