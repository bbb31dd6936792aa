// k3_output.cu -- K3, the output LayerNorm + gated output projection on tensor cores.
//
// For every pair p and output channel n:
//   out[p, n] = m_p * sigmoid(zhat_p . W_g[n] + b_g[n]) * (LN(x_p) . W_o[n] + b_o[n])
// with zhat_p = LayerNorm_{c_z}(z_p) and LN(x_p) the LayerNorm over the c_h channels of
// the contracted x (stored fp16, scaled by x_scale) ("RFProteina architecture", section "Dual-GEMM gates": the two-input
// gate with x0 the normalized input pair tensor and x1 the contracted hidden tensor;
// section "Triangle multiplication on SM90": K3 with both LayerNorms folded into its
// weights). Both norms are folded as in K1:
//   x . W_o' -> rstd_x (acc1 - mean_x sum W_o') + shift_o, with W_o' = W_o * gamma_out
// The LayerNorm over c_h ignores a constant added to every channel of a pair, so x may be
// stored less any per-pair constant (the forward stores it less a per-batch-element offset).
//   z . W_g' -> rstd_z (acc2 - mean_z sum W_g') + shift_g, with W_g' = W_g * gamma_in
//
// Tile: 128 consecutive pairs (one TMEM lane each) times 128 output channels. x arrives
// channel-major ([c_h][pairs], pairs contiguous) and is the MN-major A operand of the
// first GEMM; z is channel-last and the K-major A operand of the second. c_z = 384 uses
// three column groups (a CTA keeps one group) so each group's weights stay resident.
//
// Warps: 0-7 epilogue (two warpgroups, 64 output channels each), 8-11 LayerNorm
// statistics of x and 12-15 of z (one thread per pair each), 16 TMA producer, 17 TMEM + MMA.
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

template <int CZ, bool OUT_F32>
struct K3Cfg {
    static constexpr int C_H = kHidden;
    static constexpr int NCOL = 128;                 // output channels per group
    static constexpr int G = CZ / NCOL;
    static constexpr int XC = C_H / 64;              // x chunks per tile (64 channels each)
    static constexpr int ZC = CZ / 64;               // z chunks per tile
    static constexpr int CPT = XC + ZC;              // chunks per tile
    static constexpr int WO_BYTES = NCOL * C_H * 2;
    static constexpr int WG_BYTES = NCOL * CZ * 2;
    static constexpr int CHUNK = 128 * 64 * 2;
    static constexpr int STG_BYTES = 128 * 128;      // per warpgroup and buffer: 128 rows x 128 bytes
    static constexpr int COLS_PER_STORE = OUT_F32 ? 32 : 64;
    // staging buffers per warpgroup: fp32 out takes two stores per tile, and a second buffer
    // lets the second block be written while the first one's store still reads (c_z = 128:
    // c_z = 384 keeps its room for the input ring)
    static constexpr int NSTG = (OUT_F32 && CZ == 128) ? 2 : 1;
    static constexpr int SNB = 2;
    static constexpr int VEC_BYTES = NCOL * 16;          // folding constants of this group's columns
    static constexpr int XPART_BYTES = 4 * 128 * 8;      // x partial sums: [4 warps][128 pairs] float2
    static constexpr int FIXED = 1024 + WO_BYTES + WG_BYTES + 2 * NSTG * STG_BYTES + SNB * 128 * 32 + VEC_BYTES + XPART_BYTES + 1024;
    static constexpr int S = (232448 - FIXED) / CHUNK > 8 ? 8 : (232448 - FIXED) / CHUNK;
    static constexpr size_t SMEM = FIXED + (size_t)S * CHUNK;
    static constexpr int THREADS = 576;
    static constexpr int STATS_WARP0 = 8;
    static constexpr int TMA_WARP = 16, MMA_WARP = 17;
};

struct K3Smem {
    uint64_t wbar;
    uint64_t full[8], empty[8];
    uint64_t tfull[2], tempty[2];
    uint64_t sfull[2], sempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Per-pair values the epilogue needs, in the form it uses them: negated means, the x rstd,
// half the z rstd (the gate is evaluated as tanh of half its argument) and half the mask.
struct K3Stats {
    float nmean_z, hrstd_z, nmean_x, rstd_x, hmask, pad0, pad1, pad2;
};

// RES: out = z + update; SKIP: wholly masked tiles written as zeros without any work (p.ext
// set; never with RES). Instances without them carry none of that code.
template <int CZ, bool OUT_F32, bool RES, bool SKIP>
__global__ void __launch_bounds__(576, 1) k3_output_kernel(const __grid_constant__ K3Args p) {
    using C = K3Cfg<CZ, OUT_F32>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *wo_s = base;                              // XC chunks of [128 rows][64] bf16
    uint8_t *wg_s = wo_s + C::WO_BYTES;                // ZC chunks of [128 rows][64] bf16
    uint8_t *chunks = wg_s + C::WG_BYTES;              // S chunks
    uint8_t *staging = chunks + C::S * C::CHUNK;       // [NSTG][2 warpgroups] x 16 KB
    K3Stats *stats = reinterpret_cast<K3Stats *>(staging + 2 * C::NSTG * C::STG_BYTES);
    // folding constants of this group's columns, one array each: sum W_o', shift_o,
    // sum W_g', shift_g / 2
    float *vec_s = reinterpret_cast<float *>(stats + C::SNB * 128);   // [4][NCOL]
    float2 *xpart = reinterpret_cast<float2 *>(vec_s + 4 * C::NCOL);  // [4][128]
    K3Smem &s = *reinterpret_cast<K3Smem *>(xpart + 4 * 128);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;

    const int group = blockIdx.x % C::G;
    const int cta_in_group = blockIdx.x / C::G;
    const int ctas_per_group = gridDim.x / C::G;
    const int num_ptiles = p.B * p.tiles_per_batch;
    const int n0 = group * C::NCOL;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        for (int i = 0; i < C::S; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + 8);  // MMA commit + both statistics roles
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 8);
        }
        for (int i = 0; i < C::SNB; ++i) {
            mbar_init(&s.sfull[i], 8);     // x and z statistics warps
            mbar_init(&s.sempty[i], 8);
        }
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x < C::NCOL) {
        const float4 v = p.vec[n0 + threadIdx.x];
        vec_s[threadIdx.x] = v.x;
        vec_s[C::NCOL + threadIdx.x] = v.y;
        vec_s[2 * C::NCOL + threadIdx.x] = v.z;
        vec_s[3 * C::NCOL + threadIdx.x] = 0.5f * v.w;
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
            tma_prefetch_desc(&p.tm_x);
            tma_prefetch_desc(&p.tm_z);
            mbar_arrive_expect_tx(&s.wbar, C::WO_BYTES + C::WG_BYTES);
            for (int c = 0; c < C::XC; ++c)
                tma_load_2d(wo_s + c * C::NCOL * 128, &p.tm_wo, &s.wbar, c * 64, n0);
            for (int c = 0; c < C::ZC; ++c)
                tma_load_2d(wg_s + c * C::NCOL * 128, &p.tm_wg, &s.wbar, c * 64, n0);
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;
            TileWalk tw(cta_in_group, p.tiles_per_batch);
            for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
                const int b = tw.b;
                const int p0 = tw.t * 128;
                if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;   // nothing to load
                for (int c = 0; c < C::CPT; ++c) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                    uint8_t *dst = chunks + stage * C::CHUNK;
                    mbar_arrive_expect_tx(&s.full[stage], C::CHUNK);
                    if (c < C::XC) {
                        // x: K = channels c*64..+63 (rows), M = pairs: both 64-pair MN blocks
                        // ([block][channel][64 pairs]) in one copy
                        tma_load_4d(dst, &p.tm_x, &s.full[stage], 0, c * 64, p0 / 64, b);
                    } else {
                        tma_load_3d(dst, &p.tm_z, &s.full[stage], (c - C::XC) * 64, p0, b);
                    }
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
            const uint32_t idesc_x = idesc_f32acc(128, C::NCOL, true, false, true);    // f16 x . f16 W_o'
            const uint32_t idesc_z = idesc_f32acc(128, C::NCOL, false, false, false);  // bf16 z . bf16 W_g'
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
                const uint32_t d1 = tmem_base + abuf * 256;     // x . W_o'
                const uint32_t d2 = d1 + 128;                   // z . W_g'
                for (int c = 0; c < C::CPT; ++c) {
                    if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t *ch = chunks + stage * C::CHUNK;
                    if (c < C::XC) {
                        const uint8_t *wb = wo_s + c * C::NCOL * 128;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            uint64_t ad = smem_desc_sw128(ch + kk * 2048, 8192, 1024);
                            uint64_t bd = smem_desc_sw128(wb + kk * 32, 16, 1024);
                            tc_mma_bf16(d1, ad, bd, idesc_x, (c | kk) != 0);
                        }
                    } else {
                        const int zc = c - C::XC;
                        const uint8_t *wb = wg_s + zc * C::NCOL * 128;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            uint64_t ad = smem_desc_sw128(ch + kk * 32, 16, 1024);
                            uint64_t bd = smem_desc_sw128(wb + kk * 32, 16, 1024);
                            tc_mma_bf16(d2, ad, bd, idesc_z, (zc | kk) != 0);
                        }
                    }
                    tc_commit(&s.empty[stage]);
                    if (++stage == C::S) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(&s.tfull[abuf]);
                if (++abuf == 2) { abuf = 0; aphase ^= 1; }
            }
            tc_commit(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else if (warp >= C::STATS_WARP0) {
        // LayerNorm statistics, one thread per pair `row`: warps 8-11 take x over c_h (from the
        // x chunks), warps 12-15 z over c_z (from the z chunks). Both roles wait for and release
        // every chunk in order (releasing the other role's chunks at once): a role that skipped
        // chunks could run more than a ring ahead of the producer and then match the parity of
        // an older phase of a stage's barrier.
        const bool xrole = warp < C::STATS_WARP0 + 4;
        const int row = ((warp - C::STATS_WARP0) & 3) * 32 + lane;
        const int mblk = row >> 6;         // which 64-pair MN block of an x chunk
        const int r64 = row & 63;
        int stage = 0;
        uint32_t phase = 0;
        int sbuf = 0;
        uint32_t sphase = 0;
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
            const long long pi = (long long)p0 + row;
            uint16_t mbits = 0x3F80u;      // bf16 1.0; issued first so its latency overlaps the sums
            if (!xrole && p.mask) mbits = (pi < p.NN) ? p.mask[(long long)b * p.NN + pi] : (uint16_t)0;
            // shifted sums in packed pairs (shift = the first entry of the row)
            float sh = 0.f;
            float2 nsh = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
            bool ok = true;
            // x role: thread (octet o, group gq) sums the 8 pairs [8o, 8o + 8) over the channels
            // gq, gq + 8, ... of each x chunk from 16-byte rows; the partial sums of the 8 groups
            // of an octet are combined after the chunks (shuffle, then shared memory)
            const int xo = row & 15, xg = row >> 4;
            const uint8_t *xblk_off = nullptr;
            float2 a1[4], a2[4], xnsh[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) a1[k] = a2[k] = xnsh[k] = make_float2(0.f, 0.f);
            for (int c = 0; c < C::CPT; ++c) {
                const bool arrived = mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutEpilogue);
                if (xrole ? !group_all(arrived, 1, 128) : !__all_sync(0xffffffffu, arrived)) { ok = false; break; }
                const uint8_t *ch = chunks + stage * C::CHUNK;
                if (xrole && c < C::XC) {
                    // MN-major: K row kr holds 64 pairs per block; 16-byte unit (xo % 8) of a row
                    // of block xo / 8 holds pairs [8o, 8o + 8), swizzled with the row index
                    xblk_off = ch + (xo >> 3) * 8192;
                    if (c == 0) {
                        const uint4 w0 = *reinterpret_cast<const uint4 *>(xblk_off + sw128_offset(0, xo & 7));
                        const uint32_t h0[4] = {w0.x, w0.y, w0.z, w0.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&h0[k]));
                            xnsh[k] = make_float2(-v.x, -v.y);
                        }
                        // this thread's own pair (`row`) shift, for the final mean
                        sh = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t *>(
                            ch + mblk * 8192 + sw128_offset(0, r64 >> 3) + (r64 & 7) * 2)));
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(xblk_off + sw128_offset(xg + 8 * j, xo & 7));
                        const uint32_t hw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 d = f2_add(__half22float2(*reinterpret_cast<const __half2 *>(&hw[k])), xnsh[k]);
                            a1[k] = f2_add(a1[k], d);
                            a2[k] = f2_fma(d, d, a2[k]);
                        }
                    }
                } else if (!xrole && c >= C::XC) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(ch + sw128_offset(row, u));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                        if (c == C::XC && u == 0) {
                            sh = bf16_lo(w.x);
                            nsh = make_float2(-sh, -sh);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 d = f2_add(make_float2(bf16_lo(ws[e]), bf16_hi(ws[e])), nsh);
                            s1 = f2_add(s1, d);
                            s2 = f2_fma(d, d, s2);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.empty[stage]);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
            }
            if (xrole && ok) {
                // groups 2w and 2w + 1 of an octet sit in lanes o and o + 16 of warp w
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    a1[k].x += __shfl_xor_sync(0xffffffffu, a1[k].x, 16);
                    a1[k].y += __shfl_xor_sync(0xffffffffu, a1[k].y, 16);
                    a2[k].x += __shfl_xor_sync(0xffffffffu, a2[k].x, 16);
                    a2[k].y += __shfl_xor_sync(0xffffffffu, a2[k].y, 16);
                }
                const int xw = warp - C::STATS_WARP0;
                if (lane < 16) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        xpart[xw * 128 + 8 * xo + 2 * k] = make_float2(a1[k].x, a2[k].x);
                        xpart[xw * 128 + 8 * xo + 2 * k + 1] = make_float2(a1[k].y, a2[k].y);
                    }
                }
                named_bar_sync(1, 128);
                float2 t = xpart[row];
#pragma unroll
                for (int w4 = 1; w4 < 4; ++w4) {
                    const float2 u = xpart[w4 * 128 + row];
                    t.x += u.x;
                    t.y += u.y;
                }
                s1 = make_float2(t.x, 0.f);
                s2 = make_float2(t.y, 0.f);
                named_bar_sync(1, 128);   // every partial is read before the next tile's are written
            }
            if (!ok) break;
            const float t1 = s1.x + s1.y, t2 = s2.x + s2.y;
            const float inv_n = 1.0f / (float)(xrole ? C::C_H : CZ);
            const float dm = t1 * inv_n;
            float rs = rsqrtf(fmaxf(t2 * inv_n - dm * dm, 0.f) + (xrole ? p.eps_x : p.eps));
            // every channel of this pair's x holds the same value (the shifted square sum is
            // exactly 0): the normalized vector is exactly 0 whatever the scale, so the x-GEMM's
            // rounding residue in rstd (x . W_o' - mean sum W_o') must not be amplified by 1/sqrt(eps)
            if (xrole && t2 == 0.f) rs = 0.f;
            // an inf or NaN anywhere in this pair's x makes the shifted square sum inf or NaN
            if (xrole && !(fabsf(t2) <= 3.0e38f)) atomicOr(&g_device_error, (unsigned int)kErrRange);
            const bool freed = mbar_wait(&s.sempty[sbuf], sphase ^ 1, abort_flag, kErrTimeoutEpilogue);
            if (xrole ? !group_all(freed, 1, 128) : !__all_sync(0xffffffffu, freed)) break;
            K3Stats &st = stats[sbuf * 128 + row];
            if (xrole) {
                st.nmean_x = -(sh + dm);
                st.rstd_x = rs;
            } else {
                st.nmean_z = -(sh + dm);
                st.hrstd_z = 0.5f * rs;
                st.hmask = 0.5f * __uint_as_float((uint32_t)mbits << 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sfull[sbuf]);
            if (++sbuf == C::SNB) { sbuf = 0; sphase ^= 1; }
        }
    } else {
        // epilogue: warpgroup wg handles output channels n0 + wg*64 .. +63; warp q of it the
        // pairs [32q, 32q + 32) of the tile. Every warp runs on its own: it waits on the
        // barriers itself, stages its 32 pair rows in its own 4 KB of the warpgroup's staging
        // buffer (store block sc in buffer sc % NSTG) and issues the TMA store of that block.
        // With a residual and bf16 out, the residual rows are copied into the staging rows
        // (cp.async) before the accumulators are ready, and the output overwrites them in place.
        const int wg = warp >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const float *v_sum_o = vec_s + wg * 64, *v_shift_o = v_sum_o + C::NCOL;
        const float *v_sum_g = v_sum_o + 2 * C::NCOL, *v_hshift_g = v_sum_o + 3 * C::NCOL;
        int abuf = 0;
        uint32_t aphase = 0;
        int sbuf = 0;
        uint32_t sphase = 0;
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (SKIP && tile_masked_out(p.ext, b, p0, p.N, p.NN, p.rowdiv)) {
                // every pair of the tile is masked: out is 0 there
#pragma unroll 1
                for (int sc = 0; sc < 64 / C::COLS_PER_STORE; ++sc) {
                    uint8_t *stg = staging + ((sc % C::NSTG) * 2 + wg) * C::STG_BYTES;
                    if (lane == 0) tma_store_wait_read<C::NSTG - 1>();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4 *>(stg + sw128_offset(row, u)) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (p0 + q * 32 < p.NN) tma_store_3d(&p.tm_out, stg + q * 32 * 128, n0 + wg * 64 + sc * C::COLS_PER_STORE, p0 + q * 32, b);
                        tma_store_commit();   // a group per block, empty or not
                    }
                }
                continue;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sfull[sbuf], sphase, abort_flag, kErrTimeoutEpilogue))) break;
            const K3Stats st = stats[sbuf * 128 + row];
            const float2 nmx = make_float2(st.nmean_x, st.nmean_x), rx = make_float2(st.rstd_x, st.rstd_x);
            const float2 nmz = make_float2(st.nmean_z, st.nmean_z), hrz = make_float2(st.hrstd_z, st.hrstd_z);
            const float2 hm = make_float2(st.hmask, st.hmask);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sempty[sbuf]);
            if (++sbuf == C::SNB) { sbuf = 0; sphase ^= 1; }

            constexpr bool RES_STAGED = RES && !OUT_F32;
            if (RES_STAGED) {
                // this warp's 32 residual rows (64 channels, 128 bytes each) into its staging
                // rows, 4 rows per instruction; rows past the last pair are zero-filled
                if (lane == 0) tma_store_wait_read<0>();   // the previous tile's store has read them
                __syncwarp();
                uint8_t *stg = staging + wg * C::STG_BYTES;
                const int u = lane & 7;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = q * 32 + 4 * i + (lane >> 3);
                    const bool in = (long long)p0 + r < p.NN;
                    const uint16_t *src = p.zres + (in ? ((long long)b * p.NN + p0 + r) * CZ + n0 + wg * 64 + 8 * u : 0);
                    cp_async_16(stg + sw128_offset(r, u), src, in ? 16u : 0u);
                }
                cp_async_commit();
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&s.tfull[abuf], aphase, abort_flag, kErrTimeoutEpilogue))) break;
            tc_fence_after();
            const uint32_t t1 = tmem_base + abuf * 256 + ((uint32_t)(q * 32) << 16) + wg * 64;
            const uint32_t t2 = t1 + 128;
#pragma unroll 1
            for (int sc = 0; sc < 64 / C::COLS_PER_STORE; ++sc) {
                uint8_t *stg = staging + ((sc % C::NSTG) * 2 + wg) * C::STG_BYTES;
#pragma unroll 1
                for (int h = 0; h < C::COLS_PER_STORE / 32; ++h) {
                    const int col = sc * C::COLS_PER_STORE + h * 32;   // within this warpgroup's 64
                    float o[32], g[32];
                    tmem_ld16(t1 + col, *reinterpret_cast<float(*)[16]>(&o[0]));
                    tmem_ld16(t1 + col + 16, *reinterpret_cast<float(*)[16]>(&o[16]));
                    tmem_ld16(t2 + col, *reinterpret_cast<float(*)[16]>(&g[0]));
                    tmem_ld16(t2 + col + 16, *reinterpret_cast<float(*)[16]>(&g[16]));
                    if (h == 0 && !RES_STAGED) {
                        // the store of this buffer's previous block has read its rows (with two
                        // buffers the store just issued, from the other one, may still read)
                        if (lane == 0) tma_store_wait_read<C::NSTG - 1>();
                        __syncwarp();
                    }
                    tc_wait_ld();
                    if (sc == 64 / C::COLS_PER_STORE - 1 && h == C::COLS_PER_STORE / 32 - 1) {
                        // the last TMEM load of the tile has landed: hand the buffer back to the
                        // MMA now, not after this warp's arithmetic and store
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&s.tempty[abuf]);
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 so = *reinterpret_cast<const float4 *>(v_sum_o + col + e);
                        const float4 ho = *reinterpret_cast<const float4 *>(v_shift_o + col + e);
                        const float4 sg = *reinterpret_cast<const float4 *>(v_sum_g + col + e);
                        const float4 hg = *reinterpret_cast<const float4 *>(v_hshift_g + col + e);
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            // output channels e + 2k and e + 2k + 1 of this pair, packed
                            const float2 so2 = k == 0 ? make_float2(so.x, so.y) : make_float2(so.z, so.w);
                            const float2 ho2 = k == 0 ? make_float2(ho.x, ho.y) : make_float2(ho.z, ho.w);
                            const float2 sg2 = k == 0 ? make_float2(sg.x, sg.y) : make_float2(sg.z, sg.w);
                            const float2 hg2 = k == 0 ? make_float2(hg.x, hg.y) : make_float2(hg.z, hg.w);
                            const int i = e + 2 * k;
                            const float2 ov = f2_fma(rx, f2_fma(nmx, so2, make_float2(o[i], o[i + 1])), ho2);
                            // half the gate argument; mask * sigmoid(2 y) = (mask / 2) tanh(y) + mask / 2
                            const float2 gh = f2_fma(hrz, f2_fma(nmz, sg2, make_float2(g[i], g[i + 1])), hg2);
                            const float2 gm = f2_fma(hm, make_float2(tanh_approx(gh.x), tanh_approx(gh.y)), hm);
                            const float2 r = f2_mul(gm, ov);
                            o[i] = r.x;
                            o[i + 1] = r.y;
                        }
                    }
                    if (RES && OUT_F32 && (long long)p0 + row < p.NN) {
                        // residual: this pair's z at the block's 32 output channels (from L2: K1
                        // and this kernel's own z chunk loads have just read it)
                        const uint4 *zp = reinterpret_cast<const uint4 *>(
                            p.zres + ((long long)b * p.NN + p0 + row) * CZ + n0 + wg * 64 + col);
                        uint4 zr[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) zr[u] = zp[u];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t zw[4] = {zr[u].x, zr[u].y, zr[u].z, zr[u].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                o[8 * u + 2 * e] += bf16_lo(zw[e]);
                                o[8 * u + 2 * e + 1] += bf16_hi(zw[e]);
                            }
                        }
                    }
                    if (OUT_F32) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<float4 *>(stg + sw128_offset(row, u)) =
                                make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
                    } else {
                        if (RES_STAGED) {
                            cp_async_wait_all();
                            __syncwarp();                      // rows copied by the other lanes
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (RES_STAGED) {
                                const uint4 zr = *reinterpret_cast<const uint4 *>(stg + sw128_offset(row, h * 4 + u));
                                const uint32_t zw[4] = {zr.x, zr.y, zr.z, zr.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    o[8 * u + 2 * e] += bf16_lo(zw[e]);
                                    o[8 * u + 2 * e + 1] += bf16_hi(zw[e]);
                                }
                            }
                            uint4 w;
                            w.x = pack_bf16x2(o[8 * u + 0], o[8 * u + 1]);
                            w.y = pack_bf16x2(o[8 * u + 2], o[8 * u + 3]);
                            w.z = pack_bf16x2(o[8 * u + 4], o[8 * u + 5]);
                            w.w = pack_bf16x2(o[8 * u + 6], o[8 * u + 7]);
                            *reinterpret_cast<uint4 *>(stg + sw128_offset(row, h * 4 + u)) = w;
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    // blocks wholly past the last pair are not stored; the group is committed
                    // all the same (empty), so the most recent group is always the last block's
                    if (p0 + q * 32 < p.NN) tma_store_3d(&p.tm_out, stg + q * 32 * 128, n0 + wg * 64 + sc * C::COLS_PER_STORE, p0 + q * 32, b);
                    tma_store_commit();
                }
            }
            if (++abuf == 2) { abuf = 0; aphase ^= 1; }
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

int k3_groups(int c_z) { return c_z / 128; }

size_t k3_smem_bytes(int c_z, bool out_f32) {
    if (c_z == 128) return out_f32 ? K3Cfg<128, true>::SMEM : K3Cfg<128, false>::SMEM;
    return out_f32 ? K3Cfg<384, true>::SMEM : K3Cfg<384, false>::SMEM;
}

template <int CZ, bool F32, bool RES, bool SKIP>
static cudaError_t k3_launch_t(const K3Args &args, int grid, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k3_output_kernel<CZ, F32, RES, SKIP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K3Cfg<CZ, F32>::SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return launch_pdl(k3_output_kernel<CZ, F32, RES, SKIP>, grid, K3Cfg<CZ, F32>::THREADS, K3Cfg<CZ, F32>::SMEM, stream,
                      args);
}

template <int CZ>
static cudaError_t k3_launch_cz(bool out_f32, const K3Args &args, int grid, cudaStream_t stream) {
    if (args.zres)
        return out_f32 ? k3_launch_t<CZ, true, true, false>(args, grid, stream)
                       : k3_launch_t<CZ, false, true, false>(args, grid, stream);
    if (args.ext)
        return out_f32 ? k3_launch_t<CZ, true, false, true>(args, grid, stream)
                       : k3_launch_t<CZ, false, false, true>(args, grid, stream);
    return out_f32 ? k3_launch_t<CZ, true, false, false>(args, grid, stream)
                   : k3_launch_t<CZ, false, false, false>(args, grid, stream);
}

cudaError_t k3_launch(int c_z, bool out_f32, const K3Args &args, int grid, cudaStream_t stream) {
    if (c_z == 128) return k3_launch_cz<128>(out_f32, args, grid, stream);
    if (c_z == 384) return k3_launch_cz<384>(out_f32, args, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace trimul
