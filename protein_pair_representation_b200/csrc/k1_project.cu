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
// Two kernels. c_z = 128 (k1_project_pair_kernel, further below) runs on CTA pairs and puts one
// hidden channel on each TMEM lane. c_z = 384 (k1_project_kernel) puts one pair on each TMEM lane:
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

// Unmasked-pair counts of one batch element for the offset of the stored x (kAccSampled,
// kAccAll and kAccRows entries after the channel sums), kept by one lane per statistics warp and
// added with integer atomics when the batch element changes and at the end.
struct PairCounts {
    int b = -1;
    unsigned int sampled = 0, all = 0, rows = 0;
    __device__ __forceinline__ void flush(unsigned long long *acc) {
        if (b < 0) return;
        unsigned long long *a = acc + (size_t)b * kAccStride;
        atomicAdd(a + kAccSampled, (unsigned long long)sampled);
        atomicAdd(a + kAccAll, (unsigned long long)all);
        atomicAdd(a + kAccRows, (unsigned long long)rows);
    }
    // valid: this lane's pair is unmasked; samp: it is one of the sampled pairs; first: it is the
    // first pair of its row (a padding mask's row is valid iff its first pair is)
    __device__ __forceinline__ void add(unsigned long long *acc, int batch, bool valid, bool samp, bool first, int lane) {
        const unsigned int v = __ballot_sync(0xffffffffu, valid);
        const unsigned int s = __ballot_sync(0xffffffffu, valid && samp);
        const unsigned int f = __ballot_sync(0xffffffffu, valid && first);
        if (lane != 0) return;
        if (batch != b) {
            flush(acc);
            b = batch;
            sampled = all = rows = 0;
        }
        sampled += __popc(s);
        all += __popc(v);
        rows += __popc(f);
    }
};

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
    static constexpr int CONST_BYTES = CPG * 16;        // folding constants of the group's channels
    static constexpr int FIXED = 1024 + W_BYTES + 2 * STG_BYTES + SNB * 128 * 16 + CONST_BYTES + 1024;
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
    // the group's folding constants by channel pair k (channels 2k, 2k + 1): [k][0] = gate sums and
    // shifts {sg0, sg1, hg0, hg1}, [k][1] = projection sums and shifts
    float4 *cpair = stats + C::SNB * 128;
    K1Smem &s = *reinterpret_cast<K1Smem *>(cpair + C::CPG);

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
    if ((int)threadIdx.x < C::CPG / 2) {
        const float4 *v = p.vec + operand * C::C_H + ch0 + 2 * threadIdx.x;
        const float4 v0 = v[0], v1 = v[1];
        cpair[2 * threadIdx.x] = make_float4(v0.x, v1.x, v0.y, v1.y);
        cpair[2 * threadIdx.x + 1] = make_float4(v0.z, v1.z, v0.w, v1.w);
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
        // unmasked pairs seen so far (group 0's CTAs count them); the sampled pairs are each
        // tile's first 16, the ones whose outputs the epilogue sums
        const bool counting = p.acc != nullptr && group == 0;
        PairCounts counts;
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
            // 1 (no mask), the mask entry, or 0 past the last pair
            float m = pi < p.NN ? 1.f : 0.f;
            if (p.mask && pi < p.NN) m = __uint_as_float((uint32_t)p.mask[(long long)b * p.NN + pi] << 16);
            if (counting) counts.add(p.acc, b, m != 0.f, row < 16, pi % p.N == 0, lane);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sempty[sbuf], sphase ^ 1, abort_flag, kErrTimeoutEpilogue))) break;
            stats[sbuf * 128 + row] = make_float4(-mean, rstd, 0.5f * m, 0.f);   // the form the epilogue uses
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sfull[sbuf]);
            if (++sbuf == C::SNB) { sbuf = 0; sphase ^= 1; }
        }
        if (counting && lane == 0) counts.flush(p.acc);
    } else {
        // epilogue: warpgroup wg handles channels [ch0 + wg*CH_WG, +CH_WG)
        const int wg = warp >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;
        uint16_t *stg = reinterpret_cast<uint16_t *>(staging + wg * C::STG_BYTES);
        const bool leader = (threadIdx.x & 127) == 0;
        const CUtensorMap *tm_out = operand == 0 ? &p.tm_a : &p.tm_b;
        const float4 *cp = cpair + wg * C::CH_WG;       // this warpgroup's CH_WG / 2 channel pairs
        int abuf = 0;
        uint32_t aphase = 0;
        int sbuf = 0;
        uint32_t sphase = 0;
        // running sums of this thread's outputs per channel over batch element sum_b (the first 16
        // pairs of each tile: the sampled ones); summed over the warp and added to the channel sums
        // when the batch element changes and at the end
        unsigned long long *acc_w = p.acc ? p.acc + operand * C::C_H + ch0 + wg * C::CH_WG : nullptr;
        int sum_b = -1;
        float run[C::CH_WG];
#pragma unroll
        for (int t = 0; t < C::CH_WG; ++t) run[t] = 0.f;
        auto flush = [&](int fb) {
#pragma unroll
            for (int t = 0; t < C::CH_WG; ++t) {
                float v = run[t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) atomicAdd(acc_w + (size_t)fb * kAccStride + t, (unsigned long long)llrintf(v * kAccScale));
                run[t] = 0.f;
            }
        };
        TileWalk tw(cta_in_group, p.tiles_per_batch);
        for (int pt = cta_in_group; pt < num_ptiles; pt += ctas_per_group, tw.advance(ctas_per_group, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * 128;
            if (acc_w && b != sum_b) {
                if (sum_b >= 0) flush(sum_b);
                sum_b = b;
            }
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
            const float2 nmean2 = make_float2(st.x, st.x), rstd2 = make_float2(st.y, st.y);
            const float2 hm2 = make_float2(st.z, st.z);

            if (!group_all(mbar_wait(&s.tfull[abuf], aphase, abort_flag, kErrTimeoutEpilogue), 1 + wg, 128)) break;
            tc_fence_after();
            if (leader) tma_store_wait_read<0>();
            named_bar_sync(1 + wg, 128);
#pragma unroll
            for (int blk = 0; blk < C::BLK_WG; ++blk) {   // unrolled: run[] stays in registers
                float v[32];
                tmem_ld32(tmem_base + abuf * C::NCOL + ((uint32_t)(q * 32) << 16) + (wg * C::BLK_WG + blk) * 32, v);
                tc_wait_ld();
                // channels e, e + 1 in packed pairs: the gate as (m/2) tanh(g/2) + m/2 (gate rows
                // folded with an extra 1/2), times the projection, one f16x2 rounding
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const float4 cg = cp[blk * 16 + e], cq = cp[blk * 16 + e + 1];
                    const float2 gv = f2_fma(rstd2, f2_fma(nmean2, make_float2(cg.x, cg.y), make_float2(v[e], v[e + 1])),
                                             make_float2(cg.z, cg.w));
                    const float2 pv = f2_fma(rstd2, f2_fma(nmean2, make_float2(cq.x, cq.y), make_float2(v[16 + e], v[17 + e])),
                                             make_float2(cq.z, cq.w));
                    const float2 gm = f2_fma(make_float2(tanh_approx(gv.x), tanh_approx(gv.y)), hm2, hm2);
                    const float2 av = f2_mul(gm, pv);
                    const uint32_t h2 = pack_f16x2(av.x, av.y);
                    stg[(blk * 16 + e) * 128 + row] = (uint16_t)(h2 & 0xFFFFu);
                    stg[(blk * 16 + e + 1) * 128 + row] = (uint16_t)(h2 >> 16);
                    if (row < 16) {            // sampled pairs, unrounded: an estimate needs no more
                        run[blk * 16 + e] += av.x;
                        run[blk * 16 + e + 1] += av.y;
                    }
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
        if (acc_w && sum_b >= 0) flush(sum_b);
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
// K1 for c_z = 128 on CTA pairs: clusters of two CTAs whose tensor cores run one M = 256 MMA
// together (tcgen05 cta_group::2), one TMEM lane per hidden channel.
//
// A pair takes 128-pair tiles. CTA r holds the folded weights of operand r (gate rows, then
// projection rows: 2 x 128 channels x c_z, 64 KB, resident for the whole kernel) and loads pairs
// [64r, 64r + 64) of each tile (one 16 KB TMA box with both 64-channel halves). One thread of
// CTA 0 issues M = 256, N = 128 MMAs: A = operand 0's rows (CTA 0) over operand 1's (CTA 1),
// B = the tile's 128 pairs (64 from each CTA), and CTA r's TMEM receives D_r = 128 channels of
// operand r x 128 pairs (gate and projection accumulators of 128 columns, double-buffered: all
// 512 columns). Per k-step each CTA's shared memory supplies 4 KB of weights and 2 KB of z for
// 128 x 128 outputs; one CTA computing both operands of a 64-pair tile with M = 128, N = 64 MMAs
// supplies the same 6 KB for 128 x 64, and shared-memory bandwidth bounded that design. With
// half-tiles in the ring, five z stages fit beside the output staging.
// Each CTA computes the LayerNorm statistics of its 64 pairs and sends them to the peer's
// shared memory with st.async, which completes the peer's statistics-full barrier by bytes, so
// either epilogue has all 128 pairs' (-mean, rstd, mask / 2).
// Hand-offs across the pair (every wait bounded):
//   - CTA 1's MMA warp relays to CTA 0 that CTA 1's weights, and each of its z half-tiles, have
//     landed (remote mbarrier arrivals); every TMA copy completes on a barrier of the CTA that
//     issued it;
//   - the MMA commits arrive on both CTAs' z-free and accumulator-full barriers (multicast);
//   - the epilogue warps of both CTAs arrive on CTA 0's accumulator-free barrier and on both
//     CTAs' statistics-free barriers.
// The remote arrivals release at CTA scope (the default): each signals a completion the waiter
// needs no data from this thread for (a copy observed to have landed, loads returned, tensor
// memory read after tcgen05.fence::before_thread_sync); a cluster-scope release waited for the
// thread's outstanding memory traffic, about a microsecond per arrival here.
// Two teams of eight epilogue warps take alternate tiles, each team with its own accumulator
// buffer; warp 4h + q of a team takes pairs [64h, 64h + 64) of its tile and channels
// [32q, 32q + 32) of the CTA's operand, so that channel's folding constants stay in registers;
// the per-pair statistics are read from shared memory (broadcast; mask / 2 as bf16, exact, so one
// 16-byte load carries a step's eight); consecutive pairs of one channel are consecutive TMEM
// columns, which pack directly into 16-byte rows of the channel-major output. The arithmetic is
// fp32 in packed pairs (f32x2) up to one f16x2 rounding of the result: the gate as
// (mask/2) tanh(g/2) + mask/2 with one tanh.approx.f32 per output (the gate rows are folded with
// an extra factor 1/2), times the projection. Each warp stores its [32 channels][64 pairs] block
// of a tile with one TMA store, so every channel row is written in 128-byte segments (at
// N = 2048, where a and b cannot stay in L2, 64-byte segments took 29% longer and 32-byte ones
// twice as long). The TMEM loads of each 8-pair step are issued one step ahead.
// The sampled pairs behind the offset of the stored x are the first 8 of each 64-pair half.
// Four statistics slots (two per team) let the statistics run ahead of the epilogue, and each
// thread's mask entries are loaded two tiles ahead: in the forward, where the mask comes from HBM,
// the load took as long as a tile and stalled the statistics, and with them the epilogue.
// Warps: 0-15 epilogue, 16-19 LayerNorm statistics (one per scheduler; two warps, each with the
// pair rows of one channel half, took a tile period of their own), 20 TMA producer, 21 TMEM
// allocator and MMA issuer (CTA 0) or relay (CTA 1).
struct K1PairCfg {
    static constexpr int CZ = 128, C_H = kHidden, TP = 128, HP = 64;   // pairs per tile, per CTA
    static constexpr int W_CHUNK = 2 * C_H * 64 * 2;                   // [256 rows][64 k]: 32 KB
    static constexpr int W_BYTES = (CZ / 64) * W_CHUNK;                // 64 KB
    static constexpr int TILE = HP * CZ * 2;                           // 16 KB: [2 halves][64 pairs][64 ch]
    static constexpr int HALF = HP * 128;
    static constexpr int WARP_STG = 32 * HP * 2;                       // one [32 channels][64 pairs] block
    static constexpr int EPI_WARPS = 16;
    static constexpr int STG_TOTAL = EPI_WARPS * WARP_STG;             // 64 KB
    static constexpr int STATS_WARP0 = 16, STATS_WARPS = 4;            // one per scheduler
    static constexpr int TMA_WARP = 20, MMA_WARP = 21;
    static constexpr int THREADS = 22 * 32;
    static constexpr int STATS_BAR = 1;                                // named barrier of the statistics warps
    static constexpr int SNB = 4;                                      // statistics slots: two per team
    static constexpr int STATS_BYTES = SNB * TP * 10;                  // -mean, rstd (f32), mask / 2 (bf16)
    static constexpr int XCH_BYTES = 2 * HP * 8;                       // channel-half partials, by tile parity
    static constexpr int FIXED = 1024 + W_BYTES + STG_TOTAL + STATS_BYTES + XCH_BYTES + 512;
    static constexpr int S = (232448 - FIXED) / TILE > 8 ? 8 : (232448 - FIXED) / TILE;
    static constexpr size_t SMEM = FIXED + (size_t)S * TILE;
};

struct K1PairSmem {
    uint64_t wbar, pwbar;                 // this CTA's weights landed; (CTA 0) CTA 1's weights landed
    uint64_t full[8], empty[8], pfull[8]; // z half-tile landed / free; (CTA 0) CTA 1's half landed
    uint64_t tfull[2], tempty[2];         // accumulator buffer full; (CTA 0) free in both CTAs
    uint64_t sfull[4], sempty[4];         // statistics slot written by both CTAs / read by both
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

template <bool SKIP>
__global__ void __launch_bounds__(K1PairCfg::THREADS, 1) k1_project_pair_kernel(const __grid_constant__ K1Args p) {
    using C = K1PairCfg;
    static_assert(sizeof(K1PairSmem) <= 512, "barrier block");
    static_assert(C::S >= 2, "z ring");
    extern __shared__ uint8_t smem_raw[];
    // the same offsets in both CTAs: the MMA descriptors and the remote addresses rely on it
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *w_s = base;
    uint8_t *tiles = w_s + C::W_BYTES;
    uint8_t *staging = tiles + C::S * C::TILE;
    float *st_nmean = reinterpret_cast<float *>(staging + C::STG_TOTAL);   // [SNB][128]
    float *st_rstd = st_nmean + C::SNB * C::TP;
    uint16_t *st_hmask = reinterpret_cast<uint16_t *>(st_rstd + C::SNB * C::TP);   // mask / 2 in bf16 (exact)
    float2 *xch = reinterpret_cast<float2 *>(reinterpret_cast<uint8_t *>(st_hmask) + C::SNB * C::TP * 2);   // [2][64]
    K1PairSmem &s = *reinterpret_cast<K1PairSmem *>(reinterpret_cast<uint8_t *>(xch) + C::XCH_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;
    const uint32_t rank = cluster_ctarank();     // 0: issues the MMAs; 1: its peer
    const uint32_t peer = rank ^ 1u;
    const int pair = blockIdx.x >> 1;            // clusters are CTAs 2k, 2k + 1
    const int npairs = gridDim.x >> 1;
    const int num_tiles = p.B * p.tiles_per_batch;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        mbar_init(&s.pwbar, 1);
        for (int i = 0; i < C::S; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + C::STATS_WARPS);      // the MMA commit + this CTA's statistics warps
            mbar_init(&s.pfull[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], C::EPI_WARPS);           // the team that drains buffer i, in both CTAs
        }
        for (int i = 0; i < C::SNB; ++i) {
            mbar_init(&s.sfull[i], 2);                        // the two writing warps + the peer's statistics, by bytes
            mbar_init(&s.sempty[i], C::EPI_WARPS);           // the team that reads slot i, in both CTAs
        }
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    cluster_sync_all();                          // both CTAs' barriers exist before either signals the other
    if (warp == C::MMA_WARP) {
        tmem_alloc_pair(&s.tmem_base, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    pdl_launch_dependents();
    if (warp != C::TMA_WARP) pdl_wait();

    if (warp == C::TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_z);
            tma_prefetch_desc(&p.tm_w);
            mbar_arrive_expect_tx(&s.wbar, C::W_BYTES);
            for (int kc = 0; kc < C::CZ / 64; ++kc)
                tma_load_2d(w_s + kc * C::W_CHUNK, &p.tm_w, &s.wbar, kc * 64, (int)rank * 2 * C::C_H);
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;
            TileWalk tw(pair, p.tiles_per_batch);
            for (int t = pair; t < num_tiles; t += npairs, tw.advance(npairs, p.tiles_per_batch)) {
                const int b = tw.b;
                const long long p0 = (long long)tw.t * C::TP;
                if (SKIP && tile_masked_out<C::TP>(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
                if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                mbar_arrive_expect_tx(&s.full[stage], C::TILE);
                // a half past the last pair (NN / 64 odd) is filled with zeros by the copy
                tma_load_4d(tiles + stage * C::TILE, &p.tm_z, &s.full[stage], 0, (int)(p0 + (long long)rank * C::HP), 0, b);
                ++filled;
                if (++stage == C::S) { stage = 0; phase ^= 1; }
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
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_f32acc(256, C::TP, false, false, false);
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma) &&
                      mbar_wait_cluster(&s.pwbar, 0, abort_flag, kErrTimeoutMma);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t aphase = 0;            // bit i: buffer i's phase
            int j = 0;
            TileWalk tw(pair, p.tiles_per_batch);
            for (int t = pair; ok && t < num_tiles; t += npairs, tw.advance(npairs, p.tiles_per_batch), ++j) {
                if (SKIP && tile_masked_out<C::TP>(p.ext, tw.b, (long long)tw.t * C::TP, p.N, p.NN, p.rowdiv)) continue;
                const int abuf = j & 1;
                if (!mbar_wait(&s.tempty[abuf], ((aphase >> abuf) & 1u) ^ 1u, abort_flag, kErrTimeoutMma)) break;
                if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) break;
                if (!mbar_wait(&s.pfull[stage], phase, abort_flag, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint8_t *zt = tiles + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < C::CZ / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(zt + (kk >> 2) * C::HALF + (kk & 3) * 32, 16, 1024);
                    const uint8_t *wk = w_s + (kk >> 2) * C::W_CHUNK + (kk & 3) * 32;
#pragma unroll
                    for (int r = 0; r < 2; ++r)
                        tc_mma_bf16_pair(tmem_base + abuf * 256 + r * C::TP, smem_desc_sw128(wk + r * C::C_H * 128, 16, 1024),
                                         bd, idesc, kk != 0);
                }
                tc_commit_pair_mc(&s.empty[stage], 0x3);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
                tc_commit_pair_mc(&s.tfull[abuf], 0x3);
                aphase ^= 1u << abuf;
            }
            tc_commit_pair(&s.drain);
            mbar_drain(&s.drain, 0);
        } else if (lane == 0) {
            // CTA 1: tell CTA 0 when this CTA's weights and each of its z half-tiles have landed
            const uint32_t r_pwbar = mapa_shared(&s.pwbar, 0);
            const uint32_t r_pfull = mapa_shared(&s.pfull[0], 0);
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma);
            if (ok) mbar_arrive_cluster(r_pwbar);
            int stage = 0;
            uint32_t phase = 0;
            TileWalk tw(pair, p.tiles_per_batch);
            for (int t = pair; ok && t < num_tiles; t += npairs, tw.advance(npairs, p.tiles_per_batch)) {
                if (SKIP && tile_masked_out<C::TP>(p.ext, tw.b, (long long)tw.t * C::TP, p.N, p.NN, p.rowdiv)) continue;
                if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) break;
                mbar_arrive_remote(r_pfull + (uint32_t)stage * 8u);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp >= C::STATS_WARP0) {
        // LayerNorm statistics of this CTA's 64 pairs: warp STATS_WARP0 + s takes channel half
        // ch = s / 2 of pairs [32 (s % 2), + 32); the channel-half-1 warps hand their partial (mean,
        // sum of squared deviations) to the channel-half-0 warps, which combine the two
        // (the pairwise update of Chan, Golub and LeVeque) and write the statistics
        const int sw = warp - C::STATS_WARP0;
        const int ch = sw >> 1;
        const int row = (sw & 1) * 32 + lane;                      // the pair within this CTA's half
        const int trow = (int)rank * C::HP + row;                  // ... within the tile
        const bool writer = ch == 0;
        const uint32_t r_nmean = mapa_shared(st_nmean, peer);
        const uint32_t r_rstd = mapa_shared(st_rstd, peer);
        const uint32_t r_hmask = mapa_shared(st_hmask, peer);
        const uint32_t r_sfull = mapa_shared(&s.sfull[0], peer);
        // bytes one writing warp sends the peer per tile: -mean and rstd of its 32 pairs, and their
        // mask / 2 two to a word
        constexpr uint32_t kPeerBytes = 32 * 4 + 32 * 4 + 16 * 4;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t sphase = 0;                // bit i: statistics slot i's phase
        int j = -1;
        bool alive = true;                  // a writer's wait for its slot succeeded
        const bool counting = writer && p.acc != nullptr;
        PairCounts counts;                  // the sampled pairs are the first 8 of each half
        // this thread's mask entry (bf16 bits; 1 without a mask, 0 past the last pair) of a tile,
        // loaded two tiles ahead of its use: from HBM under the forward's traffic the load takes
        // about as long as a tile
        auto mask_bits = [&](int t, const TileWalk &w) -> uint16_t {
            if (!writer || t >= num_tiles) return 0;
            const long long pi = (long long)w.t * C::TP + trow;
            if (pi >= p.NN) return 0;
            return p.mask ? p.mask[(long long)w.b * p.NN + pi] : (uint16_t)0x3F80u;
        };
        TileWalk tw(pair, p.tiles_per_batch);
        TileWalk tw_ahead = tw;
        uint16_t m_next = mask_bits(pair, tw_ahead);
        tw_ahead.advance(npairs, p.tiles_per_batch);
        uint16_t m_next2 = mask_bits(pair + npairs, tw_ahead);
        tw_ahead.advance(npairs, p.tiles_per_batch);
        for (int t = pair; t < num_tiles; t += npairs, tw.advance(npairs, p.tiles_per_batch)) {
            const int b = tw.b;
            const long long p0 = (long long)tw.t * C::TP;
            const uint16_t mbits = m_next;
            m_next = m_next2;
            m_next2 = mask_bits(t + 2 * npairs, tw_ahead);
            tw_ahead.advance(npairs, p.tiles_per_batch);
            ++j;
            if (SKIP && tile_masked_out<C::TP>(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
            const int sbuf = j & (C::SNB - 1);      // tile j's slot; team j & 1 reads it
            const long long pi = p0 + trow;
            if (counting) counts.add(p.acc, b, (mbits & 0x7FFFu) != 0, row < 8, pi % p.N == 0, lane);
            const bool landed = __all_sync(0xffffffffu, mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutEpilogue));
            // the four warps leave together (the barrier below needs all of them)
            if (!group_all(landed && alive, C::STATS_BAR, 32 * C::STATS_WARPS)) break;
            const uint8_t *zh = tiles + stage * C::TILE + ch * C::HALF;
            float shift = 0.f;
            float2 nsh = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 w = *reinterpret_cast<const uint4 *>(zh + sw128_offset(row, u));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                if (u == 0) {
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
            // this half's mean and sum of squared deviations from it (64 channels)
            const float sd = s1.x + s1.y;
            const float mh = shift + sd * (1.0f / 64.0f);
            const float m2h = fmaxf((s2.x + s2.y) - sd * sd * (1.0f / 64.0f), 0.f);
            float2 *xs = xch + (j & 1) * C::HP;
            if (!writer) xs[row] = make_float2(mh, m2h);
            named_bar_sync(C::STATS_BAR, 32 * C::STATS_WARPS);
            if (!writer) continue;
            const float2 o = xs[row];
            const float dmean = o.x - mh;
            const float mean = mh + 0.5f * dmean;
            const float var = fmaxf(m2h + o.y + dmean * dmean * 32.0f, 0.f) * (1.0f / (float)C::CZ);
            // both CTAs' epilogues have read the slot's previous tile
            alive = __all_sync(0xffffffffu, mbar_wait(&s.sempty[sbuf], ((sphase >> sbuf) & 1u) ^ 1u, abort_flag,
                                                      kErrTimeoutEpilogue));
            if (!alive) continue;           // the next tile's agreement takes every warp out
            const float nmean = -mean, rstd = rsqrtf(var + p.eps);
            const uint16_t hm = (uint16_t)(__float_as_uint(0.5f * __uint_as_float((uint32_t)mbits << 16)) >> 16);
            const uint32_t hm_next = __shfl_down_sync(0xffffffffu, (uint32_t)hm, 1);
            const int idx = sbuf * C::TP + trow;
            st_nmean[idx] = nmean;
            st_rstd[idx] = rstd;
            st_hmask[idx] = hm;
            // into the peer's slot, completing its statistics-full barrier by bytes
            const uint32_t rbar = r_sfull + (uint32_t)sbuf * 8u;
            st_async_u32(r_nmean + (uint32_t)idx * 4u, __float_as_uint(nmean), rbar);
            st_async_u32(r_rstd + (uint32_t)idx * 4u, __float_as_uint(rstd), rbar);
            if ((lane & 1) == 0) st_async_u32(r_hmask + (uint32_t)idx * 2u, (uint32_t)hm | (hm_next << 16), rbar);
            __syncwarp();
            // this warp's pairs are written here; the peer's counterpart warp sends as many bytes
            if (lane == 0) mbar_arrive_expect_tx(&s.sfull[sbuf], kPeerBytes);
            sphase ^= 1u << sbuf;
        }
        if (counting && lane == 0) counts.flush(p.acc);
    } else {
        // two teams of eight warps take alternate tiles; warp 4h + q of a team takes the tile's pairs
        // [64h, 64h + 64) and channels [32q, 32q + 32) of the CTA's operand and stores them as one
        // [32 channels][64 pairs] block
        const int team = warp >> 3;
        const int h = (warp >> 2) & 1;
        const int q = warp & 3;
        const int c = q * 32 + lane;
        uint8_t *stg = staging + warp * C::WARP_STG;
        const CUtensorMap *tm_out = rank == 0 ? &p.tm_a : &p.tm_b;
        const float4 cv = p.vec[rank * C::C_H + c];
        const float2 cg_sum = make_float2(cv.x, cv.x), cg_shift = make_float2(cv.y, cv.y);
        const float2 cp_sum = make_float2(cv.z, cv.z), cp_shift = make_float2(cv.w, cv.w);
        const int buf = team;
        const uint32_t tbase = tmem_base + buf * 256 + h * C::HP + ((uint32_t)(q * 32) << 16);
        const uint32_t r_tempty = mapa_shared(&s.tempty[buf], 0);       // CTA 0's
        const uint32_t r_sempty0 = mapa_shared(&s.sempty[0], peer);
        unsigned long long *acc_c = p.acc ? p.acc + rank * C::C_H + c : nullptr;
        int sum_b = -1;
        float2 run = make_float2(0.f, 0.f);
        uint32_t phase = 0;
        uint32_t sphase = 0;                // bit i: statistics slot i's phase
        const int first = pair + team * npairs;
        int jt = team;                      // the pair's tile index j of this tile: team, team + 2, ...
        TileWalk tw(first, p.tiles_per_batch);
        for (int t = first; t < num_tiles; t += 2 * npairs, tw.advance(2 * npairs, p.tiles_per_batch), jt += 2) {
            const int b = tw.b;
            const long long pt0 = (long long)tw.t * C::TP;
            const long long p0 = pt0 + h * C::HP;           // this warp's 64 pairs
            const bool in_range = p0 < p.NN;                // NN is a multiple of 64
            if (acc_c && b != sum_b) {
                if (sum_b >= 0) atomicAdd(acc_c + (size_t)sum_b * kAccStride, (unsigned long long)llrintf((run.x + run.y) * kAccScale));
                sum_b = b;
                run = make_float2(0.f, 0.f);
            }
            if (SKIP && tile_masked_out<C::TP>(p.ext, b, pt0, p.N, p.NN, p.rowdiv)) {
                if (lane == 0) tma_store_wait_read<0>();
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4 *>(stg + sw128_offset(lane, u)) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && in_range) {
                    tma_store_3d(tm_out, stg, (int32_t)p0, q * 32, b);
                    tma_store_commit();
                }
                continue;
            }
            const int sb = jt & (C::SNB - 1);   // the tile's statistics slot
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sfull[sb], (sphase >> sb) & 1u, abort_flag, kErrTimeoutEpilogue) &&
                                             mbar_wait(&s.tfull[buf], phase, abort_flag, kErrTimeoutEpilogue)))
                break;
            phase ^= 1;
            sphase ^= 1u << sb;
            const float *snmean = st_nmean + sb * C::TP + h * C::HP, *srstd = st_rstd + sb * C::TP + h * C::HP;
            const uint16_t *shmask = st_hmask + sb * C::TP + h * C::HP;
            tc_fence_after();
            // 8-pair steps it = 0 .. 7, each writing 16 bytes of every channel row of the warp's
            // store block; step it + 1's TMEM loads are issued before step it's arithmetic
            constexpr int NIT = C::HP / 8;
            float g0[8], p0v[8], g1[8], p1v[8];
            tmem_ld8(tbase, g0);
            tmem_ld8(tbase + C::TP, p0v);
            auto step = [&](const int it, float (&gc)[8], float (&pc)[8], float (&gn)[8], float (&pn)[8]) {
                const int o = 8 * it;
                if (it == 0) {          // the store of this warp's previous tile has read the block
                    if (lane == 0) tma_store_wait_read<0>();
                    __syncwarp();
                }
                tc_wait_ld_regs8(gc, pc);
                if (it + 1 < NIT) {
                    tmem_ld8(tbase + o + 8, gn);
                    tmem_ld8(tbase + C::TP + o + 8, pn);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(r_tempty);
                }
                uint32_t outw[4];
                const uint4 mk8 = *reinterpret_cast<const uint4 *>(shmask + o);     // the step's 8 mask / 2
#pragma unroll
                for (int jj = 0; jj < 8; jj += 4) {
                    const float4 nm = *reinterpret_cast<const float4 *>(snmean + o + jj);
                    const float4 rs = *reinterpret_cast<const float4 *>(srstd + o + jj);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float2 nm2 = hh == 0 ? make_float2(nm.x, nm.y) : make_float2(nm.z, nm.w);
                        const float2 rs2 = hh == 0 ? make_float2(rs.x, rs.y) : make_float2(rs.z, rs.w);
                        const uint32_t mw = jj == 0 ? (hh == 0 ? mk8.x : mk8.y) : (hh == 0 ? mk8.z : mk8.w);
                        const float2 hm2 = make_float2(bf16_lo(mw), bf16_hi(mw));
                        const float2 gv = f2_fma(rs2, f2_fma(nm2, cg_sum, make_float2(gc[jj + 2 * hh], gc[jj + 2 * hh + 1])), cg_shift);
                        const float2 pv = f2_fma(rs2, f2_fma(nm2, cp_sum, make_float2(pc[jj + 2 * hh], pc[jj + 2 * hh + 1])), cp_shift);
                        const float2 gm = f2_fma(make_float2(tanh_approx(gv.x), tanh_approx(gv.y)), hm2, hm2);
                        const float2 av = f2_mul(gm, pv);
                        outw[jj / 2 + hh] = pack_f16x2(av.x, av.y);
                        if (it == 0) run = f2_add(run, av);    // the sampled pairs: the half's first 8
                    }
                }
                *reinterpret_cast<uint4 *>(stg + sw128_offset(lane, it)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                if (it == NIT - 1) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&s.sempty[sb]);
                        mbar_arrive_remote(r_sempty0 + (uint32_t)sb * 8u);
                        if (in_range) {
                            tma_store_3d(tm_out, stg, (int32_t)p0, q * 32, b);
                            tma_store_commit();
                        }
                    }
                }
            };
#pragma unroll
            for (int it = 0; it < NIT; it += 2) {
                step(it, g0, p0v, g1, p1v);
                step(it + 1, g1, p1v, g0, p0v);
            }
        }
        if (acc_c && sum_b >= 0) atomicAdd(acc_c + (size_t)sum_b * kAccStride, (unsigned long long)llrintf((run.x + run.y) * kAccScale));
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // neither CTA leaves while the other may still signal it
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

int k1_ncol(int c_z) { return c_z == 128 ? 256 : K1Cfg<384>::NCOL; }
int k1_groups(int c_z) { return c_z == 128 ? 1 : K1Cfg<384>::G; }
int k1_channels_per_warpgroup(int c_z) { return c_z == 128 ? K1PairCfg::C_H : K1Cfg<384>::CH_WG; }
int k1_row_mode(int c_z) { return c_z == 128 ? 2 : 1; }
int k1_tile_pairs(int c_z) { return c_z == 128 ? K1PairCfg::TP : 128; }
size_t k1_smem_bytes(int c_z) { return c_z == 128 ? K1PairCfg::SMEM : K1Cfg<384>::SMEM; }

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

// The CTA-pair kernel: as many pairs as the tiles need, up to the clusters of two that can be
// resident at once with its shared memory (queried once per device).
template <bool SKIP>
static cudaError_t k1_launch_pair(const K1Args &args, cudaStream_t stream) {
    static int configured_device = -1;
    static int max_pairs = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k1_project_pair_kernel<SKIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1PairCfg::SMEM);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(K1PairCfg::THREADS);
        cfg.dynamicSmemBytes = K1PairCfg::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, k1_project_pair_kernel<SKIP>, &cfg);
        if (e != cudaSuccess) return e;
        if (n < 1) return cudaErrorInvalidConfiguration;
        max_pairs = n;
        configured_device = dev;
    }
    const long long tiles = (long long)args.B * args.tiles_per_batch;
    const int pairs = tiles < (long long)max_pairs ? (int)(tiles > 0 ? tiles : 1) : max_pairs;
    return launch_pdl(k1_project_pair_kernel<SKIP>, 2 * pairs, K1PairCfg::THREADS, K1PairCfg::SMEM, stream, args, 2);
}

cudaError_t k1_launch(int c_z, const K1Args &args, int grid, cudaStream_t stream) {
    const bool skip = args.ext != nullptr;
    if (c_z == 128) return skip ? k1_launch_pair<true>(args, stream) : k1_launch_pair<false>(args, stream);
    if (c_z == 384) return skip ? k1_launch_t<384, true>(args, grid, stream) : k1_launch_t<384, false>(args, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace trimul
