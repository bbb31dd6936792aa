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
// Two kernels. c_z = 128 (k1_project_tm_kernel, further below) puts one hidden channel
// on each TMEM lane and makes both operands from each z tile. c_z = 384 (k1_project_kernel)
// puts one pair on each TMEM lane:
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
// K1 for c_z = 128: both operands from each z tile, one TMEM lane per hidden channel.
//
// A 64-pair tile of z (16 KB, one TMA box with both 64-channel halves) is read once per CTA, its
// LayerNorm statistics are computed once, and four accumulators are filled from it:
// D_r[c, p] = W'_r[c] . z_p for the four weight blocks r = a-gate, a-projection, b-gate,
// b-projection (A = the folded weights, 128 channels x c_z, resident in shared memory for the
// whole kernel: 128 KB; B = the z tile, 64 pairs x c_z; both K-major; M = 128, N = 64).
// Two teams of eight epilogue warps take alternate tiles, each team with its own TMEM buffer of
// the four accumulators (256 columns), so the MMA of a tile never waits for the other team;
// sixteen epilogue warps (four per scheduler) hide the latency of TMEM loads and of the gate
// arithmetic. (A design with 128-pair tiles, N = 128 and one single-buffered TMEM region per
// operand, drained by eight warps, read the weights half as often but ran 7% slower at N = 512:
// its epilogue was latency-bound.)
// A thread of the epilogue owns one channel of one operand for the whole kernel, so that
// channel's four folding constants stay in registers; the per-pair LayerNorm statistics are
// read from shared memory (broadcast; mask / 2 as bf16, exact, so that one 16-byte load carries
// a step's eight); consecutive pairs of one channel are consecutive TMEM
// columns, which pack directly into 16-byte rows of the channel-major output tile.
// The epilogue's arithmetic is fp32 in packed pairs (f32x2) up to one f16x2 rounding of the
// result: the gate as (mask/2) tanh(g/2) + mask/2 with one tanh.approx.f32 per output (the gate
// rows are folded with an extra factor 1/2), times the projection. With 256 gated outputs per
// pair, the transcendental / conversion pipe (16 lanes per SM) is a tight unit: one tanh and
// half a pack per output keep it under the HBM time per tile, where an f16x2 gate (inputs
// converted, tanh in halves, products rounded) took about twice as many. The TMEM loads of each
// 8-pair step are issued one step ahead. The channel sums behind the offset of the stored x are
// taken over the first 8 pairs of each tile (an estimate needs no more).
// Each epilogue warp stores its [32 channels][64 pairs] block of a tile with one TMA store, so
// every channel row is written in 128-byte segments: with 64-byte segments (two stores per tile
// from a 2 KB buffer) K1 at N = 2048, whose a and b cannot stay in L2, took 29% longer, and with
// 32-byte ones twice as long. The 4 KB blocks leave room for a two-tile z ring.
// Warps: 0-15 epilogue (team t = warp / 8; warp 4o + q of a team: operand o, channels
// [32q, 32q + 32)), 16-17 LayerNorm statistics, 18 TMA producer, 19 TMEM allocator + MMA issuer.
struct K1TmCfg {
    static constexpr int CZ = 128, C_H = kHidden, TP = 64;
    static constexpr int W_CHUNK = 4 * C_H * 64 * 2;
    static constexpr int W_BYTES = (CZ / 64) * W_CHUNK;        // 128 KB
    static constexpr int TILE = TP * CZ * 2;                   // 16 KB: [2 halves][64 pairs][64 ch]
    static constexpr int HALF = TP * 128;
    static constexpr int WARP_STG = 32 * TP * 2;                // one [32 channels][64 pairs] block
    static constexpr int EPI_WARPS = 16;
    static constexpr int STG_TOTAL = EPI_WARPS * WARP_STG;     // 64 KB
    static constexpr int STATS_WARP0 = 16, STATS_WARPS = TP / 32;
    static constexpr int TMA_WARP = 18, MMA_WARP = 19;
    static constexpr int THREADS = 20 * 32;
    static constexpr int STATS_BYTES = 2 * TP * 10;            // -mean, rstd (f32), mask / 2 (bf16)
    static constexpr int FIXED = 1024 + W_BYTES + STG_TOTAL + STATS_BYTES + 512;
    static constexpr int S = (232448 - FIXED) / TILE > 8 ? 8 : (232448 - FIXED) / TILE;
    static constexpr size_t SMEM = FIXED + (size_t)S * TILE;
};

template <bool SKIP>
__global__ void __launch_bounds__(K1TmCfg::THREADS, 1) k1_project_tm_kernel(const __grid_constant__ K1Args p) {
    using C = K1TmCfg;
    static_assert(sizeof(K1Smem) <= 512, "barrier block");
    static_assert(C::S >= 2, "z ring");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *w_s = base;
    uint8_t *tiles = w_s + C::W_BYTES;
    uint8_t *staging = tiles + C::S * C::TILE;
    float *st_nmean = reinterpret_cast<float *>(staging + C::STG_TOTAL);   // [2][64]
    float *st_rstd = st_nmean + 2 * C::TP;
    uint16_t *st_hmask = reinterpret_cast<uint16_t *>(st_rstd + 2 * C::TP);   // mask / 2 in bf16 (exact)
    K1Smem &s = *reinterpret_cast<K1Smem *>(reinterpret_cast<uint8_t *>(st_hmask) + 2 * C::TP * 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;
    const int num_tiles = p.B * p.tiles_per_batch;

    if (threadIdx.x == 0) {
        mbar_init(&s.wbar, 1);
        for (int i = 0; i < C::S; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + C::STATS_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], C::EPI_WARPS / 2);     // the team that drains buffer i
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
    if (warp != C::TMA_WARP) pdl_wait();

    if (warp == C::TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_z);
            tma_prefetch_desc(&p.tm_w);
            mbar_arrive_expect_tx(&s.wbar, C::W_BYTES);
            for (int kc = 0; kc < C::CZ / 64; ++kc)
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(w_s + kc * C::W_CHUNK + h * 256 * 128, &p.tm_w, &s.wbar, kc * 64, h * 256);
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;
            TileWalk tw(blockIdx.x, p.tiles_per_batch);
            for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tw.advance(gridDim.x, p.tiles_per_batch)) {
                const int b = tw.b;
                const int p0 = tw.t * C::TP;
                if (SKIP && tile_masked_out<C::TP>(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
                if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                mbar_arrive_expect_tx(&s.full[stage], C::TILE);
                tma_load_4d(tiles + stage * C::TILE, &p.tm_z, &s.full[stage], 0, p0, 0, b);
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
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(128, C::TP, false, false, false);
            bool ok = mbar_wait(&s.wbar, 0, abort_flag, kErrTimeoutMma);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t aphase = 0;            // bit i: buffer i's phase
            int j = 0;
            TileWalk tw(blockIdx.x, p.tiles_per_batch);
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x, tw.advance(gridDim.x, p.tiles_per_batch), ++j) {
                if (SKIP && tile_masked_out<C::TP>(p.ext, tw.b, tw.t * C::TP, p.N, p.NN, p.rowdiv)) continue;
                const int abuf = j & 1;
                if (!mbar_wait(&s.tempty[abuf], ((aphase >> abuf) & 1u) ^ 1u, abort_flag, kErrTimeoutMma)) break;
                if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint8_t *zt = tiles + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < C::CZ / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(zt + (kk >> 2) * C::HALF + (kk & 3) * 32, 16, 1024);
                    const uint8_t *wk = w_s + (kk >> 2) * C::W_CHUNK + (kk & 3) * 32;
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        tc_mma_bf16(tmem_base + abuf * 256 + r * C::TP, smem_desc_sw128(wk + r * C::C_H * 128, 16, 1024),
                                    bd, idesc, kk != 0);
                }
                tc_commit(&s.empty[stage]);
                if (++stage == C::S) { stage = 0; phase ^= 1; }
                tc_commit(&s.tfull[abuf]);
                aphase ^= 1u << abuf;
            }
            tc_commit(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else if (warp >= C::STATS_WARP0) {
        const int row = (warp - C::STATS_WARP0) * 32 + lane;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t sphase = 0;                // bit i: statistics buffer i's phase
        int j = -1;
        const bool counting = p.acc != nullptr;
        PairCounts counts;              // the sampled pairs are each tile's first 8
        TileWalk tw(blockIdx.x, p.tiles_per_batch);
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tw.advance(gridDim.x, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * C::TP;
            ++j;
            if (SKIP && tile_masked_out<C::TP>(p.ext, b, p0, p.N, p.NN, p.rowdiv)) continue;
            const int sbuf = j & 1;
            const long long pi = (long long)p0 + row;     // < NN: NN is a multiple of 64
            const uint16_t mbits = p.mask ? p.mask[(long long)b * p.NN + pi] : (uint16_t)0x3F80u;
            if (counting) counts.add(p.acc, b, (mbits & 0x7FFFu) != 0, row < 8, pi % p.N == 0, lane);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutEpilogue))) break;
            const uint8_t *zt = tiles + stage * C::TILE;
            float shift = 0.f;
            float2 nsh = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(zt + h * C::HALF + sw128_offset(row, u));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                    if (h == 0 && u == 0) {
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
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[stage]);
            if (++stage == C::S) { stage = 0; phase ^= 1; }
            const float inv_n = 1.0f / (float)C::CZ;
            const float dm = (s1.x + s1.y) * inv_n;
            const float var = fmaxf((s2.x + s2.y) * inv_n - dm * dm, 0.f);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sempty[sbuf], ((sphase >> sbuf) & 1u) ^ 1u, abort_flag, kErrTimeoutEpilogue))) break;
            st_nmean[sbuf * C::TP + row] = -(shift + dm);
            st_rstd[sbuf * C::TP + row] = rsqrtf(var + p.eps);
            st_hmask[sbuf * C::TP + row] = (uint16_t)(__float_as_uint(0.5f * __uint_as_float((uint32_t)mbits << 16)) >> 16);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.sfull[sbuf]);
            sphase ^= 1u << sbuf;
        }
        if (counting && lane == 0) counts.flush(p.acc);
    } else {
        const int team = warp >> 3;
        const int operand = (warp >> 2) & 1;
        const int q = warp & 3;
        const int c = q * 32 + lane;
        uint8_t *stg = staging + warp * C::WARP_STG;
        const CUtensorMap *tm_out = operand == 0 ? &p.tm_a : &p.tm_b;
        const float4 cv = p.vec[operand * C::C_H + c];
        const float2 cg_sum = make_float2(cv.x, cv.x), cg_shift = make_float2(cv.y, cv.y);
        const float2 cp_sum = make_float2(cv.z, cv.z), cp_shift = make_float2(cv.w, cv.w);
        const int buf = team;
        const uint32_t tbase = tmem_base + buf * 256 + operand * 2 * C::TP + ((uint32_t)(q * 32) << 16);
        const float *snmean = st_nmean + buf * C::TP, *srstd = st_rstd + buf * C::TP;
        const uint16_t *shmask = st_hmask + buf * C::TP;
        unsigned long long *acc_c = p.acc ? p.acc + operand * C::C_H + c : nullptr;
        int sum_b = -1;
        float2 run = make_float2(0.f, 0.f);
        uint32_t phase = 0;
        const int first = blockIdx.x + team * gridDim.x;
        TileWalk tw(first, p.tiles_per_batch);
        for (int t = first; t < num_tiles; t += 2 * gridDim.x, tw.advance(2 * gridDim.x, p.tiles_per_batch)) {
            const int b = tw.b;
            const int p0 = tw.t * C::TP;
            if (acc_c && b != sum_b) {
                if (sum_b >= 0) atomicAdd(acc_c + (size_t)sum_b * kAccStride, (unsigned long long)llrintf((run.x + run.y) * kAccScale));
                sum_b = b;
                run = make_float2(0.f, 0.f);
            }
            if (SKIP && tile_masked_out<C::TP>(p.ext, b, p0, p.N, p.NN, p.rowdiv)) {
                if (lane == 0) tma_store_wait_read<0>();
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4 *>(stg + sw128_offset(lane, u)) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(tm_out, stg, p0, q * 32, b);
                    tma_store_commit();
                }
                continue;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sfull[buf], phase, abort_flag, kErrTimeoutEpilogue) &&
                                             mbar_wait(&s.tfull[buf], phase, abort_flag, kErrTimeoutEpilogue)))
                break;
            phase ^= 1;
            tc_fence_after();
            // 8-pair steps it = 0 .. 7, each writing 16 bytes of every channel row of the tile's
            // store block; step it + 1's TMEM loads are issued before step it's arithmetic
            constexpr int NIT = C::TP / 8;
            float g0[8], p0v[8], g1[8], p1v[8];
            tmem_ld8(tbase, g0);
            tmem_ld8(tbase + C::TP, p0v);
            auto step = [&](const int it, float (&gc)[8], float (&pc)[8], float (&gn)[8], float (&pn)[8]) {
                const int o = 8 * it;
                if (it == 0) {          // the store of this team's previous tile has read the block
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
                    if (lane == 0) mbar_arrive(&s.tempty[buf]);
                }
                uint32_t outw[4];
                const uint4 mk8 = *reinterpret_cast<const uint4 *>(shmask + o);     // the step's 8 mask / 2
#pragma unroll
                for (int jj = 0; jj < 8; jj += 4) {
                    const float4 nm = *reinterpret_cast<const float4 *>(snmean + o + jj);
                    const float4 rs = *reinterpret_cast<const float4 *>(srstd + o + jj);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float2 nm2 = h == 0 ? make_float2(nm.x, nm.y) : make_float2(nm.z, nm.w);
                        const float2 rs2 = h == 0 ? make_float2(rs.x, rs.y) : make_float2(rs.z, rs.w);
                        const uint32_t mw = jj == 0 ? (h == 0 ? mk8.x : mk8.y) : (h == 0 ? mk8.z : mk8.w);
                        const float2 hm2 = make_float2(bf16_lo(mw), bf16_hi(mw));
                        const float2 gv = f2_fma(rs2, f2_fma(nm2, cg_sum, make_float2(gc[jj + 2 * h], gc[jj + 2 * h + 1])), cg_shift);
                        const float2 pv = f2_fma(rs2, f2_fma(nm2, cp_sum, make_float2(pc[jj + 2 * h], pc[jj + 2 * h + 1])), cp_shift);
                        const float2 gm = f2_fma(make_float2(tanh_approx(gv.x), tanh_approx(gv.y)), hm2, hm2);
                        const float2 av = f2_mul(gm, pv);
                        outw[jj / 2 + h] = pack_f16x2(av.x, av.y);
                        if (it == 0) run = f2_add(run, av);    // the sampled pairs: the tile's first 8
                    }
                }
                *reinterpret_cast<uint4 *>(stg + sw128_offset(lane, it)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                if (it == NIT - 1) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&s.sempty[buf]);
                        tma_store_3d(tm_out, stg, p0, q * 32, b);
                        tma_store_commit();
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
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

int k1_ncol(int c_z) { return c_z == 128 ? 256 : K1Cfg<384>::NCOL; }
int k1_groups(int c_z) { return c_z == 128 ? 1 : K1Cfg<384>::G; }
int k1_channels_per_warpgroup(int c_z) { return c_z == 128 ? K1TmCfg::C_H : K1Cfg<384>::CH_WG; }
int k1_row_mode(int c_z) { return c_z == 128 ? 2 : 1; }
int k1_tile_pairs(int c_z) { return c_z == 128 ? K1TmCfg::TP : 128; }
size_t k1_smem_bytes(int c_z) { return c_z == 128 ? K1TmCfg::SMEM : K1Cfg<384>::SMEM; }

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
static cudaError_t k1_launch_tm(const K1Args &args, int grid, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k1_project_tm_kernel<SKIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1TmCfg::SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return launch_pdl(k1_project_tm_kernel<SKIP>, grid, K1TmCfg::THREADS, K1TmCfg::SMEM, stream, args);
}

cudaError_t k1_launch(int c_z, const K1Args &args, int grid, cudaStream_t stream) {
    const bool skip = args.ext != nullptr;
    if (c_z == 128) return skip ? k1_launch_tm<true>(args, grid, stream) : k1_launch_tm<false>(args, grid, stream);
    if (c_z == 384) return skip ? k1_launch_t<384, true>(args, grid, stream) : k1_launch_t<384, false>(args, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace trimul
