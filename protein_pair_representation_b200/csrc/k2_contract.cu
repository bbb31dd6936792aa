// k2_contract.cu -- K2, the triangle contraction on tensor cores (sm_100a).
//
// For every (batch, channel) c the contraction is one N x N x N matrix product
// ("RFProteina architecture", section "Triangle multiplication on SM90": K2 runs
// the contraction itself, one direction at a time):
//   outgoing  X_c = A_c B_c^T   (x_ij = sum_k a_ik b_jk; both operands K-major)
//   incoming  X_c = A_c^T B_c   (x_ij = sum_k a_ki b_kj; both operands MN-major)
// a, b, x are [B*c_h][N][N] of one 16-bit type (fp16 on the update path, bf16 also
// supported), with fp32 accumulation, an optional power-of-two scale and a per-channel
// offset applied to the result before rounding (x = round(scale * sum - offset)). The
// two directions differ only in the TMA boxes and in the major-ness bits of the
// shared-memory descriptors.
//
// Persistent kernel on CTA pairs (clusters of two CTAs whose tensor cores run one M = 256 MMA
// together, tcgen05 cta_group::2), 256 x 256 output tiles, 64-deep k chunks. CTA r of a pair loads
// the tile's A rows [128r, 128r + 128) and B rows [128r, 128r + 128) (B's rows are the output's
// columns), 32 KB per chunk, into a six-stage ring; one thread of CTA 0 issues M = 256, N = 256
// MMAs, and CTA r's TMEM receives output rows [128r, 128r + 128) x 256 columns. Per k chunk an
// SM's shared memory takes 32 KB from TMA and gives 32 KB to the MMAs, where a 128 x 256 tile on
// one CTA took and gave 48 KB each for the same outputs (that bounded it at large N), and L2
// serves a third fewer bytes.
//   warp 8      TMA producer (one elected lane)
//   warp 9      TMEM allocator, and MMA issuer (CTA 0); each chunk of both CTAs completes on CTA
//               0's barrier (CTA 1's copies are the pair form, cta_group::2, which may signal the
//               peer's barrier; CTA 0 expects both halves' bytes); fp32
//               accumulators in two 256-column TMEM buffers so the epilogue of tile t overlaps the
//               MMAs of tile t+1; the commits arrive on both CTAs' barriers (multicast)
//   warps 0-7   epilogue: two warpgroups, each drains 128 of the 256 columns of the CTA's 128
//               rows (tcgen05.ld), scales, rounds to 16 bits, stages through 128B-swizzled shared
//               memory and writes with TMA stores; both CTAs' warps free a buffer on CTA 0's
//               barrier (CTA-scope release: they hand over no data).
#include "kernels.h"
#include "sm100.cuh"

namespace trimul {

namespace k2 {
constexpr int BM = 128;                            // output rows per CTA
constexpr int PM = 2 * BM;                         // ... per pair tile
constexpr int BN = 256, BK = 64;
constexpr int HN = BN / 2;                         // B rows (output columns) per CTA
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;               // 16 KB
constexpr int B_BYTES = HN * BK * 2;               // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 32 KB
constexpr int STG_BYTES = BM * 64 * 2;             // 16 KB: 128 rows x 64 bf16
constexpr int EPI_WARPS = 8;
constexpr int TMA_WARP = 8, MMA_WARP = 9;
constexpr int THREADS = 320;
constexpr int TMEM_COLS = 512;

struct Smem {
    uint64_t full[STAGES], empty[STAGES];
    uint64_t tfull[2], tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr size_t SMEM_BYTES = 1024 /*align*/ + STAGES * STAGE_BYTES + 2 * STG_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace k2

// Number of 64-deep k chunks the tile (bc, m0, n0) sums over; 0: the tile is not computed.
// With mask extents {R_b, C_b}, a[., k] and b[., k] vanish for k >= C_b (outgoing: mask
// column k all zero) or k >= R_b (incoming: mask row k all zero), so the sum stops there with
// the same result (the products left out are exact zeros). When N is a multiple of 128 the
// output kernel's 128-pair tiles lie inside one row and one 128 x 256 tile here, so tiles at
// rows >= R_b or columns >= C_b, which it never reads, are not computed either.
__device__ __forceinline__ int k2_tile_chunks(const K2Args &p, int bc, int m0, int n0) {
    if (!p.ext) return p.k_chunks;
    const int b = bc / p.C;
    const int R = __ldg(p.ext + 2 * b), Cx = __ldg(p.ext + 2 * b + 1);
    if ((p.N & 127) == 0 && (m0 >= R || n0 >= Cx)) return 0;
    const int kend = p.incoming ? R : Cx;
    // at least one chunk: a tile the output kernel may still read (N % 128 != 0) is written
    // even when no k is valid, and there its one chunk sums exact zeros
    const int nk = kend > 0 ? (kend + k2::BK - 1) / k2::BK : 1;
    return nk < p.k_chunks ? nk : p.k_chunks;
}

// The shard holding global row r (row0 ascending, row0[G] = N; rows past N: the last shard,
// whose box then reads past its rows and is zero-filled).
__device__ __forceinline__ int shard_of(const K2ShardArgs &s, int r) {
    int g = 0;
    while (g + 1 < s.G && r >= s.row0[g + 1]) ++g;
    return g;
}

__host__ __device__ __forceinline__ const K2Args &base_args(const K2Args &a) { return a; }
__host__ __device__ __forceinline__ const K2Args &base_args(const K2ShardArgs &a) { return a.base; }

// SHARD: the operands of a row-sharded update come from per-shard maps (K2ShardArgs); the
// other instance carries none of that code.
template <bool SHARD, typename Args>
__global__ void __launch_bounds__(k2::THREADS, 1) k2_contract_kernel(const __grid_constant__ Args pa) {
    using namespace k2;
    const K2Args &p = base_args(pa);
    extern __shared__ uint8_t smem_raw[];
    // the same offsets in both CTAs: the MMA descriptors and the remote addresses rely on it
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *staging = base + STAGES * STAGE_BYTES;
    Smem &s = *reinterpret_cast<Smem *>(staging + 2 * STG_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abort_flag = &s.abort_flag;
    const uint32_t rank = cluster_ctarank();     // 0: issues the MMAs; 1: its peer
    const int pair = blockIdx.x >> 1;            // clusters are CTAs 2k, 2k + 1
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);           // the MMA commit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], 2 * EPI_WARPS);   // both CTAs' epilogue warps (used in CTA 0)
        }
        mbar_init(&s.drain, 1);
        s.abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == TMA_WARP && lane == 0) {
        tma_prefetch_desc(&p.tm_a);
        tma_prefetch_desc(&p.tm_b);
        tma_prefetch_desc(&p.tm_x);
        if constexpr (SHARD) {
            for (int g = 0; g < pa.G; ++g) {
                tma_prefetch_desc(&pa.tm_sb[g]);
                if (p.incoming) tma_prefetch_desc(&pa.tm_sa[g]);
            }
        }
    }
    cluster_sync_all();                          // both CTAs' barriers exist before either signals the other
    if (warp == MMA_WARP) {
        tmem_alloc_pair(&s.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    pdl_launch_dependents();
    pdl_wait();

    const int tiles_per_channel = p.m_tiles * p.n_tiles;
    const int num_tiles = p.BC * tiles_per_channel;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0;  // number of stage fills issued (for the drain at the end)
            // every chunk completes on CTA 0's barrier: CTA 0 expects both CTAs' bytes
            const uint32_t full0 = mapa_shared(&s.full[0], 0);
            for (int t = pair; t < num_tiles; t += npairs) {
                const int bc = t / tiles_per_channel;
                const int r = t - bc * tiles_per_channel;
                const int m0 = (r / p.n_tiles) * PM;
                const int n0 = (r % p.n_tiles) * BN;
                const int nk = k2_tile_chunks(p, bc, m0, n0);
                const int mr = m0 + (int)rank * BM;      // this CTA's A rows
                const int nr = n0 + (int)rank * HN;      // this CTA's B rows
                for (int kc = 0; kc < nk; ++kc) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, kErrTimeoutProducer)) goto producer_abort;
                    uint8_t *sa = stages + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], 2 * STAGE_BYTES);
                    const uint32_t fb = full0 + (uint32_t)stage * 8u;
                    const int k0 = kc * BK;
                    if constexpr (SHARD) {
                        if (!p.incoming) {
                            tma_load_3d_pair(sa, &p.tm_a, fb, k0, mr, bc);
                            const int g = shard_of(pa, nr);     // 128 b rows lie in one shard
                            tma_load_3d_pair(sb, &pa.tm_sb[g], fb, k0, nr - pa.row0[g], bc);
                        } else {
                            const int g = shard_of(pa, k0);     // a 64-row k chunk lies in one shard
                            const int kl = k0 - pa.row0[g];
#pragma unroll
                            for (int h = 0; h < BM / 64; ++h)
                                tma_load_3d_pair(sa + h * 8192, &pa.tm_sa[g], fb, pa.i0 + mr + 64 * h, kl, bc);
#pragma unroll
                            for (int h = 0; h < HN / 64; ++h)
                                tma_load_3d_pair(sb + h * 8192, &pa.tm_sb[g], fb, nr + 64 * h, kl, bc);
                        }
                    } else if (!p.incoming) {
                        tma_load_3d_pair(sa, &p.tm_a, fb, k0, mr, bc);
                        tma_load_3d_pair(sb, &p.tm_b, fb, k0, nr, bc);
                    } else {
#pragma unroll
                        for (int h = 0; h < BM / 64; ++h)
                            tma_load_3d_pair(sa + h * 8192, &p.tm_a, fb, mr + 64 * h, k0, bc);
#pragma unroll
                        for (int h = 0; h < HN / 64; ++h)
                            tma_load_3d_pair(sb + h * 8192, &p.tm_b, fb, nr + 64 * h, k0, bc);
                    }
                    ++filled;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        producer_abort:
            // (also the normal end) let the copies already issued land before the CTA exits: CTA 0
            // through their barrier (both CTAs' bytes), CTA 1 through the MMA commits that free its
            // stages once they have been read
            for (uint32_t i = 0; i < (filled < (uint32_t)STAGES ? filled : (uint32_t)STAGES); ++i) {
                uint32_t f = filled - 1 - i;
                if (rank == 0) mbar_drain(&s.full[f % STAGES], (f / STAGES) & 1);
                else mbar_drain(&s.empty[f % STAGES], (f / STAGES) & 1);
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_f32acc(PM, BN, p.incoming, p.incoming, p.f16);
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            for (int t = pair; t < num_tiles; t += npairs) {
                const int bc = t / tiles_per_channel;
                const int r = t - bc * tiles_per_channel;
                const int nk = k2_tile_chunks(p, bc, (r / p.n_tiles) * PM, (r % p.n_tiles) * BN);
                if (nk == 0) continue;
                if (!mbar_wait(&s.tempty[abuf], aphase ^ 1, abort_flag, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + abuf * BN;
                bool ok = true;
                for (int kc = 0; kc < nk; ++kc) {
                    if (!mbar_wait(&s.full[stage], phase, abort_flag, kErrTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t *sa = stages + stage * STAGE_BYTES;
                    const uint8_t *sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        uint64_t ad, bd;
                        if (!p.incoming) {
                            ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
                            bd = smem_desc_sw128(sb + kk * 32, 16, 1024);
                        } else {
                            ad = smem_desc_sw128(sa + kk * 2048, 8192, 1024);
                            bd = smem_desc_sw128(sb + kk * 2048, 8192, 1024);
                        }
                        tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kc | kk) != 0);
                    }
                    tc_commit_pair_mc(&s.empty[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit_pair_mc(&s.tfull[abuf], 0x3);
                if (++abuf == 2) { abuf = 0; aphase ^= 1; }
            }
            // all MMAs issued by this thread are complete once this arrives
            tc_commit_pair(&s.drain);
            mbar_drain(&s.drain, 0);
        }
    } else {
        // epilogue warpgroups
        const int wg = warp >> 2;            // 0 or 1: which 128 columns
        const int q = warp & 3;              // TMEM lane quarter
        const int row = q * 32 + lane;       // accumulator row = output row within the CTA's rows
        uint8_t *stg = staging + wg * STG_BYTES;
        const bool leader = (threadIdx.x & 127) == 0;
        const uint32_t r_tempty0 = mapa_shared(&s.tempty[0], 0);   // CTA 0's
        int abuf = 0;
        uint32_t aphase = 0;
        for (int t = pair; t < num_tiles; t += npairs) {
            const int bc = t / tiles_per_channel;
            const int r = t - bc * tiles_per_channel;
            const int m0 = (r / p.n_tiles) * PM;
            const int n0 = (r % p.n_tiles) * BN;
            if (k2_tile_chunks(p, bc, m0, n0) == 0) continue;
            const int mr = m0 + (int)rank * BM;
            const float nq = -__ldg(p.xoff + (size_t)bc * p.xoff_stride);   // minus this channel's offset
            if (!group_all(mbar_wait(&s.tfull[abuf], aphase, abort_flag, kErrTimeoutEpilogue), 1 + wg, 128)) break;
            tc_fence_after();
#pragma unroll 1
            for (int sub = 0; sub < 2; ++sub) {
                if (leader) tma_store_wait_read<0>();
                named_bar_sync(1 + wg, 128);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int col = wg * 128 + sub * 64 + half * 32;
                    float v[32];
                    tmem_ld32(tmem_base + abuf * BN + ((uint32_t)(q * 32) << 16) + col, v);
                    tc_wait_ld();
                    if (sub == 1 && half == 1) {
                        // the last TMEM load of the tile has landed: hand the buffer back to the
                        // MMA now, not after the conversion and store
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(r_tempty0 + (uint32_t)abuf * 8u);
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = fmaf(v[e], p.x_scale, nq);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 w;
                        if (p.f16) {
                            w.x = pack_f16x2(v[8 * u + 0], v[8 * u + 1]);
                            w.y = pack_f16x2(v[8 * u + 2], v[8 * u + 3]);
                            w.z = pack_f16x2(v[8 * u + 4], v[8 * u + 5]);
                            w.w = pack_f16x2(v[8 * u + 6], v[8 * u + 7]);
                        } else {
                            w.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
                            w.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
                            w.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
                            w.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
                        }
                        *reinterpret_cast<uint4 *>(stg + sw128_offset(row, half * 4 + u)) = w;
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(1 + wg, 128);
                if (leader) {
                    tma_store_3d(&p.tm_x, stg, n0 + wg * 128 + sub * 64, mr, bc);
                    tma_store_commit();
                }
            }
            if (++abuf == 2) { abuf = 0; aphase ^= 1; }
        }
        if (leader) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // neither CTA leaves while the other may still signal it
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

size_t k2_smem_bytes() { return k2::SMEM_BYTES; }

// As many CTA pairs as there are tiles, up to the clusters of two that can be resident at once
// with this kernel's shared memory (queried once per device).
template <bool SHARD, typename Args>
static cudaError_t k2_launch_t(const Args &args, cudaStream_t stream) {
    static int configured_device = -1;
    static int max_pairs = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(k2_contract_kernel<SHARD, Args>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)k2::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(k2::THREADS);
        cfg.dynamicSmemBytes = k2::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, k2_contract_kernel<SHARD, Args>, &cfg);
        if (e != cudaSuccess) return e;
        if (n < 1) return cudaErrorInvalidConfiguration;
        max_pairs = n;
        configured_device = dev;
    }
    const K2Args &p = base_args(args);
    const long long tiles = (long long)p.BC * p.m_tiles * p.n_tiles;
    const int pairs = tiles < (long long)max_pairs ? (int)(tiles > 0 ? tiles : 1) : max_pairs;
    return launch_pdl(k2_contract_kernel<SHARD, Args>, 2 * pairs, k2::THREADS, k2::SMEM_BYTES, stream, args, 2);
}

cudaError_t k2_launch(const K2Args &args, int grid, cudaStream_t stream) {
    (void)grid;
    return k2_launch_t<false>(args, stream);
}

cudaError_t k2_shard_launch(const K2ShardArgs &args, int grid, cudaStream_t stream) {
    (void)grid;
    return k2_launch_t<true>(args, stream);
}

}  // namespace trimul
