// gemm2_kernel.cuh -- persistent block-scaled NVFP4 GEMM on a pair of SMs (tcgen05 cta_group::2).
//
// "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992), abstract and §1:
// NVFP4 is multiplied natively by Blackwell tensor cores.  Same contract as gemm_kernel.cuh:
// C = alpha * gA * gB * sum_k val(A) sA * val(B) sB, both operands K-major, fp32 accumulation.
//
// Why a pair: with one SM per 128x256 tile, every SM streams 216 KB of operands per K = 256
// step from L2, and the mainloop is bound by that stream (about 7.4 TB/s of TMA traffic on
// B200), not by the tensor cores.  A CTA pair computes a 256x256 tile with one
// tcgen05.mma.cta_group::2: each SM holds its own 128 rows of A and one half (128 rows) of B,
// so each SM streams 1.5x fewer bytes per flop.  Operand loads are plain TMA loads (no
// multicast) whose completion both SMs report to the leader SM's barrier.
//
// Roles, per CTA of 320 threads (10 warps), persistent over 256x256 tiles:
//   warp 0, one thread : producer.  Waits for a free stage (its own "empty" barrier); the
//                        leader arms the stage's "full" barrier with both SMs' code bytes; both
//                        load A (own 128 rows) and B (own 128 of the 256 rows) reporting to the
//                        leader, and their scale atoms (A: own rows; B: all 256 rows, because
//                        each SM's tensor memory needs the scales of every B column) reporting
//                        to their own "sf_full" barrier.
//   warp 1             : allocates/frees 512 TMEM columns (both SMs); on the leader, one thread
//                        issues the four 256x256x64 MMAs of each stage and a tcgen05.commit that
//                        frees the stage on both SMs.  Nothing else sits in the MMA pipe.
//   warps 2..5         : scale writers.  Warp w owns TMEM lane quadrant w%4: it reads the
//                        stage's scale atoms from shared memory and stores them with tcgen05.st
//                        into that stage's scale region of tensor memory, in the replicated
//                        layout the block-scaled MMA reads, then reports to the leader.
//                        (Moving them with tcgen05.cp instead costs the MMA pipe ~65 cycles per
//                        copy, 12 copies per stage -- more than the MMAs themselves.)
//   warps 6..9         : epilogue.  Warp w reads TMEM lane quadrant w%4 (all 256 columns) in
//                        32-column chunks and scales them.  bf16 output goes to a per-warp
//                        staging region of shared memory; the accumulator is released and TMA
//                        stores write the block out while the next tile's MMAs run.  fp32
//                        output (1 KB per row) is stored chunk by chunk, released after the
//                        last read.
// Tensor memory: accumulator columns [0, 256); scale region of stage s at 256 + 48 s
// (A: 4 k-blocks x 4 columns, B: 4 k-blocks x 8 columns).
// Every wait is bounded; on a timeout the CTA records QT2_ERR_TIMEOUT, both CTAs drain the
// loads they issued that were not consumed, meet at the final cluster barrier and free TMEM.
#pragma once

#include "qt2_device.cuh"

namespace qt2 {

// ------------------------------------------------------------------ cluster / pair wrappers
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA 2D tile load into this CTA's shared memory whose completion is reported to an mbarrier
// of either CTA of the pair (cta_group::2); no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *tmap, int32_t x, int32_t y,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
// Arrive once on `bar` (same offset) in both CTAs of the pair when this thread's tcgen05 work
// so far has completed.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
    const uint16_t both = 0x3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     bar),
                 "h"(both)
                 : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
// 32 lanes x 32 bits x 16 columns: thread t writes lane (quadrant*32 + t), columns [col, col+16).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// TMA 2D tile store shared -> global (tracked in this thread's bulk async-group).
__device__ __forceinline__ void tma_store_2d(const void *tmap, uint32_t src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
                 "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tc_mma_pair_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// ------------------------------------------------------------------ configuration
struct Gemm2Cfg {
    static constexpr int kStages = 4;
    static constexpr int kThreads = 320;
    static constexpr int kSfWarps = 4;
    static constexpr int kEpiWarps = 4;
    static constexpr int kA = 128 * 128;          // own 128 rows x 128 bytes (K = 256)
    static constexpr int kB = 128 * 128;          // own half of the 256 B rows
    static constexpr int kSfa = 4 * 512;          // 4 k-blocks x one 512-byte atom
    static constexpr int kSfb = 2 * 4 * 512;      // both 128-row atoms of B, 4 k-blocks each
    static constexpr int kStageBytes = kA + kB + kSfa + kSfb;   // 38912 = 38 KB, keeps 1 KB alignment
    static constexpr int kStagingBytes = 4 * 32 * 512;   // bf16 output: 4 epilogue warps x 32 rows x 256 cols
    static constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 + 256;
    static constexpr int kTmemCols = 512;         // accumulator 256 + 4 stage scale regions x 48
    static constexpr int kSfRegionCols = 48;
    // E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 256 (pair), N = 256
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (32u << 17) | (16u << 24);
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg::kThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                           const __grid_constant__ CUtensorMap tmC, const float *__restrict__ gA, const float *__restrict__ gB, float alpha,
                           void *__restrict__ Cout, int64_t ldc, int M, int N, int K, int c_dtype) {
    using Cfg = Gemm2Cfg;
    constexpr int S = Cfg::kStages;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = base + S * Cfg::kStageBytes;   // bf16 output tile, one 16 KB region per epilogue warp
    // barriers: full[S] sf_full[S] sf_ready[S] empty[S] acc_full acc_empty
    uint64_t *bars = reinterpret_cast<uint64_t *>(staging + Cfg::kStagingBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 2);
    int *consumed_slot = reinterpret_cast<int *>(tmem_slot + 1);

    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_pn = N >> 8, tiles = (M >> 8) * num_pn;
    const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
    const int nkb = K >> 6, nks = (nkb + 3) >> 2;
    const uint32_t full0 = smem_u32(bars), sf_full0 = smem_u32(bars + S), sf_ready0 = smem_u32(bars + 2 * S),
                   empty0 = smem_u32(bars + 3 * S);
    const uint32_t acc_full = smem_u32(bars + 4 * S), acc_empty = smem_u32(bars + 4 * S + 1);

    if (threadIdx.x == 0) {
        *consumed_slot = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(sf_full0 + 8 * s, 1);
            mbar_init(sf_ready0 + 8 * s, 2 * Cfg::kSfWarps);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * Cfg::kEpiWarps);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0;
    if (warp == 0 && lane == 0) {
        // -------------------------------------------------------------- producer (both CTAs)
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmSFA);
        prefetch_tmap(&tmSFB);
        const uint32_t full_leader0 = mapa_shared(full0, 0);
        bool ok = true;
        int it = 0;
        for (int tile = cluster_id; tile < tiles && ok; tile += num_clusters) {
            const int pm = tile / num_pn, pn = tile - pm * num_pn;
            const int32_t a_row = pm * 256 + (int)rank * 128, b_row = pn * 256 + (int)rank * 128;
            const int32_t sfa_row = pm * 2 + (int)rank, sfb_row = pn * 2;
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % S;
                if (it >= S && !mbar_wait(empty0 + 8 * s, ((it / S) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full_leader0 + 8 * s, sfb_bar = sf_full0 + 8 * s;
                if (leader) mbar_arrive_expect_tx(full0 + 8 * s, 2 * (Cfg::kA + Cfg::kB));
                mbar_arrive_expect_tx(sfb_bar, Cfg::kSfa + Cfg::kSfb);
                uint8_t *st = base + s * Cfg::kStageBytes;
                tma_load_2d_pair(smem_u32(st), &tmA, ks * 128, a_row, fb);
                tma_load_2d_pair(smem_u32(st + Cfg::kA), &tmB, ks * 128, b_row, fb);
                tma_load_2d(smem_u32(st + Cfg::kA + Cfg::kB), &tmSFA, ks * 256, sfa_row, sfb_bar);
                tma_load_2d(smem_u32(st + Cfg::kA + Cfg::kB + Cfg::kSfa), &tmSFB, ks * 256, sfb_row, sfb_bar);
                issued = it + 1;
            }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // -------------------------------------------------------------- MMA issuer (leader)
        bool ok = true;
        int it = 0, t_iter = 0;
        for (int tile = cluster_id; tile < tiles && ok; tile += num_clusters, ++t_iter) {
            if (t_iter > 0 && !mbar_wait(acc_empty, (t_iter - 1) & 1)) break;
            tc_fence_after();
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % S;
                const uint32_t par = (it / S) & 1;
                if (!mbar_wait(full0 + 8 * s, par) || !mbar_wait(sf_ready0 + 8 * s, par)) {
                    ok = false;
                    break;
                }
                *consumed_slot = it + 1;
                tc_fence_after();
                const int nk = min(4, nkb - ks * 4);
                const uint32_t st = smem_u32(base + s * Cfg::kStageBytes);
                const uint32_t t_sf = tmem + 256 + Cfg::kSfRegionCols * s;
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t adesc = make_smem_desc(st + 32 * kk, 16, 1024, 2);
                    const uint64_t bdesc = make_smem_desc(st + Cfg::kA + 32 * kk, 16, 1024, 2);
                    tc_mma_pair_nvfp4(tmem, adesc, bdesc, Cfg::kIdesc, t_sf + 4 * kk, t_sf + 16 + 8 * kk,
                                      (ks | kk) != 0);
                }
                tc_commit_pair_both(empty0 + 8 * s);
            }
            tc_commit_pair_both(acc_full);
        }
    } else if (warp >= 2 && warp < 2 + Cfg::kSfWarps) {
        // -------------------------------------------------------------- scale writers (both CTAs)
        // Lane r of the warp owning quadrant q writes TMEM lane 32q + r.  In the replicated layout
        // the MMA reads, that lane's 4 columns of an A k-block hold atom row r (rows r, r+32, r+64,
        // r+96 of the 128-row block, 4 scales each); its 8 columns of a B k-block hold row r of the
        // two B atoms (B rows n and n+128 of the 256-column tile).
        const int quad = warp & 3;
        const uint32_t sf_ready_leader0 = mapa_shared(sf_ready0, 0);
        int it = 0;
        bool ok = true;
        for (int tile = cluster_id; tile < tiles && ok; tile += num_clusters) {
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % S;
                if (!mbar_wait(sf_full0 + 8 * s, (it / S) & 1)) {
                    ok = false;
                    break;
                }
                const uint8_t *sfa_s = base + s * Cfg::kStageBytes + Cfg::kA + Cfg::kB;
                const uint8_t *sfb_s = sfa_s + Cfg::kSfa;
                // va: A k-blocks 0..3 (4 words each); vb[j]: B k-blocks 2j and 2j+1 (8 words each:
                // 4 from the first B atom, 4 from the second)
                uint32_t va[16], vb[2][16];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint4 a = *reinterpret_cast<const uint4 *>(sfa_s + kb * 512 + lane * 16);
                    va[4 * kb + 0] = a.x;
                    va[4 * kb + 1] = a.y;
                    va[4 * kb + 2] = a.z;
                    va[4 * kb + 3] = a.w;
                    const uint4 b0 = *reinterpret_cast<const uint4 *>(sfb_s + kb * 512 + lane * 16);
                    const uint4 b1 = *reinterpret_cast<const uint4 *>(sfb_s + 2048 + kb * 512 + lane * 16);
                    const int j = kb >> 1, o = 8 * (kb & 1);
                    vb[j][o + 0] = b0.x;
                    vb[j][o + 1] = b0.y;
                    vb[j][o + 2] = b0.z;
                    vb[j][o + 3] = b0.w;
                    vb[j][o + 4] = b1.x;
                    vb[j][o + 5] = b1.y;
                    vb[j][o + 6] = b1.z;
                    vb[j][o + 7] = b1.w;
                }
                const uint32_t t_sf = tmem + ((uint32_t)(quad * 32) << 16) + 256 + Cfg::kSfRegionCols * s;
                tmem_st_32x32b_x16(t_sf, va);
                tmem_st_32x32b_x16(t_sf + 16, vb[0]);
                tmem_st_32x32b_x16(t_sf + 32, vb[1]);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(sf_ready_leader0 + 8 * s);
            }
        }
    } else if (warp >= 2 + Cfg::kSfWarps) {
        // -------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;
        const uint32_t acc_empty_leader = mapa_shared(acc_empty, 0);
        const float sc = alpha * (*gA) * (*gB);
        int t_iter = 0;
        for (int tile = cluster_id; tile < tiles; tile += num_clusters, ++t_iter) {
            if (!mbar_wait(acc_full, t_iter & 1)) break;
            tc_fence_after();
            const int pm = tile / num_pn, pn = tile - pm * num_pn;
            const int64_t row = (int64_t)pm * 256 + rank * 128 + quad * 32 + lane;
            const int64_t col = (int64_t)pn * 256;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
            if (c_dtype == QT2_DTYPE_F32) {
                // fp32 row (1 KB): 32-column chunks stored as they are read; the accumulator is
                // released right after the last tensor-memory read
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x16(taddr + c, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_ld_32x32b_x16(taddr + c + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_ld_wait();
                    if (c == 224) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(acc_empty_leader);
                    }
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(Cout) + row * ldc + col + c);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(v[4 * i]) * sc, __uint_as_float(v[4 * i + 1]) * sc,
                                             __uint_as_float(v[4 * i + 2]) * sc, __uint_as_float(v[4 * i + 3]) * sc);
                }
            } else {
                // bf16: the warp's 32 x 256 block goes to its staging region as four 32-row x 64-column
                // boxes (128-byte swizzle), the accumulator is released, then TMA stores write it out
                uint8_t *stg = staging + (warp - 2 - Cfg::kSfWarps) * 16384;
                if (t_iter > 0) {
                    if (lane == 0) bulk_wait_read_all();   // the previous tile's stores have read it
                    __syncwarp();
                }
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x16(taddr + c, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_ld_32x32b_x16(taddr + c + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_ld_wait();
                    uint32_t p[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * sc,
                                                                  __uint_as_float(v[2 * i + 1]) * sc);
                        p[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint8_t *box = stg + (c >> 6) * 4096 + lane * 128;
                    const int k0 = (c & 63) >> 3;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4 *>(box + (((k0 + i) ^ (lane & 7)) << 4)) =
                            make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                }
                tc_fence_before();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_remote(acc_empty_leader);
                    const int32_t y0 = (int32_t)(row - lane);
#pragma unroll
                    for (int b = 0; b < 4; ++b) tma_store_2d(&tmC, smem_u32(stg + b * 4096), (int32_t)col + 64 * b, y0);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();   // this warp's output stores are complete
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // both CTAs are done; the leader's consumed count is final
    if (warp == 0 && lane == 0) {
        // Only after a timeout can issued loads still be in flight: wait (bounded) for them.
        const int consumed = (int)ld_shared_cluster_u32(mapa_shared(smem_u32(consumed_slot), 0));
        for (int it = consumed; it < issued; ++it) {
            if (leader) mbar_wait(full0 + 8 * (it % S), (it / S) & 1);
            mbar_wait(sf_full0 + 8 * (it % S), (it / S) & 1);
        }
    }
    cluster_sync_all();   // no SM frees TMEM or exits while its pair may still touch it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, Cfg::kTmemCols);
}

}  // namespace qt2
