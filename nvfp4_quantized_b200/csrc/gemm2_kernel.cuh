// gemm2_kernel.cuh -- persistent block-scaled NVFP4 GEMM on a pair of SMs (tcgen05 cta_group::2).
//
// "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992), abstract and §1:
// NVFP4 is multiplied natively by Blackwell tensor cores.  Same contract as gemm_kernel.cuh:
// C = alpha * gA * gB * sum_k val(A) sA * val(B) sB, both operands K-major, fp32 accumulation
// (with `local`, gA and gB are per-128-row arrays: the row's and the column's block scale).
//
// Why a pair: with one SM per 128x256 tile, every SM streams 216 KB of operands per K = 256
// step from L2.  A CTA pair computes a 256x256 tile with one tcgen05.mma.cta_group::2: each SM
// holds its own 128 rows of A and one half (128 rows) of B, so each SM streams 1.5x fewer bytes
// per flop.  Operand loads are plain TMA loads (no multicast) whose completion both SMs report to
// the leader SM's barrier.
//
// Issue discipline (measured on B200): every role that issues TMA or tcgen05 instructions runs
// as a whole converged warp and lets one lane chosen by elect.sync issue them.  The operands
// are then warp-uniform values the instructions take directly; issued from a lone lane of a
// diverged warp each tcgen05.cp / tcgen05.mma / TMA load cost ~30 ns of issue overhead, which
// made the 12 scale copies of a stage the bottleneck (the same kernel in that form ran the
// layer's dgrad GEMM in 0.186 ms; converged, in 0.115 ms).
//
// Roles, per CTA of 384 threads (12 warps), persistent over 256x256 tiles (K = 256 per stage):
//   warp 0             : producer.  Per stage, after "empty" (the MMAs that read the slot
//                        completed), one lane loads the stage's scales -- A scales of its own
//                        rows, B scales of all 256 rows (each SM's tensor memory needs the scales
//                        of every B column) -- reported to the leader's "sfull" barrier, then its
//                        own 128 rows of A and own 128 of the 256 B rows, reported to "full"
//                        (the leader expects both SMs' bytes on each): 38 KB a stage.
//   warp 2, leader     : scale copier.  After "sfull", copies the stage's 12 scale atoms from
//                        both SMs' shared memory into their tensor memory (tcgen05.cp 32x128b,
//                        replicated into the four lane quadrants, the layout the block-scaled
//                        MMA reads) and commits to "sftm" -- while the stage's codes are still
//                        in flight.  The stage's scale region is free by then: its data could
//                        only land after the MMAs of the stage that last used the region
//                        completed.
//   warp 1             : allocates/frees 512 TMEM columns (both SMs); on the leader, after
//                        "full" and "sftm", issues the four 256x256x64 MMAs of the stage and a
//                        tcgen05.commit that frees the slot on both SMs ("empty").
//   warps 4..11        : epilogue.  Warp w reads TMEM lane quadrant w%4, columns [0, 128) for
//                        warps 4..7 and [128, 256) for warps 8..11, all into registers, releases
//                        the accumulator, then scales and stores its rows straight to global
//                        memory (bf16 or fp32, 32-byte stores) while the next tile's MMAs run.
// Tensor memory: accumulator columns [0, 256); scale region s (of ring slot s) at 256 + 48 s
// (A: 4 k-blocks x 4 columns, B: 4 k-blocks x 8 columns).
// Every wait is bounded; on a timeout the CTA records QT2_ERR_TIMEOUT, the leader drains the
// loads (of both SMs) and tensor-core work that were issued, both CTAs meet at the final cluster
// barrier and free TMEM.
#pragma once

#include "qt2_device.cuh"

namespace qt2 {

// ------------------------------------------------------------------ cluster / pair wrappers
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
__device__ __forceinline__ void tc_mma_pair_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Copy one 512-byte scale atom (32 rows x 16 bytes) from shared memory into 32 TMEM lanes x 4
// columns, replicated into all four lane quadrants, in both CTAs of the pair (each from its own
// shared memory at the same address).
__device__ __forceinline__ void tc_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// Arrive on `bar` of the leader CTA only once this thread's tcgen05 work so far has completed.
__device__ __forceinline__ void tc_commit_pair_leader(uint32_t bar) {
    const uint16_t leader_only = 0x1;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     bar),
                 "h"(leader_only)
                 : "memory");
}

// 32-byte global store (sm_100 256-bit vector store); the address is 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t (&p)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(p[0]), "r"(p[1]), "r"(p[2]),
                 "r"(p[3]), "r"(p[4]), "r"(p[5]), "r"(p[6]), "r"(p[7])
                 : "memory");
}


// ------------------------------------------------------------------ configuration
struct Gemm2Cfg {
    static constexpr int kStages = 5;             // ring of A + B codes and their scales
    static constexpr int kThreads = 384;
    static constexpr int kEpiWarp0 = 4;
    static constexpr int kEpiWarps = 8;
    static constexpr int kA = 128 * 128;          // own 128 rows x 128 bytes (K = 256)
    static constexpr int kB = 128 * 128;          // own half of the 256 B rows
    static constexpr int kSfa = 4 * 512;          // 4 k-blocks x one 512-byte atom
    static constexpr int kSfb = 2 * 4 * 512;      // both 128-row atoms of B, 4 k-blocks each
    static constexpr int kStageBytes = kA + kB + kSfa + kSfb;   // 38 KB, keeps 1 KB alignment
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 512;
    static constexpr int kTmemCols = 512;         // accumulator 256 + 5 scale regions x 48
    static constexpr int kSfRegionCols = 48;
    // E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 256 (pair), N = 256
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (32u << 17) | (16u << 24);
};
static_assert(Gemm2Cfg::kStageBytes % 1024 == 0, "stage alignment");
static_assert(256 + Gemm2Cfg::kStages * Gemm2Cfg::kSfRegionCols <= Gemm2Cfg::kTmemCols, "TMEM columns");


__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg::kThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                           const float *__restrict__ gA, const float *__restrict__ gB, float alpha,
                           void *__restrict__ Cout, int64_t ldc, int M, int N, int K, int c_dtype, int local,
                           int m_fast) {
    using Cfg = Gemm2Cfg;
    constexpr int S = Cfg::kStages;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    // barriers: full[S] sftm[S] empty[S] acc_full acc_empty sfull[S]
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + S * Cfg::kStageBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 2);

    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_pm = M >> 8, num_pn = N >> 8, tiles = num_pm * num_pn;
    const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
    const int nkb = K >> 6, nks = (nkb + 3) >> 2;
    const int my_tiles = tiles > cluster_id ? (tiles - 1 - cluster_id) / num_clusters + 1 : 0;
    const int total = my_tiles * nks;   // stages this pair runs
    const uint32_t full0 = smem_u32(bars), sftm0 = smem_u32(bars + S), empty0 = smem_u32(bars + 2 * S);
    const uint32_t acc_full = smem_u32(bars + 3 * S), acc_empty = acc_full + 8;
    const uint32_t sfull0 = smem_u32(bars + 3 * S + 2);   // the stage's scale atoms landed


    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);    // codes: the leader's producer (expects both SMs' bytes)
            mbar_init(sfull0 + 8 * s, 1);   // scale atoms: likewise
            mbar_init(sftm0 + 8 * s, 1);    // the scale copier's commit
            mbar_init(empty0 + 8 * s, 1);   // the MMA issuer's commit
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

    // Tile order.  The ~74 tiles in flight at a time read their A row blocks and B row blocks
    // from L2; the operand whose row blocks they share should be the one that is re-read.  With
    // m_fast the tile index runs over M first, so the tiles in flight cover all of a small A and a
    // few B row blocks, and B streams from DRAM once (instead of once per row of tiles when A is
    // the smaller operand and N is wide).
    auto tile_coords = [&](int tile, int &pm, int &pn) {
        if (m_fast) {
            pn = tile / num_pm;
            pm = tile - pn * num_pm;
        } else {
            pm = tile / num_pn;
            pn = tile - pm * num_pn;
        }
    };
    auto stage_tile = [&](int it, int &pm, int &pn, int &ks) {
        const int tile = cluster_id + (it / nks) * num_clusters;
        ks = it % nks;
        tile_coords(tile, pm, pn);
    };

    int issued = 0;     // producer: stages whose loads were issued
    int mma_done = 0;   // MMA warp: stages whose MMAs were issued
    int copied = 0;     // copier warp: stages whose scales were copied
    if (warp == 0) {
        // -------------------------------------------------------------- producer (both CTAs)
        if (elect_one()) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            prefetch_tmap(&tmSFA);
            prefetch_tmap(&tmSFB);
        }
        __syncwarp();
        const uint32_t full_leader0 = mapa_shared(full0, 0);
        for (int it = 0; it < total; ++it) {
            const int s = it % S;
            if (it >= S && !mbar_wait_warp(empty0 + 8 * s, ((it / S) & 1) ^ 1)) break;
            int pm, pn, ks;
            stage_tile(it, pm, pn, ks);
            const uint32_t st = smem_u32(base + s * Cfg::kStageBytes);
            const uint32_t fb = full_leader0 + 8 * s;
            if (elect_one()) {
                // the scale atoms first, on their own barrier: the copier moves them into tensor
                // memory while the codes are still in flight
                const uint32_t sb = mapa_shared(sfull0, 0) + 8 * s;
                if (leader) {
                    mbar_arrive_expect_tx(sfull0 + 8 * s, 2 * (Cfg::kSfa + Cfg::kSfb));
                    mbar_arrive_expect_tx(full0 + 8 * s, 2 * (Cfg::kA + Cfg::kB));
                }
                tma_load_2d_pair(st + Cfg::kA + Cfg::kB, &tmSFA, ks * 256, pm * 2 + (int)rank, sb);
                tma_load_2d_pair(st + Cfg::kA + Cfg::kB + Cfg::kSfa, &tmSFB, ks * 256, pn * 2, sb);
                tma_load_2d_pair(st, &tmA, ks * 128, pm * 256 + (int)rank * 128, fb);
                tma_load_2d_pair(st + Cfg::kA, &tmB, ks * 128, pn * 256 + (int)rank * 128, fb);
            }
            __syncwarp();
            issued = it + 1;
        }
    } else if (warp == 1 && leader) {
        // -------------------------------------------------------------- MMA issuer (leader)
        int it = 0;
        bool ok = true;
        for (int t_iter = 0; t_iter < my_tiles && ok; ++t_iter) {
            if (t_iter > 0 && !mbar_wait_warp(acc_empty, (t_iter - 1) & 1)) break;
            tc_fence_after();
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % S;
                const uint32_t par = (it / S) & 1;
                if (!mbar_wait_warp(full0 + 8 * s, par)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait_warp(sftm0 + 8 * s, par)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nk = min(4, nkb - ks * 4);
                const uint32_t st = smem_u32(base + s * Cfg::kStageBytes);
                const uint32_t t_sf = tmem + 256 + Cfg::kSfRegionCols * s;
                if (elect_one()) {
                    for (int kk = 0; kk < nk; ++kk) {
                        const uint64_t adesc = make_smem_desc(st + 32 * kk, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(st + Cfg::kA + 32 * kk, 16, 1024, 2);
                        tc_mma_pair_nvfp4(tmem, adesc, bdesc, Cfg::kIdesc, t_sf + 4 * kk, t_sf + 16 + 8 * kk,
                                          (ks | kk) != 0);
                    }
                    tc_commit_pair_both(empty0 + 8 * s);
                }
                __syncwarp();
                mma_done = it + 1;
            }
            if (ok) {
                if (elect_one()) tc_commit_pair_both(acc_full);
                __syncwarp();
            }
        }
    } else if (warp == 2 && leader) {
        // -------------------------------------------------------------- scale copier (leader)
        // The stage's data landed, so the MMAs that last used its scale region completed.
        for (int j = 0; j < total; ++j) {
            const int s = j % S;
            if (!mbar_wait_warp(sfull0 + 8 * s, (j / S) & 1)) break;
            tc_fence_after();
            const int nk = min(4, nkb - (j % nks) * 4);
            const uint32_t sfa = smem_u32(base + s * Cfg::kStageBytes + Cfg::kA + Cfg::kB), sfb = sfa + Cfg::kSfa;
            const uint32_t t_sf = tmem + 256 + Cfg::kSfRegionCols * s;
            if (elect_one()) {
                for (int kk = 0; kk < nk; ++kk) {
                    tc_cp_pair_32x128b_warpx4(t_sf + 4 * kk, make_smem_desc(sfa + 512 * kk, 0, 128, 0));
                    tc_cp_pair_32x128b_warpx4(t_sf + 16 + 8 * kk, make_smem_desc(sfb + 512 * kk, 0, 128, 0));
                    tc_cp_pair_32x128b_warpx4(t_sf + 20 + 8 * kk, make_smem_desc(sfb + 2048 + 512 * kk, 0, 128, 0));
                }
                tc_commit_pair_leader(sftm0 + 8 * s);
            }
            __syncwarp();
            copied = j + 1;
        }
    } else if (warp >= Cfg::kEpiWarp0) {
        // -------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3, ew = warp - Cfg::kEpiWarp0;
        const int cb = (ew >> 2) * 128;   // this warp's 128 of the tile's 256 columns
        const uint32_t acc_empty_leader = mapa_shared(acc_empty, 0);
        const int64_t row_bytes = ldc * (c_dtype == QT2_DTYPE_F32 ? 4 : 2);
        const bool wide = (reinterpret_cast<uintptr_t>(Cout) & 31) == 0 && (row_bytes & 31) == 0;
        for (int t_iter = 0; t_iter < my_tiles; ++t_iter) {
            if (!mbar_wait_warp(acc_full, t_iter & 1)) break;
            tc_fence_after();
            const int tile = cluster_id + t_iter * num_clusters;
            int pm, pn;
            tile_coords(tile, pm, pn);
            const int64_t row = (int64_t)pm * 256 + rank * 128 + quad * 32 + lane;
            const int64_t col = (int64_t)pn * 256 + cb;
            // tensor scales: one each, or (CTA-local views) one per 128 rows of A and of B
            const float sc = local ? alpha * gA[pm * 2 + (int)rank] * gB[pn * 2 + (cb >> 7)] : alpha * (*gA) * (*gB);
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + cb;
            // All 128 columns into registers first, then release the accumulator, so the next
            // tile's MMAs overlap the scaling and the stores.
            uint32_t v[128];
#pragma unroll
            for (int c = 0; c < 128; c += 16)
                tmem_ld_32x32b_x16(taddr + c, *reinterpret_cast<uint32_t(*)[16]>(&v[c]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acc_empty_leader);
            // checked build: this thread's 128 outputs must lie inside C ((M - 1) * ldc + N elements)
            const int64_t esz = c_dtype == QT2_DTYPE_F32 ? 4 : 2;
            if (!QT2_STORE_OK(static_cast<uint8_t *>(Cout) + (row * ldc + col) * esz, 128 * esz, Cout,
                              ((int64_t)(M - 1) * ldc + N) * esz))
                continue;
            // 32-byte stores (each fills whole 32-byte sectors of its row) when C's rows are
            // 32-byte aligned, else 16-byte stores
            if (c_dtype == QT2_DTYPE_F32) {
                float *dst = static_cast<float *>(Cout) + row * ldc + col;
                if (wide) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint32_t p[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) p[k] = __float_as_uint(__uint_as_float(v[8 * i + k]) * sc);
                        st_global_v8(dst + 8 * i, p);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        reinterpret_cast<float4 *>(dst)[i] =
                            make_float4(__uint_as_float(v[4 * i]) * sc, __uint_as_float(v[4 * i + 1]) * sc,
                                        __uint_as_float(v[4 * i + 2]) * sc, __uint_as_float(v[4 * i + 3]) * sc);
                }
            } else {
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(Cout) + row * ldc + col;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint32_t p[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[16 * i + 2 * k]) * sc,
                                                                  __uint_as_float(v[16 * i + 2 * k + 1]) * sc);
                        p[k] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    if (wide) {
                        st_global_v8(dst + 16 * i, p);
                    } else {
                        reinterpret_cast<uint4 *>(dst + 16 * i)[0] = make_uint4(p[0], p[1], p[2], p[3]);
                        reinterpret_cast<uint4 *>(dst + 16 * i)[1] = make_uint4(p[4], p[5], p[6], p[7]);
                    }
                }
            }
        }
    }
    // Every role ends converged.  Only after a timeout can work still be in flight: the leader
    // waits (bounded) for the loads it issued past the last consumed stage and for the last
    // issued MMAs and copies, then both CTAs meet before TMEM is freed.
    __shared__ int consumed, issued_here;
    if (warp == 1 && leader && lane == 0) consumed = mma_done;
    if (warp == 0 && lane == 0) issued_here = issued;
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (leader && warp == 0 && lane == 0) {
        // both SMs' loads of a stage complete on the leader's barrier
        const int peer = (int)ld_shared_cluster_u32(mapa_shared(smem_u32(&issued_here), 1));
        const int last = max(issued, peer);
        for (int it = consumed; it < last; ++it) {
            mbar_wait(full0 + 8 * (it % S), (it / S) & 1);
            mbar_wait(sfull0 + 8 * (it % S), (it / S) & 1);
        }
    }
    if (leader && warp == 1 && lane == 0 && mma_done > 0) {
        const int it = mma_done - 1;
        mbar_wait(empty0 + 8 * (it % S), (it / S) & 1);
    }
    if (leader && warp == 2 && lane == 0 && copied > 0) {
        const int j = copied - 1;
        mbar_wait(sftm0 + 8 * (j % S), (j / S) & 1);
    }
    cluster_sync_all();   // no SM frees TMEM or exits while its pair may still touch it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, Cfg::kTmemCols);
}

}  // namespace qt2
