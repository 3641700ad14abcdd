// gemm_kernel.cuh -- block-scaled NVFP4 GEMM on the 5th-generation tensor cores (sm_100a).
//
// "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992), abstract and §1:
// NVFP4 (E2M1 values with FP8 block scales) is natively supported by Blackwell tensor cores,
// which multiply it at several times the FP8 rate.
//
// C[m][n] = alpha * gA * gB * sum_k val(A[m][k]) sA(m, k/16) * val(B[n][k]) sB(n, k/16)
// with both operands K-major ("TN"), 1x16 E4M3 scales, fp32 accumulation in tensor memory.
//
// Design (one CTA of 128 threads per 128 x BN output tile):
//   warp 0             : producer -- TMA loads of the A/B code tiles (128-byte swizzle, no
//                        multicast) and bulk copies of the 512-byte scale atoms into a ring of
//                        STAGES shared-memory stages, each covering K = 256.
//   warp 1             : MMA issuer -- per stage, tcgen05.cp of the scale atoms into TMEM
//                        (replicated into the four lane quadrants), then four
//                        tcgen05.mma.kind::mxf4nvf4.block_scale (K = 64 each); tcgen05.commit
//                        frees the stage once those MMAs have completed.
//   warp 2             : allocates and frees the TMEM columns.
//   all four warps     : epilogue -- tcgen05.ld of the fp32 accumulator (warp w owns lanes
//                        32w..32w+31 = tile rows), scale by alpha*gA*gB, store bf16 or fp32.
// Warps 0 and 1 run converged and let one lane chosen by elect.sync issue (TMA, bulk copies and
// tcgen05 instructions take warp-uniform operands; issued from a lone lane of a diverged warp
// each pays extra issue work).
// Every wait is bounded (mbar_wait); a timeout records QT2_ERR_TIMEOUT and the CTA still
// reaches the common exit, frees its TMEM and returns.
#pragma once

#include "qt2_device.cuh"

namespace qt2 {

constexpr int kGemmBM = 128;
constexpr int kGemmBKBytes = 128;   // 256 fp4 elements per stage per row
constexpr int kGemmThreads = 128;

template <int BN>
struct GemmCfg {
    static constexpr int kStages = (BN == 256) ? 4 : 6;
    static constexpr int kABytes = kGemmBM * kGemmBKBytes;          // 16 KB
    static constexpr int kBBytes = BN * kGemmBKBytes;               // 32 or 16 KB
    static constexpr int kSfaBytes = 4 * 512;                       // 4 k-blocks x one atom
    static constexpr int kSfbBytes = (BN / 128) * 4 * 512;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kTmemCols = (BN == 256) ? 512 : 256;       // acc BN + 16 (SFA) + BN/8 (SFB)
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
    // instruction descriptor: E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 128, N = BN
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                       ((uint32_t)(kGemmBM >> 4) << 24);
};

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfb, const float *__restrict__ gA,
                      const float *__restrict__ gB, float alpha, void *__restrict__ Cout, int64_t ldc, int K,
                      int c_dtype, int local) {
    using Cfg = GemmCfg<BN>;
    constexpr int S = Cfg::kStages;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = sA + S * Cfg::kABytes;
    uint8_t *sSFA = sB + S * Cfg::kBBytes;
    uint8_t *sSFB = sSFA + S * Cfg::kSfaBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSFB + S * Cfg::kSfbBytes);   // full[S], empty[S], accum
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 1);
    int *consumed_slot = reinterpret_cast<int *>(tmem_slot + 1);   // stages the MMA thread waited for

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * kGemmBM, n0 = (int64_t)blockIdx.x * BN;
    const int nkb = K >> 6;                         // 64-element k-blocks
    const int nks = (nkb + 3) >> 2;                 // stages of up to 4 k-blocks
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S), accum_bar = smem_u32(bars + 2 * S);

    int issued = 0;   // producer only: stages whose loads were issued
    if (threadIdx.x == 0) {
        *consumed_slot = 0;
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(accum_bar, 1);
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_acc = tmem, t_sfa = tmem + BN, t_sfb = tmem + BN + 16;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (whole warp,
        // one elected lane issues: TMA and bulk copies take warp-uniform operands)
        const uint8_t *sfa_blk = sfa + (m0 >> 7) * (int64_t)nkb * 512;
        for (int ks = 0; ks < nks; ++ks) {
            const int s = ks % S;
            if (ks >= S && !mbar_wait_warp(empty0 + 8 * s, ((ks / S) & 1) ^ 1)) break;
            const int kb0 = ks * 4, nk = min(4, nkb - kb0);
            const uint32_t fb = full0 + 8 * s;
            if (elect_one()) {
                mbar_arrive_expect_tx(fb, Cfg::kABytes + Cfg::kBBytes + nk * 512 * (1 + BN / 128));
                tma_load_2d(smem_u32(sA + s * Cfg::kABytes), &tmA, ks * kGemmBKBytes, (int32_t)m0, fb);
                tma_load_2d(smem_u32(sB + s * Cfg::kBBytes), &tmB, ks * kGemmBKBytes, (int32_t)n0, fb);
                bulk_load(smem_u32(sSFA + s * Cfg::kSfaBytes), sfa_blk + (int64_t)kb0 * 512, nk * 512, fb);
#pragma unroll
                for (int h = 0; h < BN / 128; ++h)
                    bulk_load(smem_u32(sSFB + s * Cfg::kSfbBytes + h * 2048),
                              sfb + (((n0 >> 7) + h) * (int64_t)nkb + kb0) * 512, nk * 512, fb);
            }
            __syncwarp();
            issued = ks + 1;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (whole warp,
        // one elected lane issues)
        for (int ks = 0; ks < nks; ++ks) {
            const int s = ks % S;
            if (!mbar_wait_warp(full0 + 8 * s, (ks / S) & 1)) break;
            if (lane == 0) *consumed_slot = ks + 1;
            tc_fence_after();
            const int nk = min(4, nkb - ks * 4);
            const uint32_t a_s = smem_u32(sA + s * Cfg::kABytes), b_s = smem_u32(sB + s * Cfg::kBBytes);
            const uint32_t sfa_s = smem_u32(sSFA + s * Cfg::kSfaBytes), sfb_s = smem_u32(sSFB + s * Cfg::kSfbBytes);
            if (elect_one()) {
                for (int kk = 0; kk < nk; ++kk) {
                    tc_cp_32x128b_warpx4(t_sfa + 4 * kk, make_smem_desc(sfa_s + 512 * kk, 0, 128, 0));
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h)
                        tc_cp_32x128b_warpx4(t_sfb + (BN / 32) * kk + 4 * h,
                                             make_smem_desc(sfb_s + 2048 * h + 512 * kk, 0, 128, 0));
                }
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t adesc = make_smem_desc(a_s + 32 * kk, 16, 1024, 2);
                    const uint64_t bdesc = make_smem_desc(b_s + 32 * kk, 16, 1024, 2);
                    tc_mma_nvfp4(t_acc, adesc, bdesc, Cfg::kIdesc, t_sfa + 4 * kk, t_sfb + (BN / 32) * kk,
                                 (ks | kk) != 0);
                }
                tc_commit(empty0 + 8 * s);
            }
            __syncwarp();
        }
        if (elect_one()) tc_commit(accum_bar);
    }
    __syncwarp();

    // -------------------------------------------------------------------- epilogue
    const bool acc_ok = mbar_wait_warp(accum_bar, 0);
    tc_fence_after();
    if (acc_ok) {
        const int64_t row = m0 + warp * 32 + lane;
        const uint32_t t_row = t_acc + ((uint32_t)(warp * 32) << 16);
        // checked build: this thread's BN outputs must lie inside C ((M - 1) * ldc + N elements,
        // M and N from the grid); the TMEM loads below stay warp-collective either way
        const int64_t esz = c_dtype == QT2_DTYPE_F32 ? 4 : 2;
        const bool st_ok = QT2_STORE_OK(static_cast<uint8_t *>(Cout) + (row * ldc + n0) * esz, BN * esz, Cout,
                                        (((int64_t)gridDim.y * kGemmBM - 1) * ldc + (int64_t)gridDim.x * BN) * esz);
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
            // tensor scales: one each, or (CTA-local views) one per 128 rows of A and of B
            const float sc = local ? alpha * gA[m0 >> 7] * gB[(n0 + c) >> 7] : alpha * (*gA) * (*gB);
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_row + c, v);
            tmem_ld_wait();
            if (!st_ok) continue;
            if (c_dtype == QT2_DTYPE_F32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(Cout) + row * ldc + n0 + c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]) * sc, __uint_as_float(v[4 * i + 1]) * sc,
                                         __uint_as_float(v[4 * i + 2]) * sc, __uint_as_float(v[4 * i + 3]) * sc);
            } else {
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * sc,
                                                              __uint_as_float(v[2 * i + 1]) * sc);
                    packed[i] = *reinterpret_cast<uint32_t *>(&b2);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(Cout) + row * ldc + n0 + c);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        // Only after a timeout can loads still be in flight: wait (bounded) for each of them
        // before the CTA's shared memory is released.
        for (int ks = *consumed_slot; ks < issued; ++ks) mbar_wait(full0 + 8 * (ks % S), (ks / S) & 1);
    }
    if (warp == 2) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace qt2
