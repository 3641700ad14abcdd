// msed_kernel.cuh -- MS-EDEN producer of the backward views (sm_100a).
//
// Citations (page title, then section):
//   [QII-th] "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992): "Question 1"
//            (fixed 128-dim rotation groups, one shared rotation and seed).
//   [QII-tg] Quartet II digest (quant_prune_distill post 640): "Method" (random Hadamard rotation,
//            the EDEN factor <x,x>/<Q(Rx),Rx>, stochastically rounded FP8 scales).
//   [FAF]    "Format-Aware Fusion for Fast FP4 Pretraining" (rit.work blog): one producer emits
//            both layouts the backward GEMMs need from a single read of the tensor.
//
// Per 128-block of the grouped axis: y = H D x (unnormalised Sylvester butterfly, strides 1..64);
// per 16-group p = max|y|/6 and codes = RNE_E2M1(y * (1/p)); per block
// S = sum y^2 / sum p * <val, y>; the pre-scale S*p is written (fp32, tensor-core scale order)
// for the finalize pass and the view max |y| merged with atomicMax.  Every floating-point
// step is one IEEE binary32 operation rounded to nearest-even in the reference order; the packed
// f32x2 forms below are two such operations side by side.
//
// Design: persistent CTAs of 256 threads; each thread rotates and quantizes one 128-element
// vector per tile entirely in registers (64 packed fp32 pairs).  Tiles stream in by TMA
// (128-byte swizzle, two-deep ring) while the previous one is processed:
//   both views : 128x128 tiles, threads 0..127 take rows, 128..255 take columns;
//   rows only  : 256x128 tiles (128x128 when rows % 256 != 0), one row per thread;
//   columns only: 128x256 tiles (128x128 when cols % 256 != 0), one column per thread.
#pragma once

#include "quant_kernels.cuh"

namespace qt2 {

// Butterfly stages with strides 2..64 on P[j] = (y[2j], y[2j+1]) (stride 1 is done on input).
__device__ __forceinline__ void fwht_packed_tail(uint64_t (&P)[64]) {
#pragma unroll
    for (int hp = 1; hp < 64; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            if ((j & hp) == 0) {
                const uint64_t a = P[j], b = P[j + hp];
                P[j] = f2_add(a, b);
                P[j + hp] = f2_sub(a, b);
            }
        }
    }
}

// Quantize one rotated 128-block held as packed pairs: 16 code words (element 8w+i in nibble i
// of word w), 8 pre-scales S*p, running max of |y|.
__device__ __forceinline__ void msed_quantize_packed(const uint64_t (&P)[64], uint32_t (&cw)[16], float (&Pq)[8],
                                                     float &amax) {
    float nq[8], ptq[8], pq[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float y[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) f2_split(P[8 * q + i], y[2 * i], y[2 * i + 1]);
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(y[2 * i]), fabsf(y[2 * i + 1]));
#pragma unroll
        for (int w = 8; w > 1; w >>= 1) {
#pragma unroll
            for (int i = 0; i < w / 2; ++i) m8[i] = fmaxf(m8[2 * i], m8[2 * i + 1]);
        }
        const float a = m8[0];     // max is exact: the evaluation order does not matter
        amax = fmaxf(amax, a);
        const bool live = a >= kTiny;
        const float p = live ? __fdiv_rn(a, 6.0f) : 0.0f;
        const float r = live ? __frcp_rn(p) : 0.0f;          // flushed group: sign-preserving zeros
        const uint64_t rr = f2(r, r);
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) f2_split(f2_mul(P[8 * q + i], rr), v[2 * i], v[2 * i + 1]);
        float val[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float vh[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) vh[i] = v[8 * h + i];
            cw[2 * q + h] = e2m1x8(vh);
            float dv[8];
            e2m1x8_values(cw[2 * q + h], dv);
#pragma unroll
            for (int i = 0; i < 8; ++i) val[8 * h + i] = dv[i];
        }
        // products val*y and y*y, then the 16-term trees; level 1 pairs adjacent elements,
        // levels 2..4 run on (t, n) packed together
        uint64_t tn[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float t0, t1, n0, n1;
            f2_split(f2_mul(f2(val[2 * i], val[2 * i + 1]), P[8 * q + i]), t0, t1);
            f2_split(f2_mul(P[8 * q + i], P[8 * q + i]), n0, n1);
            tn[i] = f2(__fadd_rn(t0, t1), __fadd_rn(n0, n1));
        }
#pragma unroll
        for (int w = 8; w > 1; w >>= 1) {
#pragma unroll
            for (int i = 0; i < w / 2; ++i) tn[i] = f2_add(tn[2 * i], tn[2 * i + 1]);
        }
        float tg, ng;
        f2_split(tn[0], tg, ng);
        pq[q] = p;
        nq[q] = live ? ng : 0.0f;
        ptq[q] = live ? __fmul_rn(p, tg) : 0.0f;
    }
    const float num = tree_sum<8>(nq), den = tree_sum<8>(ptq);
    const float S = den > 0.0f ? __fdiv_rn(num, den) : 1.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) Pq[q] = __fmul_rn(S, pq[q]);
}

__device__ __forceinline__ void msed_store(uint8_t *codes_dst, float *P_base, int64_t vr, int64_t j0, int64_t VC,
                                           const uint32_t (&cw)[16], const float (&P)[8]) {
    uint4 *dst = reinterpret_cast<uint4 *>(codes_dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]);
    *reinterpret_cast<float4 *>(P_base + sf_offset(vr, j0, VC)) = make_float4(P[0], P[1], P[2], P[3]);
    *reinterpret_cast<float4 *>(P_base + sf_offset(vr, j0 + 4, VC)) = make_float4(P[4], P[5], P[6], P[7]);
}

// Byte offset of tile element (r, c) in a buffer of 128x64 boxes loaded with the 128-byte swizzle.
template <int TC>
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    const int box = (r >> 7) * (TC / 64) + (c >> 6), rr = r & 127;
    return (uint32_t)(box * 16384 + rr * 128 + ((((c & 63) >> 3) ^ (rr & 7)) << 4) + ((c & 7) << 1));
}

template <int TR, int TC, bool DO_ROW, bool DO_COL>
__global__ void __launch_bounds__(256, 1)
    msed_kernel(const __grid_constant__ CUtensorMap tmap, int64_t R, int64_t C, uint64_t seed,
                uint8_t *__restrict__ row_codes, float *__restrict__ row_P, uint32_t *__restrict__ row_amax,
                uint8_t *__restrict__ col_codes, float *__restrict__ col_P, uint32_t *__restrict__ col_amax) {
    constexpr int kTileBytes = TR * TC * 2;
    constexpr int kBoxes = (TR / 128) * (TC / 64);
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *buf0 = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ uint32_t pair_mask[64];   // row view: sign bits of elements 2j, 2j+1 at bits 15 and 31
    __shared__ uint32_t elem_mask[128];  // column view: sign bit of element i at bit 31
    __shared__ uint32_t red[2][8];

    const int t = threadIdx.x;
    const int64_t tiles_c = C / TC, ntiles = (R / TR) * tiles_c;
    const uint32_t bar0 = smem_u32(&bar[0]);
    if (t == 0) {
        prefetch_tmap(&tmap);
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        fence_mbar_init();
    }
    {
        const uint4 sw = rotation_sign_words(seed);   // bit i of the 128 signs: element i negated
        const uint32_t w[4] = {sw.x, sw.y, sw.z, sw.w};
        if (t < 128) elem_mask[t] = ((w[t >> 5] >> (t & 31)) & 1u) << 31;
        if (t < 64) {
            const int e = 2 * t;
            pair_mask[t] = (((w[e >> 5] >> (e & 31)) & 1u) << 15) | (((w[(e + 1) >> 5] >> ((e + 1) & 31)) & 1u) << 31);
        }
    }
    __syncthreads();

    auto issue = [&](int64_t tile, int b) {
        const int32_t r0 = (int32_t)((tile / tiles_c) * TR), c0 = (int32_t)((tile % tiles_c) * TC);
        const uint32_t fb = bar0 + 8 * b;
        mbar_arrive_expect_tx(fb, kTileBytes);
#pragma unroll
        for (int br = 0; br < TR / 128; ++br)
#pragma unroll
            for (int bc = 0; bc < TC / 64; ++bc)
                tma_load_2d(smem_u32(buf0 + b * kTileBytes + (br * (TC / 64) + bc) * 16384), &tmap, c0 + 64 * bc,
                            r0 + 128 * br, fb);
    };
    int issued = 0;
    if (t == 0) {
        for (int b = 0; b < 2; ++b) {
            const int64_t tile = blockIdx.x + (int64_t)b * gridDim.x;
            if (tile < ntiles) {
                issue(tile, b);
                issued = b + 1;
            }
        }
    }
    (void)kBoxes;

    float amax_r = 0.0f, amax_c = 0.0f;
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        const int b = i & 1;
        const bool ok = mbar_wait(bar0 + 8 * b, (i >> 1) & 1);
        if (__syncthreads_or(!ok)) break;
        const uint8_t *tb = buf0 + b * kTileBytes;
        const int64_t r0 = (tile / tiles_c) * TR, c0 = (tile % tiles_c) * TC;
        const bool row_thread = DO_ROW && (DO_COL ? t < 128 : t < TR);
        const bool col_thread = DO_COL && (DO_ROW ? t >= 128 : t < TC);
        if (row_thread || col_thread) {
            // Only the loads and the stores differ between a row vector and a column vector; the
            // rotation and quantization below are one code path for both (instruction-cache reuse).
            uint64_t P[64];
            if (row_thread) {
                const int rr = t;   // row of the tile; its 128-block is the whole tile width (TC = 128)
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(tb + tile_off<TC>(rr, 8 * c));
                    const uint4 m = *reinterpret_cast<const uint4 *>(&pair_mask[4 * c]);
                    const uint32_t w[4] = {v.x ^ m.x, v.y ^ m.y, v.z ^ m.z, v.w ^ m.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float x0 = bf16_lo(w[k]), x1 = bf16_hi(w[k]);
                        P[4 * c + k] = f2(__fadd_rn(x0, x1), __fsub_rn(x0, x1));
                    }
                }
            } else {
                const int cc = DO_ROW ? t - 128 : t;   // column of the tile; its 128-block is rows 0..127
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const uint32_t u0 = *reinterpret_cast<const uint16_t *>(tb + tile_off<TC>(2 * j, cc));
                    const uint32_t u1 = *reinterpret_cast<const uint16_t *>(tb + tile_off<TC>(2 * j + 1, cc));
                    const float x0 = __uint_as_float((u0 << 16) ^ elem_mask[2 * j]);
                    const float x1 = __uint_as_float((u1 << 16) ^ elem_mask[2 * j + 1]);
                    P[j] = f2(__fadd_rn(x0, x1), __fsub_rn(x0, x1));
                }
            }
            fwht_packed_tail(P);
            uint32_t cw[16];
            float Pq[8];
            float vmax = 0.0f;
            msed_quantize_packed(P, cw, Pq, vmax);
            if (row_thread) {
                amax_r = fmaxf(amax_r, vmax);
                const int64_t vr = r0 + t;
                msed_store(row_codes + vr * (C >> 1) + (c0 >> 1), row_P, vr, c0 >> 4, C, cw, Pq);
            } else {
                amax_c = fmaxf(amax_c, vmax);
                const int64_t vr = c0 + (DO_ROW ? t - 128 : t);   // row of the transposed view [C][R]
                msed_store(col_codes + vr * (R >> 1) + (r0 >> 1), col_P, vr, r0 >> 4, R, cw, Pq);
            }
        }
        __syncthreads();   // every thread is done with this buffer
        if (t == 0) {
            const int64_t next = tile + 2 * (int64_t)gridDim.x;
            if (next < ntiles) {
                issue(next, b);
                issued = i + 3;
            }
        }
    }
    if (t == 0) {
        // Only after a timeout can loads still be in flight: wait (bounded) for them.
        for (int k = i; k < issued; ++k) mbar_wait(bar0 + 8 * (k & 1), (k >> 1) & 1);
    }
    const uint32_t br = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_r));
    const uint32_t bc = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_c));
    if ((t & 31) == 0) {
        red[0][t >> 5] = br;
        red[1][t >> 5] = bc;
    }
    __syncthreads();
    if (t == 0) {
        uint32_t mr = 0, mc = 0;
        for (int k = 0; k < 8; ++k) {
            mr = max(mr, red[0][k]);
            mc = max(mc, red[1][k]);
        }
        if (DO_ROW) atomicMax(row_amax, mr);
        if (DO_COL) atomicMax(col_amax, mc);
    }
}

}  // namespace qt2
