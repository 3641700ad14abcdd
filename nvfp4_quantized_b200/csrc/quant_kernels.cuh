// quant_kernels.cuh -- the HBM-bound producers of the NVFP4 views (sm_100a).
//
// Citations (page title, then section):
//   [QII-th] "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992): "Question 1"
//            (fixed 128-dim rotation groups, shared rotation and seed, no SR of tiny FP8 scales).
//   [QII-tg] Quartet II digest (quant_prune_distill post 640): "Method" (EDEN rotation and factor,
//            stochastically rounded FP8 scales, the 4/6 grid choice, 1x16 groups).
//   [FAF]    "Format-Aware Fusion for Fast FP4 Pretraining" (rit.work blog): "the speed-up is lost
//            between the matmuls" (global max is a sync point; one producer emits both layouts).
//
// Arithmetic contract: every floating-point step is one IEEE binary32 operation rounded to
// nearest-even (explicit __fmul_rn/__fadd_rn/__fsub_rn/__fdiv_rn/__frcp_rn, never contracted),
// and sums are balanced binary trees over contiguous power-of-two index ranges, so the codes
// and scales are a deterministic function of the input.
#pragma once

#include "qt2_device.cuh"

namespace qt2 {

template <int N>
__device__ __forceinline__ float tree_sum(const float *v) {
    float t[N];
#pragma unroll
    for (int i = 0; i < N; ++i) t[i] = v[i];
#pragma unroll
    for (int w = N; w > 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w / 2; ++i) t[i] = __fadd_rn(t[2 * i], t[2 * i + 1]);
    }
    return t[0];
}

// ---------------------------------------------------------------------------------------------
// Tensor max |x| of a bf16 matrix ([FAF]: global NVFP4 scales need the tensor-wide maximum).
// Magnitudes of finite bf16 values order like their bit patterns with the sign cleared, so the
// max is taken on integers; the result is an fp32 bit pattern merged with atomicMax into a word
// that the caller zeroed.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t *__restrict__ x, int64_t R, int64_t C,
                                                        int64_t ld, uint32_t *__restrict__ amax_word) {
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t vec_per_row = C >> 3;
    uint32_t m = 0;
    for (int64_t r = gwarp; r < R; r += nwarps) {
        const uint4 *row = reinterpret_cast<const uint4 *>(x + r * ld);
#pragma unroll 4
        for (int64_t v = lane; v < vec_per_row; v += 32) {
            uint4 w = __ldcs(row + v);
            m = __vmaxu2(m, w.x & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.y & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.w & 0x7FFF7FFFu);
        }
    }
    uint32_t bits = max(m & 0xFFFFu, m >> 16) << 16;   // bf16 -> fp32 bit pattern
    bits = __reduce_max_sync(0xFFFFFFFFu, bits);
    __shared__ uint32_t wmax[8];
    if (lane == 0) wmax[threadIdx.x >> 5] = bits;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b = max(b, wmax[i]);
        if (b) atomicMax(amax_word, b);
    }
}

// ---------------------------------------------------------------------------------------------
// Forward quantizer, row view: RTN onto E2M1 with the 4/6 grid choice per 1x16 group
// ([QII-tg] "Method"; [QII-th] "fairness" answer: the forward pass uses RTN).
// One thread per 16-element group; a warp covers 32 consecutive groups of one row.
// ---------------------------------------------------------------------------------------------
struct Fwd46Candidate {
    uint32_t codes[2];
    uint32_t scale;
    float err;
};

// Candidate with grid maximum k: s = RNE_E4M3(a/(g*k)), d = s*g, codes = RNE_E2M1(x*(1/d)),
// err = tree sum of (x - val*d)^2.  A zero scale gives sign-preserving zero codes (x*0) and
// err = sum x^2.
__device__ __forceinline__ Fwd46Candidate fwd46_candidate(const float (&x)[16], float a, float g, float k) {
    Fwd46Candidate c;
    const float t = __fdiv_rn(a, __fmul_rn(g, k));
    c.scale = e4m3_rne(t);
    const float d = __fmul_rn(e4m3_value(c.scale), g);
    const float r = (c.scale == 0) ? 0.0f : __frcp_rn(d);
    float sq[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(x[8 * h + i], r);
        c.codes[h] = e2m1x8(q);
        float val[8];
        e2m1x8_values(c.codes[h], val);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float e = __fsub_rn(x[8 * h + i], __fmul_rn(val[i], d));
            sq[8 * h + i] = __fmul_rn(e, e);
        }
    }
    c.err = tree_sum<16>(sq);
    return c;
}

__global__ void __launch_bounds__(256) fwd46_rows_kernel(const uint16_t *__restrict__ x, int64_t R, int64_t C,
                                                         int64_t ld, const uint32_t *__restrict__ amax_word,
                                                         uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                         float *__restrict__ tensor_scale) {
    const float A = __uint_as_float(*amax_word);
    const bool zero_tensor = !(A >= kTiny);
    const float g = zero_tensor ? 1.0f : __fdiv_rn(A, kFwd46Denominator);
    if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = g;

    const uint32_t G = (uint32_t)(C >> 4);                 // groups per row (a multiple of 8)
    const uint64_t total = (uint64_t)R * G;                // a multiple of 1024
    const int lane = threadIdx.x & 31;
    for (uint64_t gi = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < total;
         gi += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t r = gi / G;
        const uint32_t q = (uint32_t)(gi - r * G);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + r * ld + (uint64_t)q * 16);
        const uint4 w0 = __ldcs(src), w1 = __ldcs(src + 1);
        const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        float xv[16];
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            xv[2 * i] = bf16_lo(w[i]);
            xv[2 * i + 1] = bf16_hi(w[i]);
            a = fmaxf(a, fmaxf(fabsf(xv[2 * i]), fabsf(xv[2 * i + 1])));
        }
        const Fwd46Candidate c6 = fwd46_candidate(xv, a, g, 6.0f);
        const Fwd46Candidate c4 = fwd46_candidate(xv, a, g, 4.0f);
        const bool pick4 = c4.err < c6.err;                 // a tie keeps the full grid
        const uint32_t code0 = pick4 ? c4.codes[0] : c6.codes[0];
        const uint32_t code1 = pick4 ? c4.codes[1] : c6.codes[1];
        const uint32_t s = pick4 ? c4.scale : c6.scale;
        *reinterpret_cast<uint2 *>(codes + r * (uint64_t)(C >> 1) + (uint64_t)q * 8) = make_uint2(code0, code1);
        // four consecutive groups (same row, q % 4 == 0 .. 3) share one scale word
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, s, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, s, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, s, 3);
        if ((lane & 3) == 0)
            *reinterpret_cast<uint32_t *>(scales + sf_offset((int64_t)r, q, C)) = s | (s1 << 8) | (s2 << 16) | (s3 << 24);
    }
}

// ---------------------------------------------------------------------------------------------
// MS-EDEN producer ([QII-tg] "Method"; [QII-th] "Question 1"; [FAF]: both layouts in one pass).
// One CTA of 128 threads per 128x128 tile, loaded once by TMA (128-byte swizzle, two boxes of
// 64 columns).  Row view: thread t rotates and quantizes row t of the tile (a 128-block along
// the columns).  Column view: thread t does column t (a 128-block along the rows), giving row
// t of the transposed view.  Per 128-block: y = H D x, per group p = max|y|/6 and codes =
// RNE_E2M1(y * (1/p)), per block S = sum y^2 / sum p * <val, y>; the pre-scale S*p goes to
// the workspace (fp32, scale-factor order) and the view max |y| to an atomicMax word.
// ---------------------------------------------------------------------------------------------

// Unnormalised Walsh-Hadamard butterfly, strides 1..64, (a+b, a-b) with a at the lower index.
__device__ __forceinline__ void fwht128(float (&y)[128]) {
#pragma unroll
    for (int h = 1; h < 128; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
            if ((i & h) == 0) {
                const float a = y[i], b = y[i + h];
                y[i] = __fadd_rn(a, b);
                y[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

// Quantize one rotated 128-block: 16 code words (element 8w+i in nibble i of word w), 8 pre-scales.
__device__ __forceinline__ void msed_block(float (&y)[128], uint32_t (&cw)[16], float (&P)[8], float &amax) {
    float nq[8], ptq[8], pq[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(y[16 * q + i]));
        amax = fmaxf(amax, a);
        const bool live = a >= kTiny;
        const float p = live ? __fdiv_rn(a, 6.0f) : 0.0f;
        const float r = live ? __frcp_rn(p) : 0.0f;          // flushed group: sign-preserving zeros
        float tv[16], nv[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(y[16 * q + 8 * h + i], r);
            cw[2 * q + h] = e2m1x8(v);
            float val[8];
            e2m1x8_values(cw[2 * q + h], val);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float yi = y[16 * q + 8 * h + i];
                tv[8 * h + i] = __fmul_rn(val[i], yi);
                nv[8 * h + i] = __fmul_rn(yi, yi);
            }
        }
        pq[q] = p;
        nq[q] = live ? tree_sum<16>(nv) : 0.0f;
        ptq[q] = live ? __fmul_rn(p, tree_sum<16>(tv)) : 0.0f;
    }
    const float num = tree_sum<8>(nq), den = tree_sum<8>(ptq);
    const float S = den > 0.0f ? __fdiv_rn(num, den) : 1.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) P[q] = __fmul_rn(S, pq[q]);
}

// The 128 rotation signs: bit i of Philox(seed, tensor id 0) word i/32 set -> negate element i.
__device__ __forceinline__ uint4 rotation_sign_words(uint64_t seed) { return philox_block(seed, 0u, 0ull); }

__device__ __forceinline__ uint32_t sign_bit(const uint4 &sw, int i) {
    const uint32_t w = (i < 32) ? sw.x : (i < 64) ? sw.y : (i < 96) ? sw.z : sw.w;
    return ((w >> (i & 31)) & 1u) << 31;
}

__device__ __forceinline__ void store_block(uint8_t *codes_dst, float *P_base, int64_t vr, int64_t j0, int64_t VC,
                                            const uint32_t (&cw)[16], const float (&P)[8]) {
    uint4 *dst = reinterpret_cast<uint4 *>(codes_dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]);
    *reinterpret_cast<float4 *>(P_base + sf_offset(vr, j0, VC)) = make_float4(P[0], P[1], P[2], P[3]);
    *reinterpret_cast<float4 *>(P_base + sf_offset(vr, j0 + 4, VC)) = make_float4(P[4], P[5], P[6], P[7]);
}

template <bool DO_ROW, bool DO_COL>
__global__ void __launch_bounds__(128) msed_tile_kernel(const __grid_constant__ CUtensorMap tmap, int64_t R, int64_t C,
                                                        uint64_t seed, uint8_t *__restrict__ row_codes,
                                                        float *__restrict__ row_P, uint32_t *__restrict__ row_amax,
                                                        uint8_t *__restrict__ col_codes, float *__restrict__ col_P,
                                                        uint32_t *__restrict__ col_amax) {
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *tile = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t red[2][4];

    const int t = threadIdx.x;
    const int64_t c0 = (int64_t)blockIdx.x * 128, r0 = (int64_t)blockIdx.y * 128;
    const uint32_t bar_a = smem_u32(&bar);
    if (t == 0) {
        prefetch_tmap(&tmap);
        mbar_init(bar_a, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
        mbar_arrive_expect_tx(bar_a, 128 * 128 * 2);
        tma_load_2d(smem_u32(tile), &tmap, (int32_t)c0, (int32_t)r0, bar_a);
        tma_load_2d(smem_u32(tile + 16384), &tmap, (int32_t)(c0 + 64), (int32_t)r0, bar_a);
    }
    const uint4 sw = rotation_sign_words(seed);
    const bool ok = mbar_wait(bar_a, 0);

    float amax_r = 0.0f, amax_c = 0.0f;
    if (ok && DO_ROW) {
        // row t: 16 chunks of 8 bf16; chunk c of box h sits at chunk position c ^ (t & 7)
        float y[128];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = *reinterpret_cast<const uint4 *>(tile + h * 16384 + t * 128 + ((c ^ (t & 7)) << 4));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = 64 * h + 8 * c + 2 * i;
                    y[e] = __uint_as_float(__float_as_uint(bf16_lo(w[i])) ^ sign_bit(sw, e));
                    y[e + 1] = __uint_as_float(__float_as_uint(bf16_hi(w[i])) ^ sign_bit(sw, e + 1));
                }
            }
        }
        fwht128(y);
        uint32_t cw[16];
        float P[8];
        msed_block(y, cw, P, amax_r);
        const int64_t vr = r0 + t;
        store_block(row_codes + vr * (C >> 1) + (c0 >> 1), row_P, vr, c0 >> 4, C, cw, P);
    }
    if (ok && DO_COL) {
        // column t: element i is row i of the tile
        const int h = t >> 6, cc = t & 63;
        const uint8_t *base = tile + h * 16384 + ((cc & 7) << 1);
        float y[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) {
            const uint16_t b = *reinterpret_cast<const uint16_t *>(base + i * 128 + ((((cc >> 3) ^ (i & 7))) << 4));
            y[i] = __uint_as_float((((uint32_t)b) << 16) ^ sign_bit(sw, i));
        }
        fwht128(y);
        uint32_t cw[16];
        float P[8];
        msed_block(y, cw, P, amax_c);
        const int64_t vr = c0 + t;                 // row of the transposed view [C][R]
        store_block(col_codes + vr * (R >> 1) + (r0 >> 1), col_P, vr, r0 >> 4, R, cw, P);
    }
    // view maxima: warp reduce, then one atomicMax per CTA
    const uint32_t br = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_r));
    const uint32_t bc = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_c));
    if ((t & 31) == 0) {
        red[0][t >> 5] = br;
        red[1][t >> 5] = bc;
    }
    __syncthreads();
    if (t == 0) {
        if (DO_ROW) atomicMax(row_amax, max(max(red[0][0], red[0][1]), max(red[0][2], red[0][3])));
        if (DO_COL) atomicMax(col_amax, max(max(red[1][0], red[1][1]), max(red[1][2], red[1][3])));
    }
}

// ---------------------------------------------------------------------------------------------
// MS-EDEN scale finalize: group scale = SR_E4M3(S*p*(1/g)) with g = A/1536 ([QII-tg] "Method":
// the scales are stochastically rounded to FP8), RNE below 2^-6 ([QII-th] "Question 1").
// One thread per 4-group scale word; P is read in the same scale-factor order, so both the
// 16-byte reads and the 4-byte writes are contiguous across a warp.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) msed_finalize_kernel(const float4 *__restrict__ P, int64_t VR, int64_t VC,
                                                            const uint32_t *__restrict__ amax_word, uint64_t seed,
                                                            uint32_t tid, uint32_t *__restrict__ scale_words,
                                                            float *__restrict__ tensor_scale) {
    const float A = __uint_as_float(*amax_word);
    const float g = (A >= kTiny) ? __fdiv_rn(A, kMsedDenominator) : 1.0f;
    const float ginv = __frcp_rn(g);
    if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = g;
    const int64_t words = (VR * VC) >> 6;
    const int64_t atoms_per_rowblock = VC >> 6;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += (int64_t)gridDim.x * blockDim.x) {
        const int64_t atom = w >> 7, wi = w & 127;
        const int64_t r = (atom / atoms_per_rowblock) * 128 + (wi & 3) * 32 + (wi >> 2);
        const int64_t j4 = atom % atoms_per_rowblock;        // groups 4*j4 .. 4*j4+3 of view row r
        const float4 p = __ldcs(P + w);
        const uint4 u = philox_block(seed, tid, (uint64_t)(r * atoms_per_rowblock + j4));
        const float pv[4] = {p.x, p.y, p.z, p.w};
        const uint32_t uv[4] = {u.x, u.y, u.z, u.w};
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float v = __fmul_rn(pv[k], ginv);
            const uint32_t s = (v < kSrCutoff) ? e4m3_rne(v) : e4m3_sr(v, uv[k]);
            word |= s << (8 * k);
        }
        scale_words[w] = word;
    }
}

}  // namespace qt2
