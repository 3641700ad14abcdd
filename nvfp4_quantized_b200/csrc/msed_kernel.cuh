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
// f32x2 forms below are two such operations side by side, and an FMA whose product is an exact
// +-1 multiple is one rounded addition or subtraction.
//
// Design: persistent CTAs of 512 threads (16 warps at up to 128 registers, so an SM keeps 16
// warps in flight), 128x128 bf16 tiles streamed by TMA (128-byte swizzle) through a 3-deep ring.
// Two threads (adjacent lanes, h = 0, 1) share one 128-element vector: thread h holds elements
// [64h, 64h + 64) in 32 packed fp32 pairs and runs the butterfly strides 1..32 in registers;
// stride 64 crosses the pair with one shuffle per packed value.  A pair register holds elements
// k and k + 8 (the two halves of one 16-group), so every butterfly stage but stride 8 and every
// level but the last of the 16-term group trees run on packed f32x2 instructions.  Register
// slot m holds element k = (m & 7) | ((m >> 3) & 1) << 4 | (((m >> 4) & 1) ^ h) << 5 of the
// thread's half (and k + 8): thread 1 keeps its two 32-element quarters swapped, so that the
// cross step is the same instructions on both threads -- it turns thread 1's stride-32 and
// stride-64 subtractions around, and an FMA with sigma = +-1 gives each thread its own operand
// order exactly (signed zeros included).  After the butterfly thread h owns the 16-groups
// {2h, 2h+1} and {4+2h, 5+2h} of the block and quantizes them; the block sums for S meet
// through two more shuffles.
//   both views : warps 0..7 take the rows of each tile, warps 8..15 its columns;
//   one view   : warps 0..7 and 8..15 take alternate tiles.
// A ring stage is refilled by the last warp that has read it (a shared counter), so the two
// halves of the CTA drift freely by up to the ring depth.
//
// The same producer serves the elementwise-SR baseline (qt2_quant_sr): kModeMax merges max |y|
// of the rotated view(s) and writes nothing else; kModeSr then quantizes with that tensor scale
// (sr_vector).  kModeEden is MS-EDEN.  kModeFwdRowEdenCol gives both of X's views from one read
// ([FAF]): the row warps quantize the tile's rows for the forward GEMM (RTN with the 4/6 choice,
// as fwd46_coop_kernel, with the tensor max of X taken beforehand), the column warps produce the
// MS-EDEN column view.
#pragma once

#include "quant_kernels.cuh"

namespace qt2 {

struct MsedCfg {
    static constexpr int kThreads = 512;
    static constexpr int kTeamWarps = 8;
    static constexpr int kStages = 3;
    static constexpr int kTileBytes = 128 * 128 * 2;
    static constexpr int kSmemBytes = kStages * kTileBytes + 1024;
};

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// a / 6 rounded to nearest-even, for normal a >= 2^-100: q0 = a * RN(1/6), the remainder
// a - 6 q0 is exact in one FMA, and one FMA correction q0 + rem * RN(1/6) rounds to RN(a/6)
// (Markstein's correction step; verified exhaustively over every significand of a binade and
// over the extreme binades of the range, and exact scaling by powers of two extends it to all
// a in [2^-100, 2^128)).
__device__ __forceinline__ float div6_rn(float a) {
    constexpr float kSixth = 0.16666667163372039794921875f;   // RN(1/6) = 0x3E2AAAAB
    const float q0 = __fmul_rn(a, kSixth);
    const float rem = __fmaf_rn(-q0, 6.0f, a);
    return __fmaf_rn(rem, kSixth, q0);
}

// max(|a|, |b|, |c|) (sm_100a three-input max; exact, so the grouping does not matter).  The
// .NaN forms return NaN when an operand is NaN, so a non-finite input reaches the view max
// (y holds inf or NaN wherever a block of x held one) and is reported by the scale pass.
__device__ __forceinline__ float absmax3(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float max2n(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ uint64_t shfl_xor1_u64(uint64_t v) {
    uint32_t lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
    lo = __shfl_xor_sync(0xFFFFFFFFu, lo, 1);
    hi = __shfl_xor_sync(0xFFFFFFFFu, hi, 1);
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

// Shared-memory loads at 32-bit shared addresses.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

// RN(1/p) for normal p (2^-103 <= p < 2^126, so 1/p is normal): the hardware approximation y,
// then one correction y + y*(1 - p*y) with both steps fused multiply-adds (Markstein's
// reciprocal iteration, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34, 1990).  Checked bit for bit against the IEEE reciprocal over
// every significand of several binades (qt2_selftest_rcp).
__device__ __forceinline__ float rcp_rn(float p) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(p));
    const float e = __fmaf_rn(-p, y, 1.0f);
    return __fmaf_rn(y, e, y);
}

// Butterfly strides 2..64 of one vector held by a thread pair (stride 1 is taken as the tile is
// read).  In: P = the thread's half in slot order (see the layout above); sg = (sigma, sigma),
// nsg = -sg with sigma = +1 on thread 0 and -1 on thread 1.
__device__ __forceinline__ void rotate_tail(uint64_t (&P)[32], uint64_t sg, uint64_t nsg) {
    // strides 2, 4 (slot bits 1, 2): same order on both threads
#pragma unroll
    for (int hp = 2; hp <= 4; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if ((j & hp) == 0) {
                const uint64_t a = P[j], b = P[j + hp];
                P[j] = f2_add(a, b);
                P[j + hp] = f2_sub(a, b);
            }
        }
    }
    // stride 8: the two halves of each pair register
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float lo, hi;
        f2_split(P[j], lo, hi);
        P[j] = f2(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
    }
    // stride 16 (slot bit 3)
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if ((j & 8) == 0) {
            const uint64_t a = P[j], b = P[j + 8];
            P[j] = f2_add(a, b);
            P[j + 8] = f2_sub(a, b);
        }
    }
    // stride 32 (slot bit 4): thread 0 forms (u + v, u - v), thread 1 (its quarters swapped)
    // (v - u, v + u)
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint64_t u = P[j], v = P[j + 16];
        P[j] = f2_fma(sg, u, v);
        P[j + 16] = f2_fma(nsg, v, u);
    }
    // stride 64 across the pair: both threads send slot 16 + k and keep slot k.  Thread 0 keeps
    // the elements with bit 5 clear and receives thread 1's; thread 1 the other way round.
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const uint64_t recv = shfl_xor1_u64(P[16 + k]);
        const uint64_t keep = P[k];
        P[k] = f2_add(keep, recv);                        // y[i] = z[i] + z[i + 64]
        P[16 + k] = f2_fma(sg, keep, f2_mul(recv, nsg));  // y[i + 64] = z[i] - z[i + 64]
    }
}

// The 16 values of local group g (0..3) after rotate_tail: element i of the group is the low
// half of slot 8g + i for i < 8 and the high half of slot 8g + i - 8 for i >= 8.  Local groups
// 0, 1, 2, 3 are the block's groups 2h, 2h+1, 4+2h, 5+2h.
__device__ __forceinline__ void group_values(const uint64_t (&P)[32], int g, float (&y)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) f2_split(P[8 * g + i], y[i], y[i + 8]);
}

// max |y| of a group (NaN-propagating, see absmax3)
__device__ __forceinline__ float group_absmax(const float (&y)[16]) {
    const float m0 = absmax3(y[0], y[1], y[2]), m1 = absmax3(y[3], y[4], y[5]);
    const float m2 = absmax3(y[6], y[7], y[8]), m3 = absmax3(y[9], y[10], y[11]);
    const float m4 = absmax3(y[12], y[13], y[14]);
    return max2n(max3(m0, m1, m2), max3(m3, m4, fabsf(y[15])));
}

// Quantization of the thread's four local groups after rotate_tail.
// Out: cw[2g], cw[2g+1] = codes of local group g (element 8w+i of the group in nibble i of
// word w); Pq[g] = S * p of local group g.  amax = running max |y|.
__device__ __forceinline__ void msed_vector(uint64_t (&P)[32], uint64_t sg, uint64_t nsg, uint64_t nz,
                                            uint32_t (&cw)[8], float (&Pq)[4], float &amax) {
    rotate_tail(P, sg, nsg);

    float nq[4], ptq[4], pq[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float y[16];
        group_values(P, g, y);
        const float a = group_absmax(y);
        amax = max2n(amax, a);
        const bool live = a >= kTiny;
        const float p = live ? div6_rn(a) : 0.0f;
        const float r = live ? rcp_rn(p) : 0.0f;          // flushed group: sign-preserving zeros
        const uint64_t rr = f2(r, r);
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) f2_split(f2_mul(P[8 * g + i], rr), v[i], v[i + 8]);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float vh[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) vh[i] = v[8 * hh + i];
            cw[2 * g + hh] = e2m1x8(vh);
        }
        // products val*y and y*y on the pairs (i, i + 8), then the 16-term trees
        uint64_t T[8], N[8];
        e2m1x16_pairs(cw[2 * g], cw[2 * g + 1], T);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            T[i] = f2_prod(T[i], P[8 * g + i], nz);
            N[i] = f2_prod(P[8 * g + i], P[8 * g + i], nz);
        }
        const float tg = pair_tree16(T), ng = pair_tree16(N);
        pq[g] = p;
        nq[g] = live ? ng : 0.0f;
        ptq[g] = live ? __fmul_rn(p, tg) : 0.0f;
    }
    // Block sums over the 8 groups as the balanced tree ((G0+G1)+(G2+G3)) + ((G4+G5)+(G6+G7)):
    // this thread's level-1 sums are (G2h + G2h+1) and (G4+2h + G5+2h); level 2 adds the
    // partner's (addition commutes, so both threads get the same bits).
    const uint64_t lv_a = f2(__fadd_rn(nq[0], nq[1]), __fadd_rn(ptq[0], ptq[1]));
    const uint64_t lv_b = f2(__fadd_rn(nq[2], nq[3]), __fadd_rn(ptq[2], ptq[3]));
    const uint64_t lo = f2_add(lv_a, shfl_xor1_u64(lv_a)), hi = f2_add(lv_b, shfl_xor1_u64(lv_b));
    float num, den;
    f2_split(f2_add(lo, hi), num, den);
    const float S = den > 0.0f ? __fdiv_rn(num, den) : 1.0f;
#pragma unroll
    for (int g = 0; g < 4; ++g) Pq[g] = __fmul_rn(S, pq[g]);
}

// Elementwise-SR quantization of the thread's four local groups after rotate_tail: the GPU
// baseline of the pages' comparison ([QII-th] "fairness" answer: the TetraJet-v2 core, RHT
// along the inner dimension with stochastic rounding; [QII-tg] "Method").  Every decision is one
// binary32 operation: group scale code = the smallest E4M3 value >= a/(6g) (RNE, then one step
// up if RNE fell below), d = RN(s*g), r = RN(1/d), tq = min(|y|*r, 6); tq's lower E2M1 neighbour
// keeps the bits down to the top mantissa bit (the grid points of [2^k, 2^(k+1)) are 2^k and
// 1.5*2^k for k >= 0; 0.5 and 0 below 1); the spacing to the upper neighbour is a power of two,
// so frac = (tq - lo)/spacing is exact; round up iff (u>>8)*2^-24 < frac with u = Philox word e
// of (seed, tid).  e_base[g] = canonical index of local group g's first element.
__device__ __forceinline__ void sr_vector(const uint64_t (&P)[32], float g, float g6, bool zero_view, uint64_t seed,
                                          uint32_t tid, const int64_t (&e_base)[4], uint32_t (&cw)[8],
                                          uint32_t (&sc)[4], float &amax) {
#pragma unroll
    for (int gq = 0; gq < 4; ++gq) {
        float y[16];
        group_values(P, gq, y);
        const float a = group_absmax(y);
        amax = max2n(amax, a);
        float q[16];
        if (zero_view || !(a >= kTiny)) {
            sc[gq] = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(y[i], 0.0f);   // sign-preserving zeros
        } else {
            const float t = __fdiv_rn(a, g6);
            uint32_t c = e4m3_rne(t);
            if (c < 126u && e4m3_value(c) < t) ++c;                        // ceil onto E4M3
            sc[gq] = c;
            const float d = __fmul_rn(e4m3_value(c), g);
            const float r = __frcp_rn(d);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 u4 = philox_block(seed, tid, (uint64_t)((e_base[gq] >> 2) + k));
                const uint32_t uw[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                for (int i2 = 0; i2 < 4; ++i2) {
                    const int i = 4 * k + i2;
                    const float tq = fminf(__fmul_rn(fabsf(y[i]), r), 6.0f);
                    const uint32_t b = __float_as_uint(tq), e = b >> 23;
                    const bool ge1 = e >= 127u;
                    const float lo = __uint_as_float(ge1 ? (b & 0xFFC00000u) : (e == 126u ? 0x3F000000u : 0u));
                    const float sp = __uint_as_float(ge1 ? (e - 1u) << 23 : 0x3F000000u);       // spacing
                    const float inv = __uint_as_float(ge1 ? (255u - e) << 23 : 0x40000000u);     // 1/spacing
                    const float frac = __fmul_rn(__fsub_rn(tq, lo), inv);
                    const float U = __fmul_rn(__uint2float_rn(uw[i2] >> 8), 5.9604644775390625e-8f);   // 2^-24
                    const float vq = (U < frac) ? __fadd_rn(lo, sp) : lo;
                    q[i] = __uint_as_float(__float_as_uint(vq) | (__float_as_uint(y[i]) & 0x80000000u));
                }
            }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float vh[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) vh[i] = q[8 * hh + i];
            cw[2 * gq + hh] = e2m1x8(vh);   // exact: every value is a signed grid point
        }
    }
}

// Codes of the thread's groups {2h, 2h+1} and {4+2h, 5+2h} of a 128-block starting at group j0
// of view row vr (codes_row points at the block's first code byte); pre-scales in tensor-core
// scale order.
// codes_base and n_elems (the view's element count) bound the stores in the checked build.
__device__ __forceinline__ void msed_store(uint8_t *codes_row, float *P_base, int64_t vr, int64_t j0, int64_t VC,
                                           int h, const uint32_t (&cw)[8], const float (&Pq)[4],
                                           const uint8_t *codes_base, int64_t n_elems) {
    (void)codes_base;
    (void)n_elems;
    uint8_t *const c0 = codes_row + 16 * h, *const c1 = codes_row + 32 + 16 * h;
    float *const p0 = P_base + sf_offset(vr, j0 + 2 * h, VC), *const p1 = P_base + sf_offset(vr, j0 + 4 + 2 * h, VC);
    if (QT2_STORE_OK(c0, 16, codes_base, n_elems >> 1))
        *reinterpret_cast<uint4 *>(c0) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    if (QT2_STORE_OK(c1, 16, codes_base, n_elems >> 1))
        *reinterpret_cast<uint4 *>(c1) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    if (QT2_STORE_OK(p0, 8, P_base, (n_elems >> 4) * 4)) *reinterpret_cast<float2 *>(p0) = make_float2(Pq[0], Pq[1]);
    if (QT2_STORE_OK(p1, 8, P_base, (n_elems >> 4) * 4)) *reinterpret_cast<float2 *>(p1) = make_float2(Pq[2], Pq[3]);
}

// What one launch of the rotation producer emits per view (row view: [R][C]; column view: the
// transpose [C][R]).
struct RotViews {
    uint8_t *row_codes, *col_codes;     // MS-EDEN and SR codes
    float *row_P, *col_P;               // MS-EDEN fp32 pre-scales
    uint8_t *row_scales, *col_scales;   // SR E4M3 scales
    uint32_t *row_amax, *col_amax;      // max |y|: merged (MS-EDEN, max pass) or read (SR)
    float *row_g, *col_g;               // SR tensor scales, written
    uint32_t tid_row, tid_col;          // SR Philox tensor ids
};
enum RotMode { kModeEden = 0, kModeMax = 1, kModeSr = 2, kModeFwdRowEdenCol = 3 };

template <int MODE, bool DO_ROW, bool DO_COL>
__global__ void __launch_bounds__(MsedCfg::kThreads, 1)
    msed_kernel(const __grid_constant__ CUtensorMap tmap, int64_t R, int64_t C, uint64_t seed, RotViews out) {
    uint8_t *const row_codes = out.row_codes, *const col_codes = out.col_codes;
    float *const row_P = out.row_P, *const col_P = out.col_P;
    uint32_t *const row_amax = out.row_amax, *const col_amax = out.col_amax;
    using Cfg = MsedCfg;
    constexpr int NS = Cfg::kStages;
    constexpr bool kBoth = DO_ROW && DO_COL;
    constexpr uint32_t kConsumers = kBoth ? 2 * Cfg::kTeamWarps : Cfg::kTeamWarps;   // warps reading a tile
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t *buf0 = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar[NS];
    __shared__ uint32_t done_cnt[NS];           // warps done reading the stage, summed over its rounds
    __shared__ int last_issued[NS];             // local index of the last tile loaded into the stage
    // sign flips (at bit 31) of elements 2n, 2n + 1, 2n + 8, 2n + 9 in .x, .y, .z, .w: the four
    // elements of two pair registers (entries with bit 2 of n set are not used)
    __shared__ __align__(16) uint4 sgn4[64];
    __shared__ float s_nz;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int team = warp >= Cfg::kTeamWarps ? 1 : 0;
    const int h = lane & 1;
    const int64_t tiles_c = C >> 7, ntiles = (R >> 7) * tiles_c;
    const int64_t my_tiles = ntiles > (int64_t)blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t bar0 = smem_u32(&bar[0]);

    auto issue = [&](int64_t i) {   // local tile i into stage i % NS
        const int64_t tile = blockIdx.x + i * (int64_t)gridDim.x;
        const int32_t r0 = (int32_t)((tile / tiles_c) << 7), c0 = (int32_t)((tile % tiles_c) << 7);
        const int s = (int)(i % NS);
        const uint32_t fb = bar0 + 8 * s;
        last_issued[s] = (int)i;
        mbar_arrive_expect_tx(fb, Cfg::kTileBytes);
        tma_load_2d(smem_u32(buf0 + s * Cfg::kTileBytes), &tmap, c0, r0, fb);
        tma_load_2d(smem_u32(buf0 + s * Cfg::kTileBytes + 16384), &tmap, c0 + 64, r0, fb);
    };
    // A warp is done reading stage s (tile i); the last of the tile's readers refills the stage.
    auto release = [&](int s, int64_t i) {
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            const uint32_t old = atomicAdd(&done_cnt[s], 1u);
            if (old == (uint32_t)(i / NS + 1) * kConsumers - 1 && i + NS < my_tiles) issue(i + NS);
        }
    };
    if (t == 0) {
        prefetch_tmap(&tmap);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar0 + 8 * s, 1);
            done_cnt[s] = 0;
            last_issued[s] = -1;
        }
        fence_mbar_init();
    }
    if (t < 64) {
        const uint4 sw = rotation_sign_words(seed);   // bit i of the 128 signs: element i negated
        const uint32_t w[4] = {sw.x, sw.y, sw.z, sw.w};
        auto flip = [&](int e) { e &= 127; return ((w[e >> 5] >> (e & 31)) & 1u) << 31; };
        const int e = 2 * t;
        sgn4[t] = make_uint4(flip(e), flip(e + 1), flip(e + 8), flip(e + 9));
    }
    if (t == 0) s_nz = -0.0f;
    __syncthreads();
    const uint64_t nz = neg_zero_pair(&s_nz);   // addend of f2_prod
    if (t == 0)
        for (int64_t i = 0; i < NS && i < my_tiles; ++i) issue(i);

    // SR: tensor scale g = A/2688 of each view from its max pass; a view with A < 2^-100 is zero
    float g_r = 1.0f, g6_r = 6.0f, g_c = 1.0f, g6_c = 6.0f;
    bool zero_r = true, zero_c = true;
    if constexpr (MODE == kModeSr) {
        if (blockIdx.x == 0 && t == 0) {
            if (DO_ROW) check_finite_word(*row_amax);
            if (DO_COL) check_finite_word(*col_amax);
        }
        if (DO_ROW) {
            const float A = __uint_as_float(*row_amax);
            zero_r = !(A >= kTiny);
            g_r = zero_r ? 1.0f : __fdiv_rn(A, 2688.0f);
            g6_r = __fmul_rn(6.0f, g_r);
            if (blockIdx.x == 0 && t == 0) *out.row_g = g_r;
        }
        if (DO_COL) {
            const float A = __uint_as_float(*col_amax);
            zero_c = !(A >= kTiny);
            g_c = zero_c ? 1.0f : __fdiv_rn(A, 2688.0f);
            g6_c = __fmul_rn(6.0f, g_c);
            if (blockIdx.x == 0 && t == 0) *out.col_g = g_c;
        }
    }
    // forward view of the rows (kModeFwdRowEdenCol): tensor scale and the block's scale tables
    __shared__ float tab_d[128], tab_r[129];
    Fwd46Consts kc_f{0.0f, 0.0f, 0.0f, 0.0f};
    if constexpr (MODE == kModeFwdRowEdenCol) {
        if (blockIdx.x == 0 && t == 0) check_finite_word(*row_amax);   // outputs then unspecified
        const float g = fwd46_tensor_scale(row_amax);
        kc_f = fwd46_consts(g);
        if (blockIdx.x == 0 && t == 0) *out.row_g = g;
        fwd46_tables(g, tab_d, tab_r);
        __syncthreads();
        kc_f.nz = neg_zero_pair(&tab_r[128]);
    }
    const float sigma = h ? -1.0f : 1.0f;
    const uint64_t sg = f2(sigma, sigma), nsg = f2(-sigma, -sigma);
    const bool rows = kBoth ? team == 0 : DO_ROW;
    const int u = (t & (Cfg::kTeamWarps * 32 - 1)) >> 1;   // the pair's row (or column) of the tile
    float amax = 0.0f;
    const int64_t i0 = kBoth ? 0 : team, step = kBoth ? 1 : 2;
    // tile coordinates (row, column of tiles), advanced without a division per tile
    const int64_t adv = step * (int64_t)gridDim.x, adv_r = adv / tiles_c, adv_c = adv % tiles_c;
    int64_t t_r = ((int64_t)blockIdx.x + i0 * (int64_t)gridDim.x) / tiles_c;
    int64_t t_c = ((int64_t)blockIdx.x + i0 * (int64_t)gridDim.x) % tiles_c;
    for (int i = (int)i0; i < (int)my_tiles; i += (int)step) {
        const int64_t r0 = t_r << 7, c0 = t_c << 7;
        t_c += adv_c;
        t_r += adv_r;
        if (t_c >= tiles_c) {
            t_c -= tiles_c;
            ++t_r;
        }
        const int s = (int)(i % NS);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar0 + 8 * s, (uint32_t)((i / NS) & 1)))) break;   // warp-uniform
        const uint8_t *tb = buf0 + s * Cfg::kTileBytes;
        uint64_t P[32];
        // A tile is two 128x64 boxes with the 128-byte swizzle: element (r, c) sits at byte
        // (c / 64) * 16384 + r * 128 + (((c % 64) / 8) ^ (r % 8)) * 16 + (c % 8) * 2.
        const uint32_t tbu = smem_u32(tb);
        if constexpr (MODE == kModeFwdRowEdenCol) {
            if (rows) {
                // forward view of row u: groups 4h .. 4h+3 of the block (elements [64h, 64h + 64),
                // chunks c ^ (u % 8) of box h), quantized straight from shared memory; codes at
                // bytes [32h, 32h + 32) of the block, one scale word; then the stage is released
                const uint32_t rbase = tbu + h * 16384 + u * 128;
                uint32_t cw[8], scw = 0;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    const uint4 a = lds128(rbase + ((uint32_t)((2 * gq) ^ (u & 7)) << 4));
                    const uint4 b = lds128(rbase + ((uint32_t)((2 * gq + 1) ^ (u & 7)) << 4));
                    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    scw |= fwd46_group(w, kc_f, tab_d, tab_r, cw[2 * gq], cw[2 * gq + 1]) << (8 * gq);
                }
                release(s, i);
                const int64_t vr = r0 + u;
                uint8_t *const vcodes = row_codes + vr * (C >> 1) + (c0 >> 1);
                uint8_t *const sdst = out.row_scales + sf_offset(vr, (c0 >> 4) + 4 * h, C);
                if (QT2_STORE_OK(vcodes + 32 * h, 32, row_codes, R * (C >> 1))) {
                    *reinterpret_cast<uint4 *>(vcodes + 32 * h) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                    *reinterpret_cast<uint4 *>(vcodes + 32 * h + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
                }
                if (QT2_STORE_OK(sdst, 4, out.row_scales, R * (C >> 4))) *reinterpret_cast<uint32_t *>(sdst) = scw;
                continue;
            }
        }
        if (rows) {
            // row u, elements [64h, 64h + 64) of the tile row (box h).  Slot group gq = a + 2b
            // holds element chunks cl = 2a + 4b (low halves) and cl + 1 (high halves) of the
            // thread's half, with thread 1's quarters swapped (cl ^ 4h); the swizzled 16 bytes of
            // chunk c sit at chunk c ^ (u % 8) of row u.  Stride 1 is taken here.
            const uint32_t rbase = tbu + h * 16384 + u * 128, rx = (uint32_t)((4 * h) ^ (u & 7)) << 4;
            const uint32_t sbase = smem_u32(&sgn4[0]) + 512 * h, sx = 256 * h;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                const uint32_t cl = 2 * (gq & 1) + 4 * (gq >> 1);
                const uint4 L = lds128(rbase + (rx ^ (cl << 4))), H = lds128(rbase + (rx ^ ((cl + 1) << 4)));
                const uint32_t wl[4] = {L.x, L.y, L.z, L.w}, wh[4] = {H.x, H.y, H.z, H.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 m = lds128(sbase + (sx ^ (64 * cl + 16 * i)));
                    // adding 2^31 flips the sign bit
                    const uint64_t a = f2(__uint_as_float((wl[i] << 16) + m.x), __uint_as_float((wh[i] << 16) + m.z));
                    const uint64_t b = f2(__uint_as_float((wl[i] & 0xFFFF0000u) ^ m.y),
                                          __uint_as_float((wh[i] & 0xFFFF0000u) ^ m.w));
                    P[8 * gq + 2 * i] = f2_add(a, b);
                    P[8 * gq + 2 * i + 1] = f2_sub(a, b);
                }
            }
        } else {
            // column u, rows [64h, 64h + 64) of the tile.  Slot 16b + 8a + j holds rows
            // R0 + 16a + j and R0 + 16a + j + 8 with R0 = 64h + 32(b ^ h) (thread 1's quarters
            // swapped).  R0 is a multiple of 32, so the swizzle term of row R0 + r depends only
            // on r % 8: one base address per value of r % 8 and half b.  Stride 1 is taken here.
            const uint32_t colbase = (uint32_t)((u >> 6) * 16384 + (u & 7) * 2 + (((u & 63) >> 3) << 4));
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t hb = tbu + (half == 0 ? 12288u * h : 4096u + 4096u * h);
                const uint32_t sb = smem_u32(&sgn4[0]) + 512 * h + (half == 0 ? 256u * h : 256u - 256u * h);
                uint32_t X[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) X[k] = hb + (colbase ^ (uint32_t)(k << 4));
#pragma unroll
                for (int a = 0; a < 2; ++a) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int j = 2 * i, r = 16 * a + j;
                        const uint4 m = lds128(sb + 16 * i + 128 * a);
                        const uint32_t u0 = lds16(X[j] + 128 * r), u1 = lds16(X[j + 1] + 128 * (r + 1));
                        const uint32_t u2 = lds16(X[j] + 128 * (r + 8)), u3 = lds16(X[j + 1] + 128 * (r + 9));
                        const uint64_t va = f2(__uint_as_float((u0 << 16) + m.x), __uint_as_float((u2 << 16) + m.z));
                        const uint64_t vb = f2(__uint_as_float((u1 << 16) + m.y), __uint_as_float((u3 << 16) + m.w));
                        P[16 * half + 8 * a + j] = f2_add(va, vb);
                        P[16 * half + 8 * a + j + 1] = f2_sub(va, vb);
                    }
                }
            }
        }
        // The tile is in registers: release the stage; the last warp to do so refills it.
        release(s, i);
        const int64_t vr = rows ? r0 + u : c0 + u;   // view row (the column view is [C][R])
        const int64_t VC = rows ? C : R, b0 = rows ? c0 : r0;   // view row length, block start
        uint8_t *const vcodes = (rows ? row_codes : col_codes) + vr * (VC >> 1) + (b0 >> 1);
        if constexpr (MODE == kModeEden) {
            uint32_t cw[8];
            float Pq[4];
            msed_vector(P, sg, nsg, nz, cw, Pq, amax);
            msed_store(vcodes, rows ? row_P : col_P, vr, b0 >> 4, VC, h, cw, Pq, rows ? row_codes : col_codes, R * C);
        } else if constexpr (MODE == kModeFwdRowEdenCol) {   // column warps (rows returned above)
            uint32_t cw[8];
            float Pq[4];
            msed_vector(P, sg, nsg, nz, cw, Pq, amax);
            msed_store(vcodes, col_P, vr, b0 >> 4, VC, h, cw, Pq, col_codes, R * C);
        } else if constexpr (MODE == kModeMax) {
            rotate_tail(P, sg, nsg);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                float y0, y1;
                f2_split(P[k], y0, y1);
                amax = absmax3(amax, y0, y1);
            }
        } else {
            rotate_tail(P, sg, nsg);
            // local groups 0, 1, 2, 3 are the block's groups 2h, 2h+1, 4+2h, 5+2h
            const int64_t e0 = vr * VC + b0;
            const int64_t e_base[4] = {e0 + 32 * h, e0 + 32 * h + 16, e0 + 64 + 32 * h, e0 + 80 + 32 * h};
            uint32_t cw[8], scq[4];
            sr_vector(P, rows ? g_r : g_c, rows ? g6_r : g6_c, rows ? zero_r : zero_c, seed,
                      rows ? out.tid_row : out.tid_col, e_base, cw, scq, amax);
            const uint8_t *const cb = rows ? row_codes : col_codes;
            if (QT2_STORE_OK(vcodes + 16 * h, 16, cb, (R * C) >> 1))
                *reinterpret_cast<uint4 *>(vcodes + 16 * h) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            if (QT2_STORE_OK(vcodes + 32 + 16 * h, 16, cb, (R * C) >> 1))
                *reinterpret_cast<uint4 *>(vcodes + 32 + 16 * h) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            uint8_t *const sb = rows ? out.row_scales : out.col_scales;
            uint8_t *const s0 = sb + sf_offset(vr, (b0 >> 4) + 2 * h, VC), *const s1 = sb + sf_offset(vr, (b0 >> 4) + 4 + 2 * h, VC);
            if (QT2_STORE_OK(s0, 2, sb, (R * C) >> 4)) *reinterpret_cast<uint16_t *>(s0) = (uint16_t)(scq[0] | (scq[1] << 8));
            if (QT2_STORE_OK(s1, 2, sb, (R * C) >> 4)) *reinterpret_cast<uint16_t *>(s1) = (uint16_t)(scq[2] | (scq[3] << 8));
        }
    }
    if constexpr (MODE != kModeSr) {
        // (kModeFwdRowEdenCol: the row warps merge nothing; row_amax is the input's max)
        const uint32_t bm = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax));
        if (lane == 0 && bm != 0 && !(MODE == kModeFwdRowEdenCol && rows)) atomicMax(rows ? row_amax : col_amax, bm);
    }
    __syncthreads();
    if (t == 0) {
        // Only after a timeout can a load still be in flight: wait (bounded) for each stage's last one.
        for (int s = 0; s < NS; ++s)
            if (last_issued[s] >= 0) mbar_wait(bar0 + 8 * s, (uint32_t)((last_issued[s] / NS) & 1));
    }
}

}  // namespace qt2
