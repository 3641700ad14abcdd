/*
 * qt2 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded restatement of what the Quartet II NVFP4 linear
 * layer computes, used to check the CUDA path bit for bit.  Only the test suite,
 * the package smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header, table or constant generator with the CUDA library.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction: every float expression below is one IEEE-754 binary32
 * operation rounded to nearest-even, in the order written).
 *
 * Citations (page title, then section):
 *   [QII-th]  "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992):
 *             abstract; "Question 1" (hardware compromises, Fig. 9); "fairness" answer; §1 Introduction.
 *   [QII-ru]  Quartet II review by D. Avetisyan (denisavetisyan.com ?p=3427): sections
 *             "NVFP4 and micro-scaling", "Unbiased quantization with MS-EDEN and randomized methods".
 *   [FAF]     "Format-Aware Fusion for Fast FP4 Pretraining" (rit.work blog): "the speed-up is lost
 *             between the matmuls".
 *   [QII-tg]  Quartet II digest (quant_prune_distill post 640): "Method".
 *
 * Readings where the pages are silent (fixed by decision, identical on both sides):
 *   - E2M1 magnitudes {0,.5,1,1.5,2,3,4,6}; round to nearest, ties to the even code, sign
 *     kept (a negative value that rounds to zero encodes -0 = 0x8), |q| >= 6 saturates.
 *   - E4M3 scales are non-negative: RNE with subnormals, saturating at 448.
 *   - Stochastic rounding of a scale v >= 2^-6: lo/hi = the E4M3 neighbours of v, U = (u>>12)/2^20,
 *     round up iff U < (v-lo)/(hi-lo); v >= 448 gives 448.  Below 2^-6 the scale is RNE'd
 *     ([QII-th] "Question 1": very small FP8 scales, about 1/32000 of the max, skip SR).
 *   - Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): key = (lo32 seed, hi32 seed),
 *     counter = (lo32(j>>2), hi32(j>>2), tensor id, 0), word j&3 of the block.
 *   - Rotation: per 128-block, y = H (D x) with D the +-1 signs of tensor id 0 (bit i of word
 *     i>>5 set means -1) and H the unnormalised Sylvester Hadamard, evaluated as a butterfly
 *     with strides 1,2,...,64, (a+b, a-b) with a at the lower index.
 *   - Sums are balanced binary trees over contiguous power-of-two index ranges.
 *   - fwd46 tensor scale g = A/1792 (A = max|x|); MS-EDEN tensor scale g = A/1536 (A = max|y|).
 *   - Flush rules that keep every reciprocal finite: fwd46 treats a tensor with A < 2^-100 as
 *     zero (g = 1); MS-EDEN treats a group with max|y| < 2^-100 as zero.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define OR_EXPORT __attribute__((visibility("default")))

OR_EXPORT int or_version(void) { return 1; }

/* ------------------------------------------------------------------ bf16 */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
OR_EXPORT float or_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------ E2M1 */
/* NVFP4 element format: 4-bit float, values {0,+-0.5,+-1,+-1.5,+-2,+-3,+-4,+-6}
 * ([QII-th] §1 Introduction: 4-bit floats with a higher-precision block scale;
 *  [QII-tg] "Method": the full grid runs to +-6, the truncated one to +-4). */
static const float OR_E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

OR_EXPORT float or_e2m1_value(uint8_t code)
{
    float m = OR_E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Round to the nearest E2M1 magnitude by brute force over the 8 magnitudes; an exact tie
 * goes to the even code index; |q| >= 6 (including +-inf) saturates to 6; the sign bit of q
 * is kept. */
OR_EXPORT uint8_t or_e2m1_encode(float q)
{
    uint8_t sign = signbit(q) ? 8 : 0;
    float a = fabsf(q);
    if (a >= 6.0f) return (uint8_t)(sign | 7);
    int best = 0;
    double bestd = fabs((double)a - (double)OR_E2M1_MAG[0]);
    for (int i = 1; i < 8; i++) {
        double d = fabs((double)a - (double)OR_E2M1_MAG[i]);
        if (d < bestd || (d == bestd && (i % 2) == 0)) { best = i; bestd = d; }
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------ E4M3 */
/* FP8 E4M3 group scale, non-negative codes 0x00..0x7E (0x7F is NaN): exponent bias 7,
 * subnormals m*2^-9, largest finite 448 ([QII-th] §1: FP8 block scale). */
OR_EXPORT float or_e4m3_value(uint8_t code)
{
    int e = (code >> 3) & 15, m = code & 7;
    if (e == 0) return ldexpf((float)m, -9);
    return ldexpf((float)(8 + m), e - 10);
}

/* Round-to-nearest-even onto the 127 non-negative finite E4M3 codes, brute force.
 * Values above 448 saturate to 448 (code 0x7E). */
OR_EXPORT uint8_t or_e4m3_rne(float v)
{
    if (!(v > 0.0f)) return 0;
    int best = 0;
    double bestd = fabs((double)v);
    for (int c = 1; c <= 126; c++) {
        double d = fabs((double)v - (double)or_e4m3_value((uint8_t)c));
        if (d < bestd || (d == bestd && (c % 2) == 0)) { best = c; bestd = d; }
    }
    return (uint8_t)best;
}

/* Stochastic rounding onto E4M3 for v >= 2^-6 ([QII-tg] "Method": the quantization scales are
 * stochastically rounded to FP8).  lo = largest code <= v, hi = the next code; the draw
 * U = (u >> 12) / 2^20 rounds up iff U < (v - lo)/(hi - lo), so P(up) = (v-lo)/(hi-lo). */
OR_EXPORT uint8_t or_e4m3_sr(float v, uint32_t u)
{
    if (v >= 448.0f) return 126;
    int lo = 0;
    for (int c = 0; c <= 126; c++)
        if ((double)or_e4m3_value((uint8_t)c) <= (double)v) lo = c;
    double vlo = or_e4m3_value((uint8_t)lo);
    if (vlo == (double)v) return (uint8_t)lo;
    double vhi = or_e4m3_value((uint8_t)(lo + 1));
    double frac = ((double)v - vlo) / (vhi - vlo);
    double U = (double)(u >> 12) / 1048576.0;
    return (uint8_t)(U < frac ? lo + 1 : lo);
}

/* ------------------------------------------------------------------ Philox4x32-10 */
/* Counter-based generator of Salmon et al., SC'11, "Parallel Random Numbers: As Easy as 1, 2, 3":
 * ten rounds of two 32x32->64 multiplies with the Weyl key schedule. */
OR_EXPORT void or_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; round++) {
        if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Word j of the stream of (seed, tensor id). */
OR_EXPORT uint32_t or_philox_word(uint64_t seed, uint32_t tid, uint64_t j)
{
    uint64_t blk = j >> 2;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), tid, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    or_philox4x32_10(ctr, key, out);
    return out[j & 3];
}

/* ------------------------------------------------------------------ rotation */
/* The 128 random signs D of one backward call: bit i of word (seed, 0, i>>5) set -> -1
 * ([QII-th] "Question 1": fixed 128-dim rotation groups sharing one rotation and one seed). */
OR_EXPORT void or_rht_signs(uint64_t seed, float sgn[128])
{
    for (int i = 0; i < 128; i++) {
        uint32_t w = or_philox_word(seed, 0u, (uint64_t)(i >> 5));
        sgn[i] = ((w >> (i & 31)) & 1u) ? -1.0f : 1.0f;
    }
}

/* In-place unnormalised fast Walsh-Hadamard transform of 128 floats, strides 1..64. */
OR_EXPORT void or_fwht128(float y[128])
{
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i++)
            if (!(i & h)) {
                float a = y[i], b = y[i + h];
                y[i] = a + b;
                y[i + h] = a - b;
            }
}

/* Dense Sylvester Hadamard H[i][j] = (-1)^popcount(i & j), fp64 -- the check on or_fwht128. */
OR_EXPORT void or_hadamard128_dense(double *H)
{
    for (int i = 0; i < 128; i++)
        for (int j = 0; j < 128; j++)
            H[i * 128 + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
}

/* ------------------------------------------------------------------ trees */
static float or_tree(const float *v, int n)   /* n a power of two */
{
    float t[128];
    for (int i = 0; i < n; i++) t[i] = v[i];
    for (int w = n; w > 1; w >>= 1)
        for (int i = 0; i < w / 2; i++) t[i] = t[2 * i] + t[2 * i + 1];
    return t[0];
}

OR_EXPORT float or_tree_sum(const float *v, int n) { return or_tree(v, n); }

/* ------------------------------------------------------------------ amax */
OR_EXPORT float or_amax_bf16(const uint16_t *x, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float v = fabsf(or_bf16_to_f32(x[i]));
        if (v > a) a = v;
    }
    return a;
}

/* ------------------------------------------------------------------ forward: RTN + 4/6 */
#define OR_TINY 0x1p-100f

/* Tensor scale of the forward quantizer: g = A / (4*448), so that both candidate grids keep
 * every group scale at or below 448 ([FAF] "the speed-up is lost...": global NVFP4 scales
 * depend on the tensor-wide maximum). */
OR_EXPORT float or_fwd46_tensor_scale(float A)
{
    if (!(A >= OR_TINY)) return 1.0f;
    return A / 1792.0f;
}

/* One 16-element group quantized onto the grid whose largest magnitude is k (6 or 4),
 * by round-to-nearest ([QII-th] "fairness" answer: the forward pass uses RTN).
 * Writes the 16 codes, returns the E4M3 scale code, and the squared error in *err. */
static uint8_t or_fwd46_candidate(const float x[16], float a, float g, float k,
                                  uint8_t codes[16], float *err)
{
    float gk = g * k;
    float t = a / gk;
    uint8_t s = or_e4m3_rne(t);
    float d = or_e4m3_value(s) * g;
    float sq[16];
    if (s == 0) {
        for (int i = 0; i < 16; i++) {
            codes[i] = signbit(x[i]) ? 8 : 0;
            sq[i] = x[i] * x[i];
        }
    } else {
        float r = 1.0f / d;
        for (int i = 0; i < 16; i++) {
            codes[i] = or_e2m1_encode(x[i] * r);
            float e = x[i] - or_e2m1_value(codes[i]) * d;
            sq[i] = e * e;
        }
    }
    *err = or_tree(sq, 16);
    return s;
}

/* Forward quantizer over rows [r0, r1) of a bf16 [R][C] matrix grouped along C in 1x16 groups
 * ([QII-tg] "Method": 1x16 groups are used rather than 16x16 blocks; for each group the full +-6
 * grid or the truncated +-4 grid is kept, whichever has the smaller quantization error).
 * Outputs (canonical layouts): codes [R][C/2] (element 2j in the low nibble), scales [R][C/16],
 * choice [R][C/16] = 6 or 4 (nullable), err6/err4 [R][C/16] (nullable).  A tie keeps 6. */
OR_EXPORT void or_fwd46_rows(const uint16_t *x, int64_t R, int64_t C, float A, int64_t r0, int64_t r1,
                             uint8_t *codes, uint8_t *scales, uint8_t *choice, float *err6, float *err4)
{
    (void)R;
    float g = or_fwd46_tensor_scale(A);
    int zero_tensor = !(A >= OR_TINY);
    int64_t G = C / 16;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t q = 0; q < G; q++) {
            float xv[16], a = 0.0f;
            for (int i = 0; i < 16; i++) {
                xv[i] = or_bf16_to_f32(x[r * C + q * 16 + i]);
                if (fabsf(xv[i]) > a) a = fabsf(xv[i]);
            }
            uint8_t c6[16], c4[16], s6, s4;
            float e6, e4;
            if (zero_tensor) {
                for (int i = 0; i < 16; i++) c6[i] = signbit(xv[i]) ? 8 : 0;
                s6 = 0; s4 = 0;
                float sq[16];
                for (int i = 0; i < 16; i++) sq[i] = xv[i] * xv[i];
                e6 = e4 = or_tree(sq, 16);
            } else {
                s6 = or_fwd46_candidate(xv, a, g, 6.0f, c6, &e6);
                s4 = or_fwd46_candidate(xv, a, g, 4.0f, c4, &e4);
            }
            int pick4 = !zero_tensor && (e4 < e6);
            const uint8_t *cc = pick4 ? c4 : c6;
            for (int i = 0; i < 8; i++)
                codes[r * (C / 2) + q * 8 + i] = (uint8_t)(cc[2 * i] | (cc[2 * i + 1] << 4));
            scales[r * G + q] = pick4 ? s4 : s6;
            if (choice) choice[r * G + q] = pick4 ? 4 : 6;
            if (err6) err6[r * G + q] = e6;
            if (err4) err4[r * G + q] = e4;
        }
    }
}

/* Square-block forward quantizer over block rows [b0, b1) of a bf16 [R][C] matrix (R, C
 * multiples of 16): one E4M3 scale per 16x16 block, so that the quantized matrix and its
 * transpose are the same quantization and one pass serves both operand views of a weight
 * ([QII-tg] "Method": the pages compare 16x16 blocks with 1x16 groups and keep the groups for
 * their lower error; the square blocks are their faster alternative).  The steps are the forward
 * quantizer's ones with the block in place of the group: a = max|x| over the block, for k = 6
 * and k = 4 the scale E4M3_RNE(a/(g*k)) and the RTN codes of each of the 16 rows, the block's
 * squared error = balanced tree over its 256 elements in row-major order (= the tree of the 16
 * rows' 16-element trees); keep 4 iff its error is smaller (a tie keeps 6).
 * Outputs in the row view's canonical layouts: codes [R][C/2], scales [R][C/16] (every row of a
 * block repeats the block's scale); per block (nullable): choice, err6, err4 [R/16][C/16]. */
OR_EXPORT void or_fwd46_sq_blocks(const uint16_t *x, int64_t R, int64_t C, float A, int64_t b0, int64_t b1,
                                  uint8_t *codes, uint8_t *scales, uint8_t *choice, float *err6, float *err4)
{
    (void)R;
    float g = or_fwd46_tensor_scale(A);
    int zero_tensor = !(A >= OR_TINY);
    int64_t G = C / 16;
    for (int64_t rb = b0; rb < b1; rb++) {
        for (int64_t q = 0; q < G; q++) {
            float xv[16][16], a = 0.0f;
            for (int i = 0; i < 16; i++)
                for (int j = 0; j < 16; j++) {
                    xv[i][j] = or_bf16_to_f32(x[(rb * 16 + i) * C + q * 16 + j]);
                    if (fabsf(xv[i][j]) > a) a = fabsf(xv[i][j]);
                }
            uint8_t c6[16][16], c4[16][16], s6 = 0, s4 = 0;
            float r6[16], r4[16];
            for (int i = 0; i < 16; i++) {
                if (zero_tensor) {
                    float sq[16];
                    for (int j = 0; j < 16; j++) {
                        c6[i][j] = signbit(xv[i][j]) ? 8 : 0;
                        sq[j] = xv[i][j] * xv[i][j];
                    }
                    r6[i] = r4[i] = or_tree(sq, 16);
                } else {
                    s6 = or_fwd46_candidate(xv[i], a, g, 6.0f, c6[i], &r6[i]);
                    s4 = or_fwd46_candidate(xv[i], a, g, 4.0f, c4[i], &r4[i]);
                }
            }
            float e6 = or_tree(r6, 16), e4 = or_tree(r4, 16);
            int pick4 = !zero_tensor && (e4 < e6);
            for (int i = 0; i < 16; i++) {
                int64_t r = rb * 16 + i;
                uint8_t *cc = pick4 ? c4[i] : c6[i];
                for (int j = 0; j < 8; j++)
                    codes[r * (C / 2) + q * 8 + j] = (uint8_t)(cc[2 * j] | (cc[2 * j + 1] << 4));
                scales[r * G + q] = pick4 ? s4 : s6;
            }
            if (choice) choice[rb * G + q] = pick4 ? 4 : 6;
            if (err6) err6[rb * G + q] = e6;
            if (err4) err4[rb * G + q] = e4;
        }
    }
}

/* ------------------------------------------------------------------ backward: MS-EDEN */
/* The EDEN steps on one rotated 128-block y ([QII-tg] "Method", item 1; [QII-ru] "Unbiased
 * quantization with MS-EDEN"):
 *   per 16-group: a = max|y|, p = a/6, codes = RTN_E2M1(y * (1/p)),
 *                 t = sum val(code)*y, n = sum y*y;
 *   per block:    S = sum n / sum p*t  (the EDEN factor <x,x>/<Q(Rx),Rx>, taken in the
 *                 rotated domain, where both inner products are those of x up to the same
 *                 constant factor of the rotation's normalisation);
 *   pre-scale P = S * p per group.
 * Writes the block's 64 code bytes, 8 group maxima and 8 pre-scales; returns S. */
static float or_eden_block(const float y[128], uint8_t codes[64], float amax_g[8], float P[8])
{
    float nq[8], ptq[8], pq[8];
    uint8_t cq[128];
    for (int q = 0; q < 8; q++) {
        const float *yq = y + 16 * q;
        float a = 0.0f;
        for (int i = 0; i < 16; i++) if (fabsf(yq[i]) > a) a = fabsf(yq[i]);
        amax_g[q] = a;
        float tv[16], nv[16];
        if (!(a >= OR_TINY)) {
            pq[q] = 0.0f;
            for (int i = 0; i < 16; i++) cq[16 * q + i] = signbit(yq[i]) ? 8 : 0;
            nq[q] = 0.0f;
            ptq[q] = 0.0f;
            continue;
        }
        float p = a / 6.0f;
        float rcp = 1.0f / p;
        for (int i = 0; i < 16; i++) {
            uint8_t c = or_e2m1_encode(yq[i] * rcp);
            cq[16 * q + i] = c;
            tv[i] = or_e2m1_value(c) * yq[i];
            nv[i] = yq[i] * yq[i];
        }
        pq[q] = p;
        nq[q] = or_tree(nv, 16);
        ptq[q] = p * or_tree(tv, 16);
    }
    float num = or_tree(nq, 8), den = or_tree(ptq, 8);
    float S = den > 0.0f ? num / den : 1.0f;
    for (int q = 0; q < 8; q++) P[q] = S * pq[q];
    for (int i = 0; i < 64; i++) codes[i] = (uint8_t)(cq[2 * i] | (cq[2 * i + 1] << 4));
    return S;
}

/* Stage 1 of MS-EDEN over rows [r0, r1) of a bf16 [R][C] matrix grouped along C (C a multiple
 * of 128): per 128-block the randomized Hadamard rotation y = H D x, then the EDEN steps above.
 * Outputs: codes [R][C/2], amax_g [R][C/16] (= a), P [R][C/16], S [R][C/128] (nullable). */
OR_EXPORT void or_msedEN_rows_stage1(const uint16_t *x, int64_t R, int64_t C, const float sgn[128],
                                     int64_t r0, int64_t r1, uint8_t *codes, float *amax_g,
                                     float *P, float *S_out)
{
    (void)R;
    int64_t G = C / 16;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t b = 0; b < C / 128; b++) {
            float y[128];
            for (int i = 0; i < 128; i++) y[i] = sgn[i] * or_bf16_to_f32(x[r * C + b * 128 + i]);
            or_fwht128(y);
            float S = or_eden_block(y, codes + r * (C / 2) + b * 64, amax_g + r * G + b * 8, P + r * G + b * 8);
            if (S_out) S_out[r * (C / 128) + b] = S;
        }
    }
}

/* The alternative EDEN grouping the pages leave open (one factor per 16-element group instead
 * of per 128-element rotation block), kept only to compare the two readings: the same steps as
 * or_eden_block with S_q = (sum y^2) / (p * sum val*y) over each group q alone.  Returns nothing
 * per block; P[q] = S_q * p_q. */
static void or_eden_group16(const float y[128], uint8_t codes[64], float amax_g[8], float P[8])
{
    uint8_t cq[128];
    for (int q = 0; q < 8; q++) {
        const float *yq = y + 16 * q;
        float a = 0.0f;
        for (int i = 0; i < 16; i++) if (fabsf(yq[i]) > a) a = fabsf(yq[i]);
        amax_g[q] = a;
        if (!(a >= OR_TINY)) {
            P[q] = 0.0f;
            for (int i = 0; i < 16; i++) cq[16 * q + i] = signbit(yq[i]) ? 8 : 0;
            continue;
        }
        float p = a / 6.0f;
        float rcp = 1.0f / p;
        float tv[16], nv[16];
        for (int i = 0; i < 16; i++) {
            uint8_t c = or_e2m1_encode(yq[i] * rcp);
            cq[16 * q + i] = c;
            tv[i] = or_e2m1_value(c) * yq[i];
            nv[i] = yq[i] * yq[i];
        }
        float num = or_tree(nv, 16), den = p * or_tree(tv, 16);
        float S = den > 0.0f ? num / den : 1.0f;
        P[q] = S * p;
    }
    for (int i = 0; i < 64; i++) codes[i] = (uint8_t)(cq[2 * i] | (cq[2 * i + 1] << 4));
}

/* Stage 1 with the per-16-group EDEN factor (comparison of readings only; not the method). */
OR_EXPORT void or_msedEN_rows_stage1_g16(const uint16_t *x, int64_t R, int64_t C, const float sgn[128],
                                         int64_t r0, int64_t r1, uint8_t *codes, float *amax_g, float *P)
{
    (void)R;
    int64_t G = C / 16;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            float y[128];
            for (int i = 0; i < 128; i++) y[i] = sgn[i] * or_bf16_to_f32(x[r * C + b * 128 + i]);
            or_fwht128(y);
            or_eden_group16(y, codes + r * (C / 2) + b * 64, amax_g + r * G + b * 8, P + r * G + b * 8);
        }
}

/* The same EDEN steps on values already rotated by some other orthogonal map (fp32 [R][C], C a
 * multiple of 128): used to separate the EDEN steps' own unbiasedness from that of the
 * 128-point randomized Hadamard rotation (EDEN is exactly unbiased for a uniformly random
 * rotation).  Outputs as or_msedEN_rows_stage1. */
OR_EXPORT void or_msedEN_rotated_stage1(const float *y, int64_t R, int64_t C, int64_t r0, int64_t r1,
                                        uint8_t *codes, float *amax_g, float *P, float *S_out)
{
    (void)R;
    int64_t G = C / 16;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            float S = or_eden_block(y + r * C + b * 128, codes + r * (C / 2) + b * 64, amax_g + r * G + b * 8,
                                    P + r * G + b * 8);
            if (S_out) S_out[r * (C / 128) + b] = S;
        }
}

/* Tensor scale of an MS-EDEN view: g = A / (6*256) with A = max|y| over the view, leaving
 * 448/256 = 1.75x headroom for the EDEN factor and the upward stochastic rounding. */
OR_EXPORT float or_msedEN_tensor_scale(float A)
{
    if (!(A >= OR_TINY)) return 1.0f;
    return A / 1536.0f;
}

/* Stage 2: the FP8 group scales, stochastically rounded ([QII-tg] "Method", item 2), except
 * below the E4M3 normal range 2^-6 where RNE is used ([QII-th] "Question 1": very small
 * scales skip SR).  v = P * (1/g); the draw of group j (canonical index r*(C/16)+q) is
 * word j of the Philox stream (seed, tid). */
OR_EXPORT void or_msedEN_finalize(const float *P, int64_t R, int64_t C, float g, uint64_t seed,
                                  uint32_t tid, int64_t r0, int64_t r1, uint8_t *scales)
{
    (void)R;
    float ginv = 1.0f / g;
    int64_t G = C / 16;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t q = 0; q < G; q++) {
            int64_t j = r * G + q;
            float v = P[j] * ginv;
            if (v < 0x1p-6f) scales[j] = or_e4m3_rne(v);
            else scales[j] = or_e4m3_sr(v, or_philox_word(seed, tid, (uint64_t)j));
        }
}

/* ------------------------------------------------------------------ dequantization */
/* xhat = val(code) * scale * g in fp64, [R][C] from canonical codes [R][C/2] and scales [R][C/16]. */
OR_EXPORT void or_dequant(const uint8_t *codes, const uint8_t *scales, int64_t R, int64_t C, float g,
                          int64_t r0, int64_t r1, double *out)
{
    (void)R;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t c = 0; c < C; c++) {
            uint8_t byte = codes[r * (C / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * C + c] = (double)or_e2m1_value(code) * (double)or_e4m3_value(scales[r * (C / 16) + c / 16])
                             * (double)g;
        }
}

/* One dequantized row r (fp64) into out[0..C). */
OR_EXPORT void or_dequant_row(const uint8_t *codes, const uint8_t *scales, int64_t R, int64_t C, float g, int64_t r,
                              double *out)
{
    (void)R;
    for (int64_t c = 0; c < C; c++) {
        uint8_t byte = codes[r * (C / 2) + c / 2];
        uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
        out[c] = (double)or_e2m1_value(code) * (double)or_e4m3_value(scales[r * (C / 16) + c / 16]) * (double)g;
    }
}

/* Inverse rotation of rotated-domain rows (fp64): x = (1/128) D H y per 128-block. */
OR_EXPORT void or_unrotate_rows(const double *y, int64_t R, int64_t C, const float sgn[128], int64_t r0,
                                int64_t r1, double *out)
{
    (void)R;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            const double *yb = y + r * C + b * 128;
            for (int i = 0; i < 128; i++) {
                double s = 0.0;
                for (int j = 0; j < 128; j++)
                    s += ((__builtin_popcount((unsigned)(i & j)) & 1) ? -yb[j] : yb[j]);
                out[r * C + b * 128 + i] = (double)sgn[i] * s / 128.0;
            }
        }
}

/* ------------------------------------------------------------------ GEMM */
/* C[i][j] = alpha * sum_k A[i][k] * B[j][k] in fp64, rows [i0, i1): both operands K-major. */
OR_EXPORT void or_gemm_f64(const double *A, const double *B, int64_t M, int64_t N, int64_t K, double alpha,
                           int64_t i0, int64_t i1, double *Cout)
{
    (void)M;
    for (int64_t i = i0; i < i1; i++)
        for (int64_t j = 0; j < N; j++) {
            double s = 0.0;
            for (int64_t k = 0; k < K; k++) s += A[i * K + k] * B[j * K + k];
            Cout[i * N + j] = alpha * s;
        }
}

/* ------------------------------------------------------------------ SR baseline */
/* Max |y| over rotated rows [r0, r1) (the tensor max the plain-NVFP4 SR baseline scales by). */
OR_EXPORT float or_rotated_amax_rows(const uint16_t *x, int64_t R, int64_t C, const float sgn[128],
                                     int64_t r0, int64_t r1)
{
    (void)R;
    float A = 0.0f;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            float y[128];
            for (int i = 0; i < 128; i++) y[i] = sgn[i] * or_bf16_to_f32(x[r * C + b * 128 + i]);
            or_fwht128(y);
            for (int i = 0; i < 128; i++) if (fabsf(y[i]) > A) A = fabsf(y[i]);
        }
    return A;
}

/* The elementwise-SR quantizer of the rotated view as the GPU baseline computes it: every
 * decision in binary32, so codes and scales are exactly reproducible ([QII-th] abstract and
 * "fairness" answer: the SR-based TetraJet-v2 core, RHT along the inner dimension, is the
 * baseline MS-EDEN is compared with; [QII-tg] "Method": SR rounds to one of the two grid
 * neighbours with probability set by the distance).  Reading (the pages give no scale rule for
 * the baseline): tensor scale g = A/2688 (A = max|y| over the view, 2688 = 6*448); the group
 * scale is the smallest E4M3 value s with s >= a/(6g) (a = max|y| of the group, t = a/RN(6g)
 * in binary32), so no element leaves the grid and SR stays unbiased; d = RN(s*g), r = RN(1/d),
 * tq = min(|y|*r, 6); lo/hi = the E2M1 neighbours of tq; round up iff U < (tq-lo)/(hi-lo) with
 * U = (u>>8)/2^24 and u = word e of the Philox stream (seed, tid), e = the element's canonical
 * index r*C + c.  A view with A < 2^-100 is zero (g = 1); a group with a < 2^-100 gets scale 0
 * and sign-only zero codes.  Codes keep the sign of y (a negative y that rounds to 0 is 0x8). */
OR_EXPORT float or_sr_tensor_scale(float A) { return (A >= OR_TINY) ? A / 2688.0f : 1.0f; }

OR_EXPORT void or_sr_rows(const uint16_t *x, int64_t R, int64_t C, const float sgn[128], float A, uint64_t seed,
                          uint32_t tid, int64_t r0, int64_t r1, uint8_t *codes, uint8_t *scales)
{
    (void)R;
    const float g = or_sr_tensor_scale(A);
    const float g6 = 6.0f * g;
    const int zero_view = !(A >= OR_TINY);
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            float y[128];
            for (int i = 0; i < 128; i++) y[i] = sgn[i] * or_bf16_to_f32(x[r * C + b * 128 + i]);
            or_fwht128(y);
            for (int q = 0; q < 8; q++) {
                const int64_t j = b * 8 + q;   /* group index within the row */
                float a = 0.0f;
                for (int i = 0; i < 16; i++) if (fabsf(y[16 * q + i]) > a) a = fabsf(y[16 * q + i]);
                uint8_t nib[16];
                if (zero_view || !(a >= OR_TINY)) {
                    scales[r * (C / 16) + j] = 0;
                    for (int i = 0; i < 16; i++) nib[i] = signbit(y[16 * q + i]) ? 0x8 : 0x0;
                } else {
                    const float t = a / g6;
                    int sc = 0;
                    while (sc < 126 && or_e4m3_value((uint8_t)sc) < t) sc++;   /* ceil onto E4M3 */
                    scales[r * (C / 16) + j] = (uint8_t)sc;
                    const float d = or_e4m3_value((uint8_t)sc) * g;
                    const float rr = 1.0f / d;
                    for (int i = 0; i < 16; i++) {
                        const float v = y[16 * q + i];
                        float tq = fabsf(v) * rr;
                        if (tq > 6.0f) tq = 6.0f;
                        int lo = 0;
                        for (int m = 1; m < 8; m++) if (OR_E2M1_MAG[m] <= tq) lo = m;
                        if (lo < 7) {
                            const float frac = (tq - OR_E2M1_MAG[lo]) / (OR_E2M1_MAG[lo + 1] - OR_E2M1_MAG[lo]);
                            const uint32_t u = or_philox_word(seed, tid, (uint64_t)(r * C + 16 * j + i));
                            const float U = (float)(u >> 8) * (1.0f / 16777216.0f);
                            if (U < frac) lo++;
                        }
                        nib[i] = (uint8_t)((signbit(v) ? 0x8 : 0x0) | lo);
                    }
                }
                for (int i = 0; i < 8; i++)
                    codes[r * (C / 2) + j * 8 + i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
            }
        }
}

/* Plain NVFP4 with elementwise stochastic rounding, in the rotated domain -- the unbiased but
 * noisier estimator the pages compare MS-EDEN against ([QII-th] abstract; [QII-tg] "Method":
 * SR rounds up or down with probability set by the distance to the two neighbouring grid
 * points).  NVFP4 scaling with tensor scale g = A/(6*448); the group scale is the smallest
 * E4M3 value s with s >= a/(6g), so that no element exceeds the grid (|y|/(s g) <= 6) and the
 * estimator stays exactly unbiased; elements t = |y|/(s g) are stochastically rounded onto
 * the E2M1 grid.  Element e of the view draws word e of the Philox stream (seed, tid).
 * Writes the dequantized rotated values (fp64). */
OR_EXPORT void or_sr_rows_dequant(const uint16_t *x, int64_t R, int64_t C, const float sgn[128], float A,
                                  uint64_t seed, uint32_t tid, int64_t r0, int64_t r1, double *out)
{
    (void)R;
    float g = (A >= OR_TINY) ? A / 2688.0f : 1.0f;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t b = 0; b < C / 128; b++) {
            float y[128];
            for (int i = 0; i < 128; i++) y[i] = sgn[i] * or_bf16_to_f32(x[r * C + b * 128 + i]);
            or_fwht128(y);
            for (int q = 0; q < 8; q++) {
                float a = 0.0f;
                for (int i = 0; i < 16; i++) if (fabsf(y[16 * q + i]) > a) a = fabsf(y[16 * q + i]);
                double t = (double)a / ((double)g * 6.0);
                int sc = 0;
                while (sc < 126 && (double)or_e4m3_value((uint8_t)sc) < t) sc++;
                double d = (double)or_e4m3_value((uint8_t)sc) * (double)g;
                for (int i = 0; i < 16; i++) {
                    int64_t e = r * C + b * 128 + 16 * q + i;
                    if (d == 0.0) { out[e] = 0.0; continue; }
                    double tq = fabs((double)y[16 * q + i]) / d;
                    if (tq > 6.0) tq = 6.0;
                    int lo = 0;
                    for (int m = 0; m < 8; m++) if ((double)OR_E2M1_MAG[m] <= tq) lo = m;
                    double vlo = OR_E2M1_MAG[lo], mag = vlo;
                    if (lo < 7 && vlo < tq) {
                        double vhi = OR_E2M1_MAG[lo + 1];
                        double U = (double)(or_philox_word(seed, tid, (uint64_t)e) >> 8) / 16777216.0;
                        if (U < (tq - vlo) / (vhi - vlo)) mag = vhi;
                    }
                    out[e] = (y[16 * q + i] < 0.0f ? -mag : mag) * d;
                }
            }
        }
}
