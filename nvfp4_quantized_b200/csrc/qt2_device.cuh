// qt2_device.cuh -- device helpers of the qt2 CUDA kernels (sm_100a only); included by the
// library's single translation unit.
//
// Number formats follow the NVFP4 definition: E2M1 elements (values 0, .5, 1, 1.5, 2, 3, 4, 6 and
// their negatives) with unsigned E4M3 group scales ("Quartet II ... MS-EDEN" Thai translation,
// §1 Introduction: 4-bit floats with a higher-precision FP8 block scale).  Conversions use the
// sm_100a hardware converts with round-to-nearest-even and saturation.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "qt2_internal.h"

namespace qt2 {

// ------------------------------------------------------------------------------------------
// Device status word: the first error a kernel reports (0 = none).  Read back by
// qt2_device_status().  Kernels never trap; a failed bounded wait records QT2_ERR_TIMEOUT.
// ------------------------------------------------------------------------------------------
__device__ int g_device_status = 0;

__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_device_status, 0, code); }

// ------------------------------------------------------------------------------------------
// Store checks of the checked build (compiled with -DQT2_CHECKED into libqt2_checked.so): every
// global store of the kernels' outputs first checks that its bytes [p, p + bytes) lie inside the
// output array [base, base + extent) the launch was given; a store that would leave it is
// skipped and QT2_ERR_BOUNDS recorded in the status word.  In the product build the check is
// the constant true and costs nothing.
// ------------------------------------------------------------------------------------------
#ifdef QT2_CHECKED
__device__ __noinline__ bool store_in_bounds(const void *p, uint64_t bytes, const void *base, uint64_t extent) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
    if (a >= b && a - b <= extent && bytes <= extent - (a - b)) return true;
    set_device_error(QT2_ERR_BOUNDS);
    return false;
}
#define QT2_STORE_OK(p, bytes, base, extent) \
    (::qt2::store_in_bounds((p), (uint64_t)(bytes), (base), (uint64_t)(extent)))
#else
#define QT2_STORE_OK(p, bytes, base, extent) ((void)(p), (void)(bytes), (void)(base), (void)(extent), true)
#endif

// Upper bound of any single wait inside a kernel (ns).  A correct launch never comes close.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------------------------------
// bf16 / number formats
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight floats -> eight E2M1 codes packed in a word: v[i] goes to nibble i (v[0] in bits 3..0).
// The convert places its first operand in the high nibble of each byte.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Sixteen E2M1 codes (c0: elements 0..7, c1: elements 8..15, element i in nibble i % 8) -> their
// exact values as fp32 pairs V[i] = (value of element i, value of element i + 8).
__device__ __forceinline__ void e2m1x16_pairs(uint32_t c0, uint32_t c1, uint64_t (&V)[8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        asm("{\n\t.reg .b8 p, q;\n\t.reg .b32 hp, hq;\n\t.reg .f16 p0, p1, q0, q1;\n\t.reg .f32 a, b, c, d;\n\t"
            "cvt.u8.u32 p, %2;\n\tcvt.u8.u32 q, %3;\n\t"
            "cvt.rn.f16x2.e2m1x2 hp, p;\n\tcvt.rn.f16x2.e2m1x2 hq, q;\n\t"
            "mov.b32 {p0, p1}, hp;\n\tmov.b32 {q0, q1}, hq;\n\t"
            "cvt.f32.f16 a, p0;\n\tcvt.f32.f16 b, q0;\n\tcvt.f32.f16 c, p1;\n\tcvt.f32.f16 d, q1;\n\t"
            "mov.b64 %0, {a, b};\n\tmov.b64 %1, {c, d};\n\t}"
            : "=l"(V[2 * j]), "=l"(V[2 * j + 1])
            : "r"(c0 >> (8 * j)), "r"(c1 >> (8 * j)));
    }
}

// Non-negative float -> E4M3 byte, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rne(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;
}

// E4M3 byte -> exact fp32 value.
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
    float out;
    uint16_t in = (uint16_t)(byte & 0xFF);
    asm("{\n\t.reg .b32 h2;\n\t.reg .f16 lo, hi;\n\tcvt.rn.f16x2.e4m3x2 h2, %1;\n\t"
        "mov.b32 {lo, hi}, h2;\n\tcvt.f32.f16 %0, lo;\n\t}"
        : "=f"(out)
        : "h"(in));
    return out;
}

// Stochastic rounding of v in [2^-6, inf) onto E4M3 with the 20-bit draw u >> 12: the fp32
// encoding of v keeps 3 of its 23 mantissa bits in E4M3, so the 20 discarded bits f measure
// (v - lo)/(hi - lo) * 2^20 exactly; round up iff the draw is below f.  Results above 448
// saturate.
__device__ __forceinline__ uint32_t e4m3_sr(float v, uint32_t u) {
    uint32_t bits = __float_as_uint(v);
    uint32_t f = bits & 0xFFFFFu;
    uint32_t t = (bits & ~0xFFFFFu) + (((u >> 12) < f) ? 0x100000u : 0u);
    return e4m3_rne(__uint_as_float(t));   // exact unless above 448, where it saturates
}

// ------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11, "Parallel Random Numbers: As Easy as 1, 2, 3").
// Stream (seed, tensor id): word j is element j&3 of the block at counter
// (lo32(j>>2), hi32(j>>2), tensor id, 0) under key (lo32(seed), hi32(seed)).
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

__device__ __forceinline__ uint4 philox_block(uint64_t seed, uint32_t tid, uint64_t blk) {
    return philox4x32_10(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), tid, 0u),
                         make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
}

// ------------------------------------------------------------------------------------------
// Scale-factor order of the tensor cores (scales of 128 rows x 4 groups in one 512-byte atom).
// ------------------------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t j, int64_t C) {
    return ((r >> 7) * (C >> 6) + (j >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// ------------------------------------------------------------------------------------------
// Shared memory / mbarrier / TMA / bulk-copy wrappers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase: returns false (and records QT2_ERR_TIMEOUT) after
// kWaitLimitNs without completion.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
            set_device_error(QT2_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait by a whole warp, for warps that go on to warp-collective (.sync.aligned)
// tcgen05 instructions: every lane polls, and the vote reconverges the warp and makes the
// outcome uniform (false if any lane gave up).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity));
}

// 2D tiled TMA load (no multicast) of box {x, y} into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t x, int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Non-tensor bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// One lane of a converged warp (PTX elect.sync).
__device__ __forceinline__ bool elect_one() {
    uint32_t p;
    asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xFFFFFFFF;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(p));
    return p != 0;
}

// ------------------------------------------------------------------------------------------
// Thread-block cluster helpers
// ------------------------------------------------------------------------------------------
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
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}

// ------------------------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core) wrappers, cta_group::1
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Signals `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Copy 32 rows x 16 bytes of shared memory (one 512-byte scale atom) into TMEM, replicated
// into all four 32-lane quadrants, 4 columns wide.
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] x B[smem] with NVFP4 block scales from TMEM (K = 64 per instruction).
__device__ __forceinline__ void tc_mma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 bits x 16 columns: thread t of the warp gets lane (quadrant*32 + t), columns
// [col, col+16).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of the 5th-generation tensor core: start address, leading
// and stride byte offsets (16-byte units), version 1, layout type (2 = 128-byte swizzle,
// 0 = no swizzle).
__device__ __forceinline__ uint64_t make_smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                                   uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7) << 61;
    return d;
}

}  // namespace qt2
