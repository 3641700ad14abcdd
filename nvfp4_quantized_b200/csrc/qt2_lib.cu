// qt2_lib.cu -- the qt2 library: kernel launchers and the C ABI declared in include/qt2.h.
//
// One translation unit (the kernels are included) so that the device status word is a single
// symbol.  Built for sm_100a only:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo --fmad=false -shared ...
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>

#include "qt2_internal.h"
#include "qt2_device.cuh"
#include "quant_kernels.cuh"
#include "msed_kernel.cuh"
#include "gemm_kernel.cuh"
#include "gemm2_kernel.cuh"

namespace qt2 {

// ---------------------------------------------------------------------------------------------
// host-side fault injection and per-device caches
// ---------------------------------------------------------------------------------------------
static std::atomic<qt2_fault_hook> g_fault_hook{nullptr};
static std::atomic<void *> g_fault_user{nullptr};

int fault_at(const char *site) {
    const qt2_fault_hook h = g_fault_hook.load(std::memory_order_acquire);
    if (h == nullptr) return kFaultNone;
    const int a = h(site, g_fault_user.load(std::memory_order_acquire));
    return (a == kFaultFail || a == kFaultSkip) ? a : kFaultNone;
}

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return dev;
}

// One-time set-up per device (function attributes, occupancy): f() runs with the device
// current until it has succeeded once there.  A process that drives several GPUs sets every
// kernel up on each of them.
struct PerDeviceOnce {
    std::atomic<int> done[kMaxDevices];
    template <class F>
    cudaError_t run(F &&f) {
        const int dev = current_device();
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
        const cudaError_t e = f();
        if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
        return e;
    }
};

// Launch sites consult the fault hook: a failure is reported as a failed launch, a skip as a
// successful one, and in both cases nothing is launched.
#define QT2_LAUNCH_SITE()                                        \
    do {                                                         \
        const int fa_ = fault_at("launch");                      \
        if (fa_ == kFaultFail) return cudaErrorLaunchFailure;    \
        if (fa_ == kFaultSkip) return cudaSuccess;               \
    } while (0)

static cudaError_t memset_async(void *p, size_t n, cudaStream_t s) {
    const int fa = fault_at("memset");
    if (fa == kFaultFail) return cudaErrorInvalidValue;
    if (fa == kFaultSkip) return cudaSuccess;
    return cudaMemsetAsync(p, 0, n, s);
}

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
static int sm_count() {
    static std::atomic<int> cached[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int v = cached[dev].load();
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            v = 148;
        }
        cached[dev].store(v);
    }
    return v;
}

cudaError_t launch_amax_bf16(const uint16_t *x, int64_t R, int64_t C, int64_t ld, uint32_t *amax_word,
                             cudaStream_t s) {
    QT2_LAUNCH_SITE();
    const int64_t warps_needed = R;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((warps_needed + 7) / 8, (int64_t)sm_count() * 8));
    amax_bf16_kernel<<<blocks, 256, 0, s>>>(x, R, C, ld, amax_word);
    return cudaGetLastError();
}


// The forward quantizer as one cooperative launch (words: 2 zeroed words, the max and the
// barrier's arrivals).  The grid is every CTA that fits on the device at once.
cudaError_t launch_fwd46_coop(const uint16_t *x, int64_t R, int64_t C, int64_t ld, uint32_t *words, DevView out,
                              cudaStream_t s) {
    QT2_LAUNCH_SITE();
    static PerDeviceOnce once;
    static std::atomic<int> occupancy[kMaxDevices];
    const cudaError_t occ_err = once.run([] {
        int v = 0;
        const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fwd46_coop_kernel, 256, 0);
        if (e == cudaSuccess) occupancy[current_device()].store(v);
        return e;
    });
    if (occ_err != cudaSuccess) return occ_err;
    const int per_sm = occupancy[current_device()].load();
    if (per_sm < 1) return cudaErrorLaunchOutOfResources;
    const int64_t groups = R * (C >> 4);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((groups + 255) / 256, (int64_t)per_sm * sm_count()));
    uint8_t *codes = out.codes, *scales = out.scales;
    float *ts = out.tensor_scale;
    void *args[] = {(void *)&x, (void *)&R, (void *)&C, (void *)&ld, (void *)&words, (void *)&codes, (void *)&scales,
                    (void *)&ts};
    return cudaLaunchCooperativeKernel((const void *)fwd46_coop_kernel, dim3((unsigned)blocks), dim3(256), args, 0, s);
}

// Self-test of the error path of a device wait: one thread waits on an mbarrier that nothing
// arrives at; the bounded wait gives up after kWaitLimitNs and records QT2_ERR_TIMEOUT.
__global__ void selftest_wait_kernel() {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0);
}

// Self-test of the checked build's store check: one byte at offset 40 of a 64-byte array,
// checked against a stated extent of 32 bytes (skipped and reported in the checked build; made,
// inside the array, in the product build, which has no checks).
__device__ unsigned char g_bounds_probe[64];
__global__ void selftest_bounds_kernel() {
    unsigned char *const p = g_bounds_probe + 40;
    if (threadIdx.x == 0 && QT2_STORE_OK(p, 1, g_bounds_probe, 32)) *p = 1;
}

// Self-test of the quantizers' division shortcuts: for every binary32 value x whose biased
// exponent lies in [e_lo, e_hi] (every significand), rcp_rn(x) against the IEEE reciprocal
// (counted in mismatches[0]) and div6_rn(x) against the IEEE quotient x/6 (mismatches[1]).
__global__ void selftest_division_kernel(uint32_t e_lo, uint32_t e_hi, unsigned long long *mismatches) {
    const uint64_t n = (uint64_t)(e_hi - e_lo + 1) << 23;
    unsigned bad_r = 0, bad_d = 0;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
        const float x = __uint_as_float((uint32_t)(((uint64_t)e_lo << 23) + i));
        bad_r += __float_as_uint(rcp_rn(x)) != __float_as_uint(__frcp_rn(x));
        bad_d += __float_as_uint(div6_rn(x)) != __float_as_uint(__fdiv_rn(x, 6.0f));
    }
    bad_r = __reduce_add_sync(0xFFFFFFFFu, bad_r);
    bad_d = __reduce_add_sync(0xFFFFFFFFu, bad_d);
    if ((threadIdx.x & 31) == 0) {
        if (bad_r) atomicAdd(&mismatches[0], (unsigned long long)bad_r);
        if (bad_d) atomicAdd(&mismatches[1], (unsigned long long)bad_d);
    }
}

cudaError_t launch_fwd46_local(const uint16_t *x, int64_t R, int64_t C, int64_t ld, DevView out, cudaStream_t s) {
    QT2_LAUNCH_SITE();
    fwd46_local_kernel<<<(unsigned)(R / 128 * kLocalCluster), kLocalThreads, 0, s>>>(x, R, C, ld, out.codes,
                                                                                     out.scales, out.tensor_scale);
    return cudaGetLastError();
}

cudaError_t launch_fwd46_sq(const uint16_t *x, int64_t R, int64_t C, int64_t ld, const uint32_t *amax_word,
                            DevView row, DevView col, cudaStream_t s) {
    QT2_LAUNCH_SITE();
    const int64_t pairs = (R / 16) * (C / 16) / 2;   // two 16x16 blocks per warp
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((pairs + 7) / 8, (int64_t)sm_count() * 16));
    fwd46_sq_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, R, C, ld, amax_word, row.codes, row.scales, row.tensor_scale,
                                                     col.codes, col.scales, col.tensor_scale);
    return cudaGetLastError();
}

template <int MODE, bool ROW, bool COL>
static cudaError_t launch_rot_variant(const CUtensorMap &tmap, int64_t R, int64_t C, uint64_t seed,
                                      const RotViews &out, cudaStream_t s) {
    QT2_LAUNCH_SITE();
    static PerDeviceOnce once;
    const cudaError_t attr_err = once.run([] {
        return cudaFuncSetAttribute(msed_kernel<MODE, ROW, COL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    MsedCfg::kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int64_t ntiles = (R >> 7) * (C >> 7);
    // one CTA per SM; a single view needs two tiles per CTA to keep both halves busy
    const int64_t per_cta = (ROW && COL) ? 1 : 2;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((ntiles + per_cta - 1) / per_cta, sm_count()));
    msed_kernel<MODE, ROW, COL><<<(unsigned)grid, MsedCfg::kThreads, MsedCfg::kSmemBytes, s>>>(tmap, R, C, seed, out);
    return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_rot(const CUtensorMap &tmap, int64_t R, int64_t C, bool do_row, bool do_col, uint64_t seed,
                              const RotViews &out, cudaStream_t s) {
    if (do_row && do_col) return launch_rot_variant<MODE, true, true>(tmap, R, C, seed, out, s);
    if (do_row) return launch_rot_variant<MODE, true, false>(tmap, R, C, seed, out, s);
    return launch_rot_variant<MODE, false, true>(tmap, R, C, seed, out, s);
}

cudaError_t launch_msed_tiles(const CUtensorMap &tmap, int64_t R, int64_t C, bool do_row, bool do_col,
                              uint64_t seed, DevView row, DevView col, float *P_row, float *P_col,
                              uint32_t *amax_row, uint32_t *amax_col, cudaStream_t s) {
    RotViews out{};
    out.row_codes = row.codes;
    out.col_codes = col.codes;
    out.row_P = P_row;
    out.col_P = P_col;
    out.row_amax = amax_row;
    out.col_amax = amax_col;
    return launch_rot<kModeEden>(tmap, R, C, do_row, do_col, seed, out, s);
}

// X's forward row view and MS-EDEN column view from one read (amax_x: the max pass's word,
// read; amax_col: the column view's max |y|, merged).
cudaError_t launch_fwd46_msed_col(const CUtensorMap &tmap, int64_t R, int64_t C, uint64_t seed, DevView row,
                                  DevView col, float *P_col, uint32_t *amax_x, uint32_t *amax_col, cudaStream_t s) {
    RotViews out{};
    out.row_codes = row.codes;
    out.row_scales = row.scales;
    out.row_g = row.tensor_scale;
    out.row_amax = amax_x;
    out.col_codes = col.codes;
    out.col_P = P_col;
    out.col_amax = amax_col;
    return launch_rot_variant<kModeFwdRowEdenCol, true, true>(tmap, R, C, seed, out, s);
}

static FinalizeJob finalize_job(const float *P, int64_t R, int64_t C, const uint32_t *amax_word, uint32_t tid,
                                DevView out, int64_t max_blocks) {
    const int64_t words = (R * C) >> 6;
    FinalizeJob j{reinterpret_cast<const float4 *>(P), R, C, amax_word, tid,
                  reinterpret_cast<uint32_t *>(out.scales), out.tensor_scale, 0};
    j.blocks = std::max<int64_t>(1, std::min<int64_t>((words + 255) / 256, max_blocks));
    return j;
}

// Finalize one view, or two in one launch when `P_b` is given (the grid is split by size).
cudaError_t launch_msed_finalize(const float *P_a, int64_t R_a, int64_t C_a, const uint32_t *amax_a, uint32_t tid_a,
                                 DevView out_a, const float *P_b, int64_t R_b, int64_t C_b, const uint32_t *amax_b,
                                 uint32_t tid_b, DevView out_b, uint64_t seed, cudaStream_t s) {
    QT2_LAUNCH_SITE();
    const int64_t cap = (int64_t)sm_count() * 16;
    FinalizeJob ja = finalize_job(P_a, R_a, C_a, amax_a, tid_a, out_a, P_b ? cap / 2 : cap);
    FinalizeJob jb = P_b ? finalize_job(P_b, R_b, C_b, amax_b, tid_b, out_b, cap / 2) : ja;
    const int64_t blocks = ja.blocks + (P_b ? jb.blocks : 0);
    msed_finalize_kernel<<<(unsigned)blocks, 256, 0, s>>>(ja, jb, seed);
    return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_gemm_bn(const CUtensorMap &tmA, const CUtensorMap &tmB, DevView a, DevView b, int64_t M,
                                  int64_t N, int64_t K, float alpha, void *c, int c_dtype, int64_t ldc,
                                  cudaStream_t s, int local) {
    QT2_LAUNCH_SITE();
    static PerDeviceOnce once;
    const cudaError_t attr_err = once.run([] {
        return cudaFuncSetAttribute(gemm_nvfp4_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    GemmCfg<BN>::kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    dim3 grid((unsigned)(N / BN), (unsigned)(M / kGemmBM));
    gemm_nvfp4_kernel<BN><<<grid, kGemmThreads, GemmCfg<BN>::kSmemBytes, s>>>(
        tmA, tmB, a.scales, b.scales, a.tensor_scale, b.tensor_scale, alpha, c, ldc, (int)K, c_dtype, local);
    return cudaGetLastError();
}

cudaError_t launch_gemm_nvfp4(const CUtensorMap &tmA, const CUtensorMap &tmB, DevView a, DevView b, int64_t M,
                              int64_t N, int64_t K, float alpha, void *c, int c_dtype, int64_t ldc, cudaStream_t s,
                              int local) {
    if (N % 256 == 0) return launch_gemm_bn<256>(tmA, tmB, a, b, M, N, K, alpha, c, c_dtype, ldc, s, local);
    return launch_gemm_bn<128>(tmA, tmB, a, b, M, N, K, alpha, c, c_dtype, ldc, s, local);
}

cudaError_t launch_gemm_nvfp4_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmSFA,
                                   const CUtensorMap &tmSFB, DevView a, DevView b, int64_t M,
                                   int64_t N, int64_t K, float alpha, void *c, int c_dtype, int64_t ldc,
                                   cudaStream_t s, int local) {
    QT2_LAUNCH_SITE();
    static PerDeviceOnce once;
    const cudaError_t attr_err = once.run([] {
        return cudaFuncSetAttribute(gemm_nvfp4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Gemm2Cfg::kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int64_t tiles = (M / 256) * (N / 256);
    const int64_t clusters = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count() / 2));
    // run the tiles along M first when A is the smaller operand (see the kernel's tile order)
    const int m_fast = M < N ? 1 : 0;
    gemm_nvfp4_pair_kernel<<<(unsigned)(2 * clusters), Gemm2Cfg::kThreads, Gemm2Cfg::kSmemBytes, s>>>(
        tmA, tmB, tmSFA, tmSFB, a.tensor_scale, b.tensor_scale, alpha, c, ldc, (int)M, (int)N, (int)K, c_dtype,
        local, m_fast);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime; no libcuda link needed)
// ---------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    const int fa = fault_at("tensor_map");
    if (fa == kFaultFail) return false;
    if (fa == kFaultSkip) {
        std::memset(map, 0, sizeof(*map));
        return true;
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace qt2

// =============================================================================================
// C ABI
// =============================================================================================
using namespace qt2;

namespace {

constexpr size_t kWsAlign = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Dimensions reach the kernels as 32-bit ints (GEMM extents, TMA coordinates): below 2^31.
bool dim_ok(int64_t d) { return d > 0 && d % 128 == 0 && d < (int64_t(1) << 31); }

qt2_status check_device() {
    const int fa = fault_at("device");
    if (fa == kFaultFail) return QT2_ERR_DEVICE;
    if (fa == kFaultSkip) return QT2_OK;
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return QT2_ERR_DEVICE;
    }
    if (dev < 64) {
        int v = cached[dev].load();
        if (v == 1) return QT2_OK;
        if (v == 2) return QT2_ERR_DEVICE;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return QT2_ERR_DEVICE;
    }
    const bool ok = (major == 10 && minor == 0);
    if (dev < 64) cached[dev].store(ok ? 1 : 2);
    return ok ? QT2_OK : QT2_ERR_DEVICE;
}

qt2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QT2_OK : QT2_ERR_CUDA; }

// Bump allocator over the caller's workspace.
struct Carve {
    uint8_t *base;
    size_t used = 0;
    explicit Carve(void *b) : base(static_cast<uint8_t *>(b)) {}
    uint8_t *take(size_t bytes) {
        uint8_t *p = base ? base + used : nullptr;
        used = align_up(used + bytes, kWsAlign);
        return p;
    }
};

bool view_ok(const qt2_nvfp4_view *v) {
    return v && v->codes && v->scales && v->tensor_scale && aligned16(v->codes) && aligned16(v->scales) &&
           (reinterpret_cast<uintptr_t>(v->tensor_scale) & 3u) == 0;
}

DevView dev_view(const qt2_nvfp4_view *v) {
    return DevView{static_cast<uint8_t *>(v->codes), static_cast<uint8_t *>(v->scales), v->tensor_scale};
}

// Workspace of one MS-EDEN call: amax words (2), then P_row, P_col.
size_t msed_ws(int64_t rows, int64_t cols, int mask, float **P_row, float **P_col, uint32_t **amax, void *ws) {
    Carve c(ws);
    *amax = reinterpret_cast<uint32_t *>(c.take(2 * sizeof(uint32_t)));
    *P_row = (mask & QT2_LAYOUT_ROW) ? reinterpret_cast<float *>(c.take((size_t)rows * cols / 16 * 4)) : nullptr;
    *P_col = (mask & QT2_LAYOUT_COL) ? reinterpret_cast<float *>(c.take((size_t)rows * cols / 16 * 4)) : nullptr;
    return c.used;
}

qt2_status validate_bf16(const void *x, int64_t rows, int64_t cols, int64_t ld) {
    if (!x) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols) || ld < cols) return QT2_ERR_SHAPE;
    if (!aligned16(x) || ld % 8 != 0) return QT2_ERR_ALIGN;
    return QT2_OK;
}

// Enqueue an MS-EDEN quantization of x (rows x cols, ld) into the requested views.
qt2_status msed_enqueue(const void *x, int64_t rows, int64_t cols, int64_t ld, int mask, uint64_t seed, uint32_t tid_row,
                        uint32_t tid_col, DevView row, DevView col, float *P_row, float *P_col, uint32_t *amax,
                        cudaStream_t s) {
    CUtensorMap tmap;
    if (!encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, 64,
                        128, CU_TENSOR_MAP_SWIZZLE_128B))
        return QT2_ERR_CUDA;
    cudaError_t e = memset_async(amax, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    e = launch_msed_tiles(tmap, rows, cols, (mask & QT2_LAYOUT_ROW) != 0, (mask & QT2_LAYOUT_COL) != 0, seed, row, col,
                          P_row, P_col, amax, amax + 1, s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    if ((mask & QT2_LAYOUT_ROW) && (mask & QT2_LAYOUT_COL))
        e = launch_msed_finalize(P_row, rows, cols, amax, tid_row, row, P_col, cols, rows, amax + 1, tid_col, col,
                                 seed, s);
    else if (mask & QT2_LAYOUT_ROW)
        e = launch_msed_finalize(P_row, rows, cols, amax, tid_row, row, nullptr, 0, 0, nullptr, 0, row, seed, s);
    else
        e = launch_msed_finalize(P_col, cols, rows, amax + 1, tid_col, col, nullptr, 0, 0, nullptr, 0, col, seed, s);
    return from_cuda(e);
}

// X's forward view and MS-EDEN column view: max pass, one fused pass, the column view's finalize.
// amax: 2 words (the input's max |x|, the column view's max |y|).
qt2_status fwd46_msed_col_enqueue(const void *x, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
                                  uint32_t tid_col, DevView row, DevView col, float *P_col, uint32_t *amax,
                                  cudaStream_t s) {
    CUtensorMap tmap;
    if (!encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, 64,
                        128, CU_TENSOR_MAP_SWIZZLE_128B))
        return QT2_ERR_CUDA;
    cudaError_t e = memset_async(amax, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    e = launch_amax_bf16(static_cast<const uint16_t *>(x), rows, cols, ld, amax, s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    e = launch_fwd46_msed_col(tmap, rows, cols, seed, row, col, P_col, amax, amax + 1, s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    return from_cuda(
        launch_msed_finalize(P_col, cols, rows, amax + 1, tid_col, col, nullptr, 0, 0, nullptr, 0, col, seed, s));
}

qt2_status fwd46_sq_enqueue(const void *x, int64_t rows, int64_t cols, int64_t ld, DevView row, DevView col,
                            uint32_t *amax, cudaStream_t s) {
    cudaError_t e = memset_async(amax, sizeof(uint32_t), s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    e = launch_amax_bf16(static_cast<const uint16_t *>(x), rows, cols, ld, amax, s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    return from_cuda(launch_fwd46_sq(static_cast<const uint16_t *>(x), rows, cols, ld, amax, row, col, s));
}

// The forward quantizer: one cooperative launch (max, grid barrier, quantization).
// words: 2 words of scratch (the max and the barrier's arrival count).
qt2_status fwd46_enqueue(const void *x, int64_t rows, int64_t cols, int64_t ld, DevView out, uint32_t *words,
                         cudaStream_t s) {
    cudaError_t e = memset_async(words, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    return from_cuda(launch_fwd46_coop(static_cast<const uint16_t *>(x), rows, cols, ld, words, out, s));
}

qt2_status gemm_enqueue(DevView a, DevView b, int64_t M, int64_t N, int64_t K, float alpha, void *c, int c_dtype,
                        int64_t ldc, cudaStream_t s, int local = 0) {
    CUtensorMap tmA, tmB;
    if (M % 256 == 0 && N % 256 == 0) {
        // pair kernel: 128-row code boxes per SM, scale atoms as rows of K/64 512-byte atoms
        CUtensorMap tmSFA, tmSFB;
        if (!encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2,
                            128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, b.codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                            128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_tmap_2d(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT64, a.scales, (uint64_t)K, (uint64_t)M / 128,
                            (uint64_t)K * 8, 256, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_tmap_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT64, b.scales, (uint64_t)K, (uint64_t)N / 128,
                            (uint64_t)K * 8, 256, 2, CU_TENSOR_MAP_SWIZZLE_NONE))
            return QT2_ERR_CUDA;
        return from_cuda(
            launch_gemm_nvfp4_pair(tmA, tmB, tmSFA, tmSFB, a, b, M, N, K, alpha, c, c_dtype, ldc, s, local));
    }
    const int bn = (N % 256 == 0) ? 256 : 128;
    if (!encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, 128,
                        kGemmBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, b.codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 128,
                        (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B))
        return QT2_ERR_CUDA;
    return from_cuda(launch_gemm_nvfp4(tmA, tmB, a, b, M, N, K, alpha, c, c_dtype, ldc, s, local));
}

// Views carved from a workspace: codes, scales, tensor scale.
DevView carve_view(Carve &c, int64_t R, int64_t C) {
    DevView v;
    v.codes = c.take((size_t)R * C / 2);
    v.scales = c.take((size_t)R * C / 16);
    v.tensor_scale = reinterpret_cast<float *>(c.take(sizeof(float)));
    return v;
}

size_t linear_fwd_layout(int64_t M, int64_t K, int64_t N, void *ws, DevView *vx, DevView *vw, uint32_t **amax) {
    Carve c(ws);
    *amax = reinterpret_cast<uint32_t *>(c.take(4 * sizeof(uint32_t)));   // 2 words per quantizer call
    *vx = carve_view(c, M, K);
    *vw = carve_view(c, N, K);
    return c.used;
}

struct BwdLayout {
    DevView dy_row, dy_col, w_col, x_col;
    float *P_dy_row, *P_dy_col, *P_w_col, *P_x_col;
    uint32_t *amax;   // 6 words: dY row/col, W (col at +1), X (col at +1)
};

size_t linear_bwd_layout(int64_t M, int64_t K, int64_t N, void *ws, BwdLayout *L) {
    Carve c(ws);
    L->amax = reinterpret_cast<uint32_t *>(c.take(6 * sizeof(uint32_t)));
    L->dy_row = carve_view(c, M, N);
    L->dy_col = carve_view(c, N, M);
    L->w_col = carve_view(c, K, N);
    L->x_col = carve_view(c, K, M);
    L->P_dy_row = reinterpret_cast<float *>(c.take((size_t)M * N / 16 * 4));
    L->P_dy_col = reinterpret_cast<float *>(c.take((size_t)M * N / 16 * 4));
    L->P_w_col = reinterpret_cast<float *>(c.take((size_t)N * K / 16 * 4));
    L->P_x_col = reinterpret_cast<float *>(c.take((size_t)M * K / 16 * 4));
    return c.used;
}

// Workspace of qt2_linear_bwd_views: dY's two views and their pre-scales.
struct BwdViewsLayout {
    DevView dy_row, dy_col;
    float *P_dy_row, *P_dy_col;
    uint32_t *amax;   // 2 words: dY row, col
};

size_t linear_bwd_views_layout(int64_t M, int64_t N, void *ws, BwdViewsLayout *L) {
    Carve c(ws);
    L->amax = reinterpret_cast<uint32_t *>(c.take(2 * sizeof(uint32_t)));
    L->dy_row = carve_view(c, M, N);
    L->dy_col = carve_view(c, N, M);
    L->P_dy_row = reinterpret_cast<float *>(c.take((size_t)M * N / 16 * 4));
    L->P_dy_col = reinterpret_cast<float *>(c.take((size_t)M * N / 16 * 4));
    return c.used;
}

}  // namespace

namespace qt2 {

// Hooks for the library's other translation unit (the workspace-free MS-EDEN entry point).
// They reuse the checks and the enqueue sequence of qt2_quant_msedEN on caller-given scratch.
qt2_status msed_check_args(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                           const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out) {
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (layout_mask < 1 || layout_mask > 3) return QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_ROW) && !view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_COL) && !view_ok(col_out)) return col_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    return QT2_OK;
}

size_t msed_scratch_bytes(int64_t rows, int64_t cols, int layout_mask) {
    float *a, *b;
    uint32_t *c;
    return msed_ws(rows, cols, layout_mask, &a, &b, &c, nullptr);
}

qt2_status msed_device_check() { return check_device(); }

// Elementwise-SR view(s) of the rotated tensor: a max pass over the rotated view(s), then the
// quantize pass (the SR scales need the tensor scale first).
size_t sr_ws(uint32_t **amax, void *ws) {
    Carve c(ws);
    *amax = reinterpret_cast<uint32_t *>(c.take(2 * sizeof(uint32_t)));
    return c.used;
}
qt2_status sr_enqueue(const void *x, int64_t rows, int64_t cols, int64_t ld, int mask, uint64_t seed, uint32_t tid_row,
                      uint32_t tid_col, DevView row, DevView col, uint32_t *amax, cudaStream_t s) {
    CUtensorMap tmap;
    if (!encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, 64,
                        128, CU_TENSOR_MAP_SWIZZLE_128B))
        return QT2_ERR_CUDA;
    cudaError_t e = memset_async(amax, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    const bool do_row = (mask & QT2_LAYOUT_ROW) != 0, do_col = (mask & QT2_LAYOUT_COL) != 0;
    RotViews out{};
    out.row_codes = row.codes;
    out.col_codes = col.codes;
    out.row_scales = row.scales;
    out.col_scales = col.scales;
    out.row_amax = amax;
    out.col_amax = amax + 1;
    out.row_g = row.tensor_scale;
    out.col_g = col.tensor_scale;
    out.tid_row = tid_row;
    out.tid_col = tid_col;
    e = launch_rot<kModeMax>(tmap, rows, cols, do_row, do_col, seed, out, s);
    if (e != cudaSuccess) return QT2_ERR_CUDA;
    e = launch_rot<kModeSr>(tmap, rows, cols, do_row, do_col, seed, out, s);
    return from_cuda(e);
}

qt2_status msed_enqueue_on_scratch(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                                   uint64_t seed, uint32_t tensor_id_row, uint32_t tensor_id_col,
                                   const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *scratch,
                                   cudaStream_t stream) {
    float *P_row, *P_col;
    uint32_t *amax;
    msed_ws(rows, cols, layout_mask, &P_row, &P_col, &amax, scratch);
    const DevView none{nullptr, nullptr, nullptr};
    return msed_enqueue(x_bf16, rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
                        (layout_mask & QT2_LAYOUT_ROW) ? dev_view(row_out) : none,
                        (layout_mask & QT2_LAYOUT_COL) ? dev_view(col_out) : none, P_row, P_col, amax, stream);
}

}  // namespace qt2

extern "C" {

int qt2_version(void) { return 101; }

void qt2_set_fault_hook(qt2_fault_hook hook, void *user) {
    g_fault_user.store(user, std::memory_order_release);
    g_fault_hook.store(hook, std::memory_order_release);
}

const char *qt2_status_string(qt2_status s) {
    switch (s) {
        case QT2_OK: return "ok";
        case QT2_ERR_INVALID_ARG: return "invalid argument";
        case QT2_ERR_SHAPE: return "bad shape (dimensions must be positive multiples of 128, ld >= cols)";
        case QT2_ERR_ALIGN: return "misaligned pointer or leading dimension (16-byte alignment required)";
        case QT2_ERR_WORKSPACE: return "workspace missing or too small";
        case QT2_ERR_CUDA: return "CUDA error";
        case QT2_ERR_TIMEOUT: return "device-side wait timed out";
        case QT2_ERR_DEVICE: return "no sm_100 device";
        case QT2_ERR_NONFINITE: return "input holds inf or NaN";
        case QT2_ERR_BOUNDS: return "a kernel store left its output array (checked build; store skipped)";
    }
    return "unknown status";
}

qt2_status qt2_device_status(qt2_stream_t stream, int *code) {
    QT2_TRACE();
    if (!code) return QT2_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return QT2_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return QT2_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return QT2_ERR_CUDA;
    *code = v;
    return QT2_OK;
}

qt2_status qt2_quant_fwd46_workspace_size(int64_t rows, int64_t cols, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols)) return QT2_ERR_SHAPE;
    *bytes = kWsAlign;
    return QT2_OK;
}

qt2_status qt2_quant_fwd46(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                           const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                           size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    (void)col_out;
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (layout_mask != QT2_LAYOUT_ROW || !row_out) return QT2_ERR_INVALID_ARG;
    if (!view_ok(row_out)) return row_out->codes && row_out->scales && row_out->tensor_scale ? QT2_ERR_ALIGN
                                                                                             : QT2_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < kWsAlign) return QT2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QT2_ERR_ALIGN;
    if ((st = check_device()) != QT2_OK) return st;
    return fwd46_enqueue(x_bf16, rows, cols, ld, dev_view(row_out), static_cast<uint32_t *>(workspace),
                         reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_quant_msedEN_workspace_size(int64_t rows, int64_t cols, int layout_mask, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (layout_mask < 1 || layout_mask > 3) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols)) return QT2_ERR_SHAPE;
    float *a, *b;
    uint32_t *c;
    *bytes = msed_ws(rows, cols, layout_mask, &a, &b, &c, nullptr);
    return QT2_OK;
}

qt2_status qt2_quant_msedEN(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                            uint64_t seed, uint32_t tensor_id_row, uint32_t tensor_id_col,
                            const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                            size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (layout_mask < 1 || layout_mask > 3) return QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_ROW) && !view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_COL) && !view_ok(col_out)) return col_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    float *P_row, *P_col;
    uint32_t *amax;
    if (ws_bytes < msed_ws(rows, cols, layout_mask, &P_row, &P_col, &amax, workspace)) return QT2_ERR_WORKSPACE;
    if ((st = check_device()) != QT2_OK) return st;
    const DevView none{nullptr, nullptr, nullptr};
    return msed_enqueue(x_bf16, rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
                        (layout_mask & QT2_LAYOUT_ROW) ? dev_view(row_out) : none,
                        (layout_mask & QT2_LAYOUT_COL) ? dev_view(col_out) : none, P_row, P_col, amax,
                        reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_quant_sr_workspace_size(int64_t rows, int64_t cols, int layout_mask, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (layout_mask < 1 || layout_mask > 3) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols)) return QT2_ERR_SHAPE;
    uint32_t *a;
    *bytes = sr_ws(&a, nullptr);
    return QT2_OK;
}
qt2_status qt2_quant_sr(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask, uint64_t seed,
                        uint32_t tensor_id_row, uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                        const qt2_nvfp4_view *col_out, void *workspace, size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (layout_mask < 1 || layout_mask > 3) return QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_ROW) && !view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if ((layout_mask & QT2_LAYOUT_COL) && !view_ok(col_out)) return col_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    uint32_t *amax;
    if (ws_bytes < sr_ws(&amax, workspace)) return QT2_ERR_WORKSPACE;
    if ((st = check_device()) != QT2_OK) return st;
    const DevView none{nullptr, nullptr, nullptr};
    return sr_enqueue(x_bf16, rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
                      (layout_mask & QT2_LAYOUT_ROW) ? dev_view(row_out) : none,
                      (layout_mask & QT2_LAYOUT_COL) ? dev_view(col_out) : none, amax,
                      reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_gemm_nvfp4(const qt2_nvfp4_view *a, const qt2_nvfp4_view *b, int64_t M, int64_t N, int64_t K,
                          float alpha, void *c, int c_dtype, int64_t ldc, qt2_stream_t stream) {
    QT2_TRACE();
    if (!a || !b || !c) return QT2_ERR_INVALID_ARG;
    if (c_dtype != QT2_DTYPE_BF16 && c_dtype != QT2_DTYPE_F32) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K) || ldc < N) return QT2_ERR_SHAPE;
    if (!view_ok(a) || !view_ok(b)) return (a->codes && a->scales && a->tensor_scale && b->codes && b->scales &&
                                            b->tensor_scale)
                                               ? QT2_ERR_ALIGN
                                               : QT2_ERR_INVALID_ARG;
    if (!aligned16(c) || ldc % 8 != 0) return QT2_ERR_ALIGN;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    return gemm_enqueue(dev_view(a), dev_view(b), M, N, K, alpha, c, c_dtype, ldc,
                        reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_linear_fwd_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    DevView a, b;
    uint32_t *w;
    *bytes = linear_fwd_layout(M, K, N, nullptr, &a, &b, &w);
    return QT2_OK;
}

qt2_status qt2_linear_fwd(const void *x, const void *w, int64_t M, int64_t K, int64_t N, void *y_bf16,
                          void *workspace, size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    if (!x || !w || !y_bf16) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y_bf16)) return QT2_ERR_ALIGN;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    DevView vx, vw;
    uint32_t *amax;
    if (ws_bytes < linear_fwd_layout(M, K, N, workspace, &vx, &vw, &amax)) return QT2_ERR_WORKSPACE;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = fwd46_enqueue(x, M, K, K, vx, amax, s)) != QT2_OK) return st;
    if ((st = fwd46_enqueue(w, N, K, K, vw, amax + 2, s)) != QT2_OK) return st;
    return gemm_enqueue(vx, vw, M, N, K, 1.0f, y_bf16, QT2_DTYPE_BF16, N, s);
}

qt2_status qt2_linear_bwd_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    BwdLayout L;
    *bytes = linear_bwd_layout(M, K, N, nullptr, &L);
    return QT2_OK;
}

qt2_status qt2_linear_bwd(const void *dy, const void *x, const void *w, int64_t M, int64_t K, int64_t N,
                          uint64_t seed, void *dx_bf16, void *dw, int dw_dtype, void *workspace, size_t ws_bytes,
                          qt2_stream_t stream) {
    QT2_TRACE();
    if (!dy || !x || !w || !dx_bf16 || !dw) return QT2_ERR_INVALID_ARG;
    if (dw_dtype != QT2_DTYPE_BF16 && dw_dtype != QT2_DTYPE_F32) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    if (!aligned16(dy) || !aligned16(x) || !aligned16(w) || !aligned16(dx_bf16) || !aligned16(dw))
        return QT2_ERR_ALIGN;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    BwdLayout L;
    if (ws_bytes < linear_bwd_layout(M, K, N, workspace, &L)) return QT2_ERR_WORKSPACE;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // dY: both views from one read; W and X: column views (rotated along N and M respectively)
    if ((st = msed_enqueue(dy, M, N, N, QT2_LAYOUT_BOTH, seed, QT2_TID_DY_ROW, QT2_TID_DY_COL, L.dy_row, L.dy_col,
                           L.P_dy_row, L.P_dy_col, L.amax, s)) != QT2_OK)
        return st;
    const DevView none{nullptr, nullptr, nullptr};
    if ((st = msed_enqueue(w, N, K, K, QT2_LAYOUT_COL, seed, 0, QT2_TID_W_COL, none, L.w_col, nullptr, L.P_w_col,
                           L.amax + 2, s)) != QT2_OK)
        return st;
    if ((st = msed_enqueue(x, M, K, K, QT2_LAYOUT_COL, seed, 0, QT2_TID_X_COL, none, L.x_col, nullptr, L.P_x_col,
                           L.amax + 4, s)) != QT2_OK)
        return st;
    // dgrad: dX[M][K] = 2^-7 * dY_row[M][N] . W_col[K][N]^T
    if ((st = gemm_enqueue(L.dy_row, L.w_col, M, K, N, 0x1p-7f, dx_bf16, QT2_DTYPE_BF16, K, s)) != QT2_OK) return st;
    // wgrad: dW[N][K] = 2^-7 * dY_col[N][M] . X_col[K][M]^T
    return gemm_enqueue(L.dy_col, L.x_col, N, K, M, 0x1p-7f, dw, dw_dtype, K, s);
}

qt2_status qt2_selftest_wait_timeout(qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    const int fa = fault_at("launch");
    if (fa == kFaultFail) return QT2_ERR_CUDA;
    if (fa == kFaultSkip) return QT2_OK;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return from_cuda(cudaGetLastError());
}

int qt2_build_checked(void) {
#ifdef QT2_CHECKED
    return 1;
#else
    return 0;
#endif
}

qt2_status qt2_selftest_bounds(qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    const int fa = fault_at("launch");
    if (fa == kFaultFail) return QT2_ERR_CUDA;
    if (fa == kFaultSkip) return QT2_OK;
    selftest_bounds_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return from_cuda(cudaGetLastError());
}

qt2_status qt2_selftest_division(uint32_t exp_lo, uint32_t exp_hi, unsigned long long *mismatches,
                                  qt2_stream_t stream) {
    QT2_TRACE();
    if (!mismatches || exp_lo < 1 || exp_hi > 254 || exp_lo > exp_hi) return QT2_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mismatches) & 7u) != 0) return QT2_ERR_ALIGN;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    const int fa = fault_at("launch");
    if (fa == kFaultFail) return QT2_ERR_CUDA;
    if (fa == kFaultSkip) return QT2_OK;
    selftest_division_kernel<<<(unsigned)sm_count() * 8, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        exp_lo, exp_hi, mismatches);
    return from_cuda(cudaGetLastError());
}

qt2_status qt2_quant_fwd46_local(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                 const qt2_nvfp4_view *row_out, qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (!view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if ((st = check_device()) != QT2_OK) return st;
    return from_cuda(launch_fwd46_local(static_cast<const uint16_t *>(x_bf16), rows, cols, ld, dev_view(row_out),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

qt2_status qt2_gemm_nvfp4_local(const qt2_nvfp4_view *a, const qt2_nvfp4_view *b, int64_t M, int64_t N, int64_t K,
                                float alpha, void *c, int c_dtype, int64_t ldc, qt2_stream_t stream) {
    QT2_TRACE();
    if (!a || !b || !c) return QT2_ERR_INVALID_ARG;
    if (c_dtype != QT2_DTYPE_BF16 && c_dtype != QT2_DTYPE_F32) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K) || ldc < N) return QT2_ERR_SHAPE;
    if (!view_ok(a) || !view_ok(b)) return (a->codes && a->scales && a->tensor_scale && b->codes && b->scales &&
                                            b->tensor_scale)
                                               ? QT2_ERR_ALIGN
                                               : QT2_ERR_INVALID_ARG;
    if (!aligned16(c) || ldc % 8 != 0) return QT2_ERR_ALIGN;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    return gemm_enqueue(dev_view(a), dev_view(b), M, N, K, alpha, c, c_dtype, ldc,
                        reinterpret_cast<cudaStream_t>(stream), 1);
}

qt2_status qt2_quant_fwd46_sq_workspace_size(int64_t rows, int64_t cols, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols)) return QT2_ERR_SHAPE;
    *bytes = kWsAlign;
    return QT2_OK;
}

qt2_status qt2_quant_fwd46_sq(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                              const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                              size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (!view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!view_ok(col_out)) return col_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < kWsAlign) return QT2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QT2_ERR_ALIGN;
    if ((st = check_device()) != QT2_OK) return st;
    return fwd46_sq_enqueue(x_bf16, rows, cols, ld, dev_view(row_out), dev_view(col_out),
                            static_cast<uint32_t *>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_quant_fwd46_msedEN_col_workspace_size(int64_t rows, int64_t cols, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(rows) || !dim_ok(cols)) return QT2_ERR_SHAPE;
    float *a, *b;
    uint32_t *c;
    *bytes = msed_ws(rows, cols, QT2_LAYOUT_COL, &a, &b, &c, nullptr);
    return QT2_OK;
}

qt2_status qt2_quant_fwd46_msedEN_col(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
                                      uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                                      const qt2_nvfp4_view *col_out, void *workspace, size_t ws_bytes,
                                      qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = validate_bf16(x_bf16, rows, cols, ld);
    if (st != QT2_OK) return st;
    if (!view_ok(row_out)) return row_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!view_ok(col_out)) return col_out ? QT2_ERR_ALIGN : QT2_ERR_INVALID_ARG;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    float *P_row, *P_col;
    uint32_t *amax;
    if (ws_bytes < msed_ws(rows, cols, QT2_LAYOUT_COL, &P_row, &P_col, &amax, workspace)) return QT2_ERR_WORKSPACE;
    if ((st = check_device()) != QT2_OK) return st;
    return fwd46_msed_col_enqueue(x_bf16, rows, cols, ld, seed, tensor_id_col, dev_view(row_out), dev_view(col_out),
                                  P_col, amax, reinterpret_cast<cudaStream_t>(stream));
}

qt2_status qt2_linear_bwd_views_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes) {
    if (!bytes) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    BwdViewsLayout L;
    *bytes = linear_bwd_views_layout(M, N, nullptr, &L);
    return QT2_OK;
}

qt2_status qt2_linear_bwd_views(const void *dy, int64_t M, int64_t K, int64_t N, uint64_t seed,
                                const qt2_nvfp4_view *x_col, const qt2_nvfp4_view *w_col, void *dx_bf16, void *dw,
                                int dw_dtype, void *workspace, size_t ws_bytes, qt2_stream_t stream) {
    QT2_TRACE();
    if (!dy || !x_col || !w_col || !dx_bf16 || !dw) return QT2_ERR_INVALID_ARG;
    if (dw_dtype != QT2_DTYPE_BF16 && dw_dtype != QT2_DTYPE_F32) return QT2_ERR_INVALID_ARG;
    if (!dim_ok(M) || !dim_ok(K) || !dim_ok(N)) return QT2_ERR_SHAPE;
    if (!view_ok(x_col) || !view_ok(w_col)) return QT2_ERR_ALIGN;
    if (!aligned16(dy) || !aligned16(dx_bf16) || !aligned16(dw)) return QT2_ERR_ALIGN;
    if (!workspace) return QT2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsAlign - 1)) != 0) return QT2_ERR_ALIGN;
    BwdViewsLayout L;
    if (ws_bytes < linear_bwd_views_layout(M, N, workspace, &L)) return QT2_ERR_WORKSPACE;
    qt2_status st = check_device();
    if (st != QT2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = msed_enqueue(dy, M, N, N, QT2_LAYOUT_BOTH, seed, QT2_TID_DY_ROW, QT2_TID_DY_COL, L.dy_row, L.dy_col,
                           L.P_dy_row, L.P_dy_col, L.amax, s)) != QT2_OK)
        return st;
    // dgrad: dX[M][K] = 2^-7 * dY_row[M][N] . W_col[K][N]^T; wgrad: dW[N][K] = 2^-7 * dY_col[N][M] . X_col[K][M]^T
    if ((st = gemm_enqueue(L.dy_row, dev_view(w_col), M, K, N, 0x1p-7f, dx_bf16, QT2_DTYPE_BF16, K, s)) != QT2_OK)
        return st;
    return gemm_enqueue(L.dy_col, dev_view(x_col), N, K, M, 0x1p-7f, dw, dw_dtype, K, s);
}

}  // extern "C"
