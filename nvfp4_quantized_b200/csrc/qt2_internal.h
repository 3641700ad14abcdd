// qt2_internal.h -- declarations shared by the qt2 library's translation units (host side).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "qt2.h"

namespace qt2 {

// One quantized view on the device (see the layout in qt2.h).
struct DevView {
    uint8_t *codes;
    uint8_t *scales;
    float *tensor_scale;
};

// Tensor-scale constants and the flush threshold of the quantizers.
constexpr float kFwd46Denominator = 1792.0f;   // 4 * 448: both 4/6 candidates keep scales <= 448
constexpr float kMsedDenominator = 1536.0f;    // 6 * 256: 1.75x headroom for the EDEN factor and SR
constexpr float kTiny = 0x1p-100f;             // below this a tensor (fwd46) or a group (MS-EDEN) is zero
constexpr float kSrCutoff = 0x1p-6f;           // E4M3 scales below 2^-6 are rounded to nearest

// Kernel launchers (one translation unit: qt2_lib.cu).  Each returns the launch status.
cudaError_t launch_amax_bf16(const uint16_t *x, int64_t R, int64_t C, int64_t ld, uint32_t *amax_word,
                             cudaStream_t s);
cudaError_t launch_msed_tiles(const CUtensorMap &tmap, int64_t R, int64_t C, bool do_row, bool do_col,
                              uint64_t seed, DevView row, DevView col, float *P_row, float *P_col,
                              uint32_t *amax_row, uint32_t *amax_col, cudaStream_t s);
cudaError_t launch_msed_finalize(const float *P_a, int64_t R_a, int64_t C_a, const uint32_t *amax_a, uint32_t tid_a,
                                 DevView out_a, const float *P_b, int64_t R_b, int64_t C_b, const uint32_t *amax_b,
                                 uint32_t tid_b, DevView out_b, uint64_t seed, cudaStream_t s);
// local = 1: a.tensor_scale / b.tensor_scale are per-128-row arrays (CTA-local views)
cudaError_t launch_gemm_nvfp4(const CUtensorMap &tmA, const CUtensorMap &tmB, DevView a, DevView b, int64_t M,
                              int64_t N, int64_t K, float alpha, void *c, int c_dtype, int64_t ldc, cudaStream_t s,
                              int local = 0);

cudaError_t launch_gemm_nvfp4_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmSFA,
                                   const CUtensorMap &tmSFB, DevView a, DevView b, int64_t M,
                                   int64_t N, int64_t K, float alpha, void *c, int c_dtype, int64_t ldc,
                                   cudaStream_t s, int local = 0);

// 2D tensor map for TMA (no multicast anywhere in this library).
bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// Host-side fault injection (qt2_set_fault_hook).  Every CUDA call the library makes while
// enqueuing passes through fault_at(site) first: kFaultNone = make the call, kFaultFail = report
// the call as failed without making it, kFaultSkip = report success without making it.
enum FaultAction { kFaultNone = 0, kFaultFail = 1, kFaultSkip = 2 };
int fault_at(const char *site);

// One NVTX range per C call, named after the call (free unless a profiler is attached).
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
};
#define QT2_TRACE() ::qt2::TraceRange qt2_trace_range_(__func__)

// Device ordinal of the calling thread (-1 when there is none).  Attribute and occupancy caches
// are kept per device, for the first kMaxDevices devices.
constexpr int kMaxDevices = 64;
int current_device();

// Hooks used by the workspace-free MS-EDEN entry point (qt2_noalloc.cu).
qt2_status msed_check_args(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                           const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out);
size_t msed_scratch_bytes(int64_t rows, int64_t cols, int layout_mask);
qt2_status msed_device_check();
qt2_status msed_enqueue_on_scratch(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                                   uint64_t seed, uint32_t tensor_id_row, uint32_t tensor_id_col,
                                   const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *scratch,
                                   cudaStream_t stream);

}  // namespace qt2
