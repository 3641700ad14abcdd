// qt2_noalloc.cu -- MS-EDEN quantization without a caller-provided workspace.
//
// Some callers cannot give this library device memory for scratch: a runtime that has already
// divided all of its device memory among its own pools, a latency-critical path that must not
// call cudaMalloc (which can synchronize the device), or a plugin whose host framework owns
// the allocator and does not expose it.  For them, qt2_quant_msedEN_noalloc keeps MS-EDEN's
// scratch (the fp32 pre-scales S*p of each view and the two view maxima) in a fixed array
// that lives in this library's device image.  The array is created when a GPU loads the
// library and stays on that GPU until the process exits; nothing here allocates.
#include <mutex>

#include "qt2_internal.h"

namespace {

// The scratch array.  In host code this name is only a host-side stand-in for the device
// array: host code must never hand it to a kernel.  Its device address is looked up once per
// device (scratch_address) and that address is what the kernels receive.
static __device__ __align__(256) unsigned char g_msed_scratch[QT2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_msed_scratch on the current device; looked up at the first call on
// that device, with that device current.
qt2_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QT2_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> guard(g_lock);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_msed_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return QT2_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return QT2_OK;
}

}  // namespace

extern "C" qt2_status qt2_quant_msedEN_noalloc(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                               int layout_mask, uint64_t seed, uint32_t tensor_id_row,
                                               uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                                               const qt2_nvfp4_view *col_out, qt2_stream_t stream) {
    qt2_status st = qt2::msed_check_args(x_bf16, rows, cols, ld, layout_mask, row_out, col_out);
    if (st != QT2_OK) return st;
    if (qt2::msed_scratch_bytes(rows, cols, layout_mask) > (size_t)QT2_NOALLOC_SCRATCH_BYTES)
        return QT2_ERR_WORKSPACE;   // the tensor needs more scratch than the built-in array holds
    if ((st = qt2::msed_device_check()) != QT2_OK) return st;
    void *scratch = nullptr;
    if ((st = scratch_address(&scratch)) != QT2_OK) return st;
    // The view maxima in the scratch are zeroed by the enqueue itself; the pre-scales are
    // fully rewritten before they are read, so stale contents of an earlier call never leak.
    return qt2::msed_enqueue_on_scratch(x_bf16, rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
                                        row_out, col_out, scratch, reinterpret_cast<cudaStream_t>(stream));
}
