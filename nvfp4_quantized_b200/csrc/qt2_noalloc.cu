// qt2_noalloc.cu -- MS-EDEN quantization without a caller-provided workspace.
//
// Some callers cannot give this library device memory for scratch: a runtime that has already
// divided all of its device memory among its own pools, a latency-critical path that must not
// call cudaMalloc (which can synchronize the device), or a plugin whose host framework owns
// the allocator and does not expose it.  For them, qt2_quant_msedEN_noalloc keeps MS-EDEN's
// scratch (the two view maxima and the fp32 pre-scales S*p of each view) in a fixed array that
// lives in this library's device image.  The array is created when a GPU loads the library and
// stays on that GPU until the process exits; nothing here allocates.
#include "qt2_internal.h"

namespace {

// The view maxima take the first 256-byte slot (the same carve-up as a caller's workspace);
// the pre-scales get the QT2_NOALLOC_SCRATCH_BYTES after it.
constexpr size_t kHeaderBytes = 256;

// The scratch array.  In host code this name is only a host-side stand-in for the device
// array: host code must never hand it to a kernel.  Its device address is looked up with the
// calling device current (scratch_address), and that address is what the kernels receive.
static __device__ __align__(256) unsigned char g_msed_scratch[kHeaderBytes + QT2_NOALLOC_SCRATCH_BYTES];

// Device address of g_msed_scratch on the current device, looked up on every call: the lookup
// costs far less than the launches, and an address cached across a device reset (after which
// the library's device code is loaded again, possibly elsewhere) would be stale.
qt2_status scratch_address(void **out) {
    const int fa = qt2::fault_at("symbol");
    if (fa == qt2::kFaultFail) return QT2_ERR_CUDA;
    void *p = nullptr;
    if (fa != qt2::kFaultSkip) {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_msed_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return QT2_ERR_CUDA;
        }
    }
    *out = p;
    return QT2_OK;
}

}  // namespace

extern "C" qt2_status qt2_quant_msedEN_noalloc(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                               int layout_mask, uint64_t seed, uint32_t tensor_id_row,
                                               uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                                               const qt2_nvfp4_view *col_out, qt2_stream_t stream) {
    QT2_TRACE();
    qt2_status st = qt2::msed_check_args(x_bf16, rows, cols, ld, layout_mask, row_out, col_out);
    if (st != QT2_OK) return st;
    if (qt2::msed_scratch_bytes(rows, cols, layout_mask) > kHeaderBytes + (size_t)QT2_NOALLOC_SCRATCH_BYTES)
        return QT2_ERR_WORKSPACE;   // the tensor needs more scratch than the built-in array holds
    if ((st = qt2::msed_device_check()) != QT2_OK) return st;
    void *scratch = nullptr;
    if ((st = scratch_address(&scratch)) != QT2_OK) return st;
    // The view maxima in the scratch are zeroed by the enqueue itself; the pre-scales are
    // fully rewritten before they are read, so stale contents of an earlier call never leak.
    return qt2::msed_enqueue_on_scratch(x_bf16, rows, cols, ld, layout_mask, seed, tensor_id_row, tensor_id_col,
                                        row_out, col_out, scratch, reinterpret_cast<cudaStream_t>(stream));
}
