/*
 * qt2.h -- C ABI of the Quartet II NVFP4 linear layer for NVIDIA B200 (sm_100a).
 *
 * Citations (page title, then section):
 *   [QII-th] "Quartet II ... MS-EDEN" Thai translation (itsolotime.com archives 22992): abstract,
 *            "Question 1" (fixed 128-dim rotation groups, shared rotation, small FP8 scales), §1.
 *   [QII-ru] Quartet II review, D. Avetisyan (denisavetisyan.com ?p=3427): "NVFP4 and
 *            micro-scaling", "Unbiased quantization with MS-EDEN and randomized methods".
 *   [FAF]    "Format-Aware Fusion for Fast FP4 Pretraining" (rit.work blog): "the speed-up is lost
 *            between the matmuls" (global scale sync point; both layouts from one producer).
 *   [QII-tg] Quartet II digest (quant_prune_distill post 640): "Method".
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device; the caller owns all
 *     memory (inputs, outputs, workspace).  Nothing is allocated by the library.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Returning QT2_OK means the launches were enqueued, not that they finished.
 *   - Arguments are validated on the host before any launch; on error nothing is enqueued and
 *     a negative qt2_status is returned.  Launch failures map to QT2_ERR_CUDA.  No call aborts.
 *   - bf16 matrices are row-major with a leading dimension `ld` (elements between rows,
 *     ld >= cols, ld a multiple of 8) and 16-byte aligned base pointers.
 *   - Every dimension must be a positive multiple of 128, below 2^31.
 *   - The device must be compute capability 10.0 (B200); otherwise QT2_ERR_DEVICE.
 *   - Inputs must be finite.  A quantizer that meets inf or NaN in its input records
 *     QT2_ERR_NONFINITE in the device status word (qt2_device_status); what its outputs then
 *     hold is unspecified.  The rotating quantizers (MS-EDEN, SR) report the same when the
 *     rotation overflows binary32 (a block sum of 128 inputs beyond 3.4e38, i.e. |x| above
 *     about 2^121).  The method is defined on real numbers only.
 *   - One NVTX range per call, named after the call, marks it for profilers.
 *
 * NVFP4 view layout (one quantized operand of a "TN" GEMM, grouped along its contraction axis):
 *   R = rows (non-contraction axis), C = columns (contraction axis), both multiples of 128.
 *   codes        [R][C/2] bytes, row-major; element 2j in the low nibble of byte j, element 2j+1
 *                in the high nibble.  Nibble = E2M1: bit 3 sign, bits 2..0 index into
 *                {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   scales       one unsigned E4M3 byte per 16-element group, R*C/16 bytes, in the tensor-core
 *                scale-factor order: the scale of row r, group j (0 <= j < C/16) is at byte
 *                  ((r/128)*(C/64) + j/4)*512 + (r%32)*16 + ((r%128)/32)*4 + (j%4).
 *   tensor_scale one fp32 g.  The value of element (r, c) is  val(code) * E4M3(scale) * g.
 */
#ifndef QT2_H
#define QT2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QT2_API __attribute__((visibility("default")))
#else
#define QT2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qt2_stream_t; /* the same type as cudaStream_t */

typedef enum {
    QT2_OK = 0,
    QT2_ERR_INVALID_ARG = -1, /* null pointer, bad enum, unsupported layout request */
    QT2_ERR_SHAPE = -2,       /* a dimension not a positive multiple of 128, or ld < cols */
    QT2_ERR_ALIGN = -3,       /* a pointer not 16-byte aligned, or ld not a multiple of 8 */
    QT2_ERR_WORKSPACE = -4,   /* workspace null or smaller than the size query returned */
    QT2_ERR_CUDA = -5,        /* a CUDA runtime/driver call or launch failed */
    QT2_ERR_TIMEOUT = -6,     /* a device-side bounded wait gave up (see qt2_device_status) */
    QT2_ERR_DEVICE = -7,      /* no device, or the current device is not sm_100 */
    QT2_ERR_NONFINITE = -8,   /* device-side: an input held inf or NaN (see qt2_device_status) */
    QT2_ERR_BOUNDS = -9       /* device-side, checked build only: a store index left its output
                                 array; the store was skipped (see qt2_build_checked) */
} qt2_status;

enum { QT2_LAYOUT_ROW = 1, QT2_LAYOUT_COL = 2, QT2_LAYOUT_BOTH = 3 };
enum { QT2_DTYPE_BF16 = 0, QT2_DTYPE_F32 = 1 };

/* Tensor ids of the Philox streams used by qt2_linear_bwd (id 0 draws the rotation signs). */
enum { QT2_TID_SIGNS = 0, QT2_TID_DY_ROW = 1, QT2_TID_DY_COL = 2, QT2_TID_W_COL = 3, QT2_TID_X_COL = 4 };

typedef struct {
    void *codes;         /* device, R*C/2 bytes */
    void *scales;        /* device, R*C/16 bytes, scale-factor order above */
    float *tensor_scale; /* device, 1 float */
} qt2_nvfp4_view;

QT2_API int qt2_version(void);
QT2_API const char *qt2_status_string(qt2_status s);

/* Reads and clears the library's device-side status word after synchronizing `stream`.
 * *code = 0 when no kernel reported a problem; QT2_ERR_TIMEOUT when a bounded wait gave up;
 * QT2_ERR_NONFINITE when a quantizer met inf or NaN in its input; QT2_ERR_BOUNDS (checked build
 * only) when a kernel skipped a store that would have left its output array (the first report
 * wins).
 * Synchronizes the stream; meant for tests and debugging, not the hot path. */
QT2_API qt2_status qt2_device_status(qt2_stream_t stream, int *code);

/* Host-side fault injection, for testing callers' error handling without a GPU fault.
 * While a hook is set, every CUDA call the library makes while enqueuing work is first
 * announced as hook(site, user), site one of "device" (the device query), "tensor_map" (a TMA
 * descriptor), "memset", "launch" and "symbol" (the scratch lookup of qt2_quant_msedEN_noalloc).  The hook returns 0 to let the call happen, 1 to make it
 * fail without being made (the entry point then returns QT2_ERR_DEVICE for "device" and
 * QT2_ERR_CUDA otherwise, having enqueued nothing further), or 2 to skip it and report success
 * (so a test can walk past the device query on a machine without a GPU).  NULL removes the
 * hook.  Meant for tests: set it while no other thread is calling into the library. */
typedef int (*qt2_fault_hook)(const char *site, void *user);
QT2_API void qt2_set_fault_hook(qt2_fault_hook hook, void *user);

/* ---------------------------------------------------------------------------------------
 * Forward quantizer: round-to-nearest onto E2M1 in 1x16 groups with the "4/6" grid choice.
 * [QII-tg] "Method": per group the full grid (+-6) or the truncated grid (+-4) is used,
 * whichever gives the smaller quantization error; 1x16 groups rather than 16x16 blocks.
 * [QII-th] "fairness" answer: the forward pass uses RTN.  [FAF]: the fp32 tensor scale depends
 * on the tensor-wide max, a sync point before packing.
 *
 * x_bf16 [rows][cols] (leading dimension ld) is grouped along cols.  Computes A = max|x|,
 * g = A/1792 (g = 1 and an all-zero result when A < 2^-100), then per group, for k = 6 then 4:
 * s_k = RNE_E4M3(a/(g*k)), d = s_k*g, codes = RNE_E2M1(x * (1/d)), err_k = sum (x - val*d)^2;
 * keeps k = 4 iff err_4 < err_6.  Results are bit-identical to the reference algorithm.
 * layout_mask must be QT2_LAYOUT_ROW (the forward GEMM consumes row views only); row_out
 * receives the view (R = rows, C = cols); col_out is ignored and may be NULL.
 * One cooperative launch: its thread blocks merge the tensor max, meet at a grid barrier and
 * then quantize (a tensor that fits in L2 is read from HBM once).  Work kept running by other
 * streams on the same GPU can delay the barrier; after 2 s the call gives up, quantizes nothing
 * and reports QT2_ERR_TIMEOUT through qt2_device_status.
 * Workspace: at least qt2_quant_fwd46_workspace_size() bytes, 16-byte aligned; it holds the
 * tensor max and the barrier's counter and is overwritten.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_fwd46_workspace_size(int64_t rows, int64_t cols, size_t *bytes);
QT2_API qt2_status qt2_quant_fwd46(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                           const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                           size_t ws_bytes, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * CTA-local forward quantizer and GEMM ([FAF] "the speed-up is lost between the matmuls": in
 * the CTA-local NVFP4 variant the scale dependency stays inside one thread block; rows and
 * columns get their own corrections, constant over the summation and applied after it, so no
 * block waits for the tensor-wide maximum; the numeric contract differs from global NVFP4).
 * qt2_quant_fwd46_local: x_bf16 [rows][cols] (ld) -> a view like qt2_quant_fwd46's except
 *   that row_out->tensor_scale points to rows/128 floats: block b of 128 rows is quantized with
 *   g_b = A_b/1792, A_b = max|x| over its rows (g_b = 1 below 2^-100).  One launch, no
 *   workspace, no tensor-wide reduction.
 * qt2_gemm_nvfp4_local: as qt2_gemm_nvfp4 for two such views (a: M/128 scales, b: N/128):
 *   c[m][n] = alpha * ga[m/128] * gb[n/128] * sum_k val(a)*sa * val(b)*sb.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_fwd46_local(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                         const qt2_nvfp4_view *row_out, qt2_stream_t stream);
QT2_API qt2_status qt2_gemm_nvfp4_local(const qt2_nvfp4_view *a, const qt2_nvfp4_view *b, int64_t M, int64_t N,
                                        int64_t K, float alpha, void *c, int c_dtype, int64_t ldc,
                                        qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Square-block forward quantizer: one E4M3 scale per 16x16 block ([QII-tg] "Method": the pages
 * compare 16x16 blocks with the 1x16 groups the method keeps for their lower error; with square
 * blocks a weight and its transpose are the same quantization, so one pass serves both of its
 * GEMM operand views).  x_bf16 [rows][cols] (ld):
 *   row_out: view with R = rows, C = cols (groups along cols; the 16 rows of a block repeat its
 *            scale), e.g. W [N][K] for the forward GEMM;
 *   col_out: view of x^T with R = cols, C = rows: the same quantized values transposed, e.g.
 *            W^T [K][N] for a dgrad GEMM with unrotated operands.
 * Per block: a = max|x| over its 256 elements; for k = 6 and 4 the scale E4M3_RNE(a/(g*k)) and
 * the RTN codes of every element; the block's squared error is the balanced tree over its 256
 * elements in row-major order; keep 4 iff its error is smaller (a tie keeps 6); g = A/1792 as
 * qt2_quant_fwd46.  Bit-identical to the reference algorithm.
 * Workspace: at least qt2_quant_fwd46_sq_workspace_size() bytes, 16-byte aligned.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_fwd46_sq_workspace_size(int64_t rows, int64_t cols, size_t *bytes);
QT2_API qt2_status qt2_quant_fwd46_sq(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                      const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                                      size_t ws_bytes, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Backward quantizer MS-EDEN (MicroScaling EDEN).  [QII-tg] "Method": a random Hadamard rotation
 * and a factor <x,x>/<Q(Rx),Rx> (EDEN), plus stochastic rounding of the FP8 scales;
 * [QII-th] "Question 1": fixed 128-element rotation groups, one shared rotation and seed, and
 * no SR for very small scales.  [FAF]: one producer emits both layouts the backward GEMMs need.
 *
 * x_bf16 [rows][cols] (leading dimension ld).  A view groups along the contraction axis:
 *   QT2_LAYOUT_ROW: groups along cols -> row_out view with R = rows, C = cols
 *   QT2_LAYOUT_COL: groups along rows -> col_out view of x^T with R = cols, C = rows
 *   QT2_LAYOUT_BOTH: both views from one read of x.
 * Per 128-block of the grouped axis: y = H D x (D = the 128 signs of Philox(seed, tensor id 0),
 * bit i of word i/32 set -> -1; H = unnormalised Sylvester Hadamard, butterfly strides 1..64);
 * per group p = max|y|/6, codes = RNE_E2M1(y * (1/p)); per block S = sum y^2 / sum p*<val, y>;
 * view tensor scale g = max|y|/1536; group scale = SR_E4M3(S*p/g) with the draw of canonical
 * group index r*(C/16)+j from Philox(seed, tensor_id of the view), RNE below 2^-6.
 * The rotated views multiply with alpha = 2^-7 (qt2_gemm_nvfp4).  Bit-identical to the
 * reference algorithm for the same seed and tensor ids.
 * Workspace: at least qt2_quant_msedEN_workspace_size() bytes, 256-byte aligned (pre-scales
 * S*p in fp32 and the view maxima); overwritten.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_msedEN_workspace_size(int64_t rows, int64_t cols, int layout_mask, size_t *bytes);
QT2_API qt2_status qt2_quant_msedEN(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                            uint64_t seed, uint32_t tensor_id_row, uint32_t tensor_id_col,
                            const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                            size_t ws_bytes, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Backward quantizer with elementwise stochastic rounding: the baseline the Quartet II pages
 * compare MS-EDEN against ([QII-th] abstract and the "fairness of the comparison" answer: the
 * GPU-feasible TetraJet-v2 core, RHT along the inner dimension with stochastic rounding;
 * [QII-tg] "Method": SR rounds to one of the two neighbouring grid points with probability set
 * by the distance).  Same arguments, views and rotation as qt2_quant_msedEN; per view:
 *   g = A/2688 (A = max|y| over the rotated view; A < 2^-100 gives a zero view with g = 1);
 *   group scale = the smallest E4M3 value >= a/RN(6g) (a = max|y| of the group), so no element
 *   leaves the grid and the estimate stays unbiased (the pages give no scale rule for the
 *   baseline; this is the library's reading); d = RN(scale*g), r = RN(1/d);
 *   element code = sign(y) | the E2M1 neighbour of min(|y|*r, 6) picked by stochastic
 *   rounding with U = (u>>8)/2^24, u = word e of Philox(seed, tensor_id of the view), e = the
 *   element's canonical index r*C + c in the view; a group with a < 2^-100 gets scale 0.
 * Two passes over x (the max of the rotated view, then the quantization): the codes depend on
 * the tensor scale.  Bit-identical to the reference algorithm for the same seed and ids.
 * Workspace: at least qt2_quant_sr_workspace_size() bytes, 256-byte aligned (the view maxima).
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_sr_workspace_size(int64_t rows, int64_t cols, int layout_mask, size_t *bytes);
QT2_API qt2_status qt2_quant_sr(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, int layout_mask,
                                uint64_t seed, uint32_t tensor_id_row, uint32_t tensor_id_col,
                                const qt2_nvfp4_view *row_out, const qt2_nvfp4_view *col_out, void *workspace,
                                size_t ws_bytes, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * MS-EDEN without a workspace.  The Quartet II pages have no counterpart to this call; it is a
 * convenience of this library for callers that cannot allocate device memory for scratch (a
 * runtime that has handed all device memory to its own pools, a latency-critical path that
 * must not call cudaMalloc, a plugin whose host framework owns the allocator).
 *
 * Same arguments and results as qt2_quant_msedEN (bit-identical outputs), minus the
 * workspace: the scratch lives in a fixed device array inside the library -- a 256-byte slot
 * for the two view maxima plus QT2_NOALLOC_SCRATCH_BYTES (32 MiB) for the fp32 pre-scales --
 * which every GPU that loads the library holds until the process exits.  The pre-scales take
 * rows*cols/4 bytes per requested view, so the call accepts up to 64 Mi elements with
 * QT2_LAYOUT_BOTH (for example 8192 x 8192) and up to 128 Mi elements with one view (for
 * example 8192 x 16384); larger tensors return QT2_ERR_WORKSPACE and enqueue nothing.
 * Every call looks up the array's device address (cudaGetSymbolAddress) with the calling
 * device current, so the address stays right after a device reset.  The first call on a device
 * may load the library's device code there; make it before any stream capture.
 * All calls on a device share the one array: the call zeroes the view maxima it needs and
 * rewrites every pre-scale before reading it, but two calls whose work overlaps on the GPU
 * (different streams without ordering between them) race on the array and give wrong results.
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine is called.
 * --------------------------------------------------------------------------------------- */
#define QT2_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
QT2_API qt2_status qt2_quant_msedEN_noalloc(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                            int layout_mask, uint64_t seed, uint32_t tensor_id_row,
                                            uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                                            const qt2_nvfp4_view *col_out, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Block-scaled NVFP4 GEMM on the 5th-generation tensor cores ([QII-th] abstract and §1: NVFP4 is
 * natively supported by Blackwell GPUs).  "TN": a is an [M][K] view, b an [N][K] view, both
 * grouped along K.  c[m][n] = alpha * gA * gB * sum_k val(a)*sa * val(b)*sb, accumulated in fp32,
 * written as bf16 or fp32 (c_dtype) with leading dimension ldc >= N (a multiple of 8).
 * alpha = 1 for forward operands, 2^-7 for two MS-EDEN operands sharing a rotation.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_gemm_nvfp4(const qt2_nvfp4_view *a, const qt2_nvfp4_view *b, int64_t M, int64_t N, int64_t K,
                          float alpha, void *c, int c_dtype, int64_t ldc, qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Quartet II linear layer ([QII-ru] "Unbiased quantization ...": a computation graph with every
 * linear-layer GEMM in NVFP4; [QII-th] abstract: better estimates in all major matmuls).
 * x [M][K], w [N][K] (PyTorch Linear layout), dy [M][N]; all bf16, contiguous.
 * Forward:  y = X W^T with both operands through the forward quantizer; y bf16 [M][N].
 * Backward: dX = dY W  (dY row view, W column view, rotated along N),
 *           dW = dY^T X (dY column view, X column view, rotated along M),
 *           tensor ids QT2_TID_*; dx bf16 [M][K]; dw [N][K] bf16 or fp32 (dw_dtype).
 * Workspace: the size queries below; 256-byte aligned; holds the quantized views.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_linear_fwd_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes);
QT2_API qt2_status qt2_linear_fwd(const void *x, const void *w, int64_t M, int64_t K, int64_t N, void *y_bf16,
                          void *workspace, size_t ws_bytes, qt2_stream_t stream);
QT2_API qt2_status qt2_linear_bwd_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes);
QT2_API qt2_status qt2_linear_bwd(const void *dy, const void *x, const void *w, int64_t M, int64_t K, int64_t N,
                          uint64_t seed, void *dx_bf16, void *dw, int dw_dtype, void *workspace, size_t ws_bytes,
                          qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Both views of a layer input from one read ([FAF] "the speed-up is lost between the
 * matmuls": a producer that emits every layout the GEMMs need from one read of the tensor;
 * the pages stress fusing the quantizers around the GEMMs).  x_bf16 [rows][cols] (ld):
 *   row_out: the forward view (R = rows, C = cols), exactly what qt2_quant_fwd46 gives;
 *   col_out: the MS-EDEN column view of x^T (R = cols, C = rows), exactly what
 *            qt2_quant_msedEN gives with QT2_LAYOUT_COL, the same seed and tensor_id_col.
 * A max pass over x comes first (the forward codes depend on the tensor scale), then one pass
 * reads x once for both views.  For a layer, call it on X with the seed and QT2_TID_X_COL that
 * the backward will use, and pass col_out to qt2_linear_bwd_views.
 * Workspace: at least qt2_quant_fwd46_msedEN_col_workspace_size() bytes, 256-byte aligned.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_quant_fwd46_msedEN_col_workspace_size(int64_t rows, int64_t cols, size_t *bytes);
QT2_API qt2_status qt2_quant_fwd46_msedEN_col(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                              uint64_t seed, uint32_t tensor_id_col, const qt2_nvfp4_view *row_out,
                                              const qt2_nvfp4_view *col_out, void *workspace, size_t ws_bytes,
                                              qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Backward of the linear layer from column views quantized beforehand: x_col is X's MS-EDEN
 * column view ([K][M] view, e.g. from qt2_quant_fwd46_msedEN_col), w_col is W's MS-EDEN column
 * view ([K][N] view, qt2_quant_msedEN with QT2_LAYOUT_COL), both made with the same `seed` as
 * this call (the rotation is shared) and tensor ids QT2_TID_X_COL / QT2_TID_W_COL to match
 * qt2_linear_bwd.  W's view can be made once and reused by every micro-batch that runs with
 * that seed.  dY gets both views here (QT2_TID_DY_ROW / _COL); then dX = dY W and dW = dY^T X
 * as qt2_linear_bwd, whose results it reproduces bit for bit for the same inputs.
 * Workspace: at least qt2_linear_bwd_views_workspace_size() bytes, 256-byte aligned.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_linear_bwd_views_workspace_size(int64_t M, int64_t K, int64_t N, size_t *bytes);
QT2_API qt2_status qt2_linear_bwd_views(const void *dy, int64_t M, int64_t K, int64_t N, uint64_t seed,
                                        const qt2_nvfp4_view *x_col, const qt2_nvfp4_view *w_col, void *dx_bf16,
                                        void *dw, int dw_dtype, void *workspace, size_t ws_bytes,
                                        qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Self-test of the device error path: enqueues one kernel whose single wait (on a barrier that
 * nothing completes) gives up after the library's wait limit (2 s) and records QT2_ERR_TIMEOUT
 * in the device status word, exactly as a real wait would; qt2_device_status then returns it
 * (and clears it).  Nothing else is touched; the context stays usable.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_selftest_wait_timeout(qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Self-test of the quantizers' division shortcuts (the method's group scales need RN(a/6) and
 * RN(1/p) in binary32; the kernels form them with fused multiply-adds): for every binary32
 * value whose biased exponent lies in [exp_lo, exp_hi] (1 <= exp_lo <= exp_hi <= 254, every
 * significand), compares the kernels' reciprocal with the IEEE reciprocal and their division by
 * 6 with the IEEE quotient, and adds the numbers of mismatching results to mismatches[0]
 * (reciprocal) and mismatches[1] (division by 6): two device counters, 8-byte aligned, zeroed
 * by the caller.  The kernels use the reciprocal on group scales p in [2^-103, 2^126) (biased
 * exponents 24..252) and the division on group maxima in [2^-100, 2^128) (27..254).
 * Enqueued on `stream`.
 * --------------------------------------------------------------------------------------- */
QT2_API qt2_status qt2_selftest_division(uint32_t exp_lo, uint32_t exp_hi, unsigned long long *mismatches,
                                         qt2_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Checked build.  The same sources compiled with QT2_CHECKED give libqt2_checked.so (built beside
 * libqt2.so, the same entry points): every global store of every kernel first checks that the
 * bytes it writes lie inside the output array the call was given (the view's codes, scales or
 * pre-scales, the GEMM's C rows) and, if not, skips the store and records QT2_ERR_BOUNDS in the
 * device status word.  It runs slower and is meant for testing and debugging, not the hot path.
 * qt2_build_checked returns 1 in the checked build, 0 in the product build.
 * qt2_selftest_bounds enqueues one kernel that stores one byte through that check into a
 * 64-byte array of the library's own, at offset 40 against a stated extent of 32 bytes: the
 * checked build skips the store and records QT2_ERR_BOUNDS (read it with qt2_device_status);
 * the product build, which has no checks, makes the store (still inside the array) and records
 * nothing.  Enqueued on `stream`.
 * --------------------------------------------------------------------------------------- */
QT2_API int qt2_build_checked(void);
QT2_API qt2_status qt2_selftest_bounds(qt2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QT2_H */
