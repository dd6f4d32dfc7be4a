/*
 * wqmm.h -- C ABI of libwqmm, a B200 (sm_100a) implementation of the compute
 * part of two weight-quantised matmul operators:
 *
 *   wqmm_*  anti-quant ("pseudo-quant") weight GEMM, after
 *           aclnnWeightQuantMatmulAllReduce ("计算公式"):
 *             output = x1 @ ((x2 + antiquantOffset) * antiquantScale) + bias + x3
 *   qmm_*   int8 x int8 GEMM, after aclnnQuantMatmulAllReduceV2 ("Function",
 *           cases 1 and 2):
 *             output = dequantScale * pertokenScale * (x1_int8 @ x2_int8 + bias_int32) + x3
 *
 * The AllReduce of both operators is the identity for one rank and is not
 * performed by these entry points; across ranks (row-parallel, x1 and x2
 * split along k) the Python package runs the GEMM per rank and sums the
 * outputs with an NCCL all-reduce (weight_quantized_gemm_anti_b200.allreduce).  Every call follows the two-phase convention of those pages
 * ("两段式接口与函数原型"; "Function Prototype"): phase 1 validates the
 * arguments, plans the launch and reports the device workspace it needs; the
 * caller allocates that workspace (only when the size is > 0) and calls phase
 * 2 once on a CUDA stream.  Argument order follows the pages.
 *
 * Conventions for every entry point
 *  - Tensors are described by wqmm_tensor: a DEVICE pointer plus shape and
 *    strides in ELEMENTS (for int4, in logical 4-bit elements).  The caller
 *    owns all device memory (inputs, output, workspace); the library never
 *    allocates device memory and never frees caller memory.
 *  - Optional tensors are passed as NULL descriptors.
 *  - Return value: WQMM_SUCCESS (0) or an error code; on error a message is
 *    available from wqmm_last_error() in the calling thread.  Phase 1 errors
 *    launch nothing.  Phase 2 launches asynchronously on `stream`; a CUDA
 *    launch failure is reported as WQMM_ERR_CUDA (+ message).
 *  - Check order in phase 1 is null -> dtype -> attributes -> shape, as in
 *    "返回值与错误码" of the anti-quant page (CheckNotNull, CheckDtypeValid,
 *    CheckAttr, CheckShape).
 *  - Executors are one-shot: phase 2 consumes and frees the executor whether it
 *    succeeds or not ("第二段接口不可重复调用").  An executor that is never run
 *    must be released with wqmm_executor_destroy.
 *  - Entry points are thread-safe with respect to each other; an executor must
 *    not be shared between threads.
 */
#ifndef WQMM_H_
#define WQMM_H_

#include <stdint.h>

#if defined(__GNUC__)
#define WQMM_API __attribute__((visibility("default")))
#else
#define WQMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
/* Codes 161001/161002/561002 keep the values of the aclnn return codes the
 * pages cite (ACLNN_ERR_PARAM_NULLPTR, ACLNN_ERR_PARAM_INVALID,
 * ACLNN_ERR_INNER_TILING_ERROR); 500000+ are this library's own. */
typedef int32_t wqmm_status;
#define WQMM_SUCCESS 0
#define WQMM_ERR_PARAM_NULLPTR 161001 /* a required pointer is NULL */
#define WQMM_ERR_PARAM_INVALID 161002 /* dtype, attribute, shape or layout not supported */
#define WQMM_ERR_INNER_TILING 561002  /* no kernel plan for an accepted problem */
#define WQMM_ERR_CUDA 500001          /* a CUDA runtime / driver call failed */
#define WQMM_ERR_WORKSPACE 500002     /* workspace NULL or smaller than phase 1 reported */
#define WQMM_ERR_EXECUTOR 500003      /* executor NULL, already consumed, or of the other operator */
#define WQMM_ERR_TIMEOUT 500004       /* wqmm_stream_wait deadline passed */

/* ------------------------------------------------------------------ dtypes */
#define WQMM_DT_F16 1
#define WQMM_DT_BF16 2
#define WQMM_DT_F32 3
#define WQMM_DT_I8 4
#define WQMM_DT_I4 5 /* two per byte, two's complement, low nibble = even index of the contiguous axis */
#define WQMM_DT_I32 6
#define WQMM_DT_FP8E4M3 7 /* OCP FP8 E4M3FN */
#define WQMM_DT_I64 8
#define WQMM_DT_U64 9

/* ------------------------------------------------------------------ formats */
#define WQMM_FORMAT_ND 0     /* plain strided tensor */
#define WQMM_FORMAT_PACKED 1 /* a weight produced by wqmm_pack_weight (shape/strides describe the (k, n) logical matrix) */

typedef struct wqmm_tensor {
    void* data;          /* device address (host memory is never accepted) */
    int32_t dtype;       /* WQMM_DT_* */
    int32_t ndim;        /* 1..3 */
    int64_t shape[3];    /* logical shape */
    int64_t strides[3];  /* in elements (logical 4-bit elements for int4) */
    int32_t format;      /* WQMM_FORMAT_* */
    int32_t reserved;    /* must be 0 */
} wqmm_tensor;

typedef struct wqmm_executor wqmm_executor;
typedef struct CUstream_st* wqmm_stream; /* a cudaStream_t; NULL = the legacy default stream */

/* ================================================================ anti-quant GEMM
 *
 * wqmm_get_workspace_size -- phase 1 (aclnnWeightQuantMatmulAllReduceGetWorkspaceSize).
 *
 *  x1                (m, k) or (b, s, k), f16 or bf16, row-major contiguous (not transposed).
 *  x2                (k, n) weight: int8, int4 or fp8-e4m3; ND row-major, ND "transposed"
 *                    (strides (1, k): the last two axes swapped, stored (n, k)), or
 *                    WQMM_FORMAT_PACKED from wqmm_pack_weight.  An x2 of the x1 dtype
 *                    (f16 / bf16) selects the non-quantised scenario of the same
 *                    operator family ("非量化场景" of npu_mm_all_reduce_base, "x2":
 *                    its dtype then equals x1's): output = x1 @ x2 + bias + x3, with
 *                    antiquant_scale and antiquant_offset NULL and G = 0.
 *  bias              optional, (n), dtype of x1.
 *  antiquant_scale   required for int8 / int4 / fp8 weights (a NULL scale there is
 *                    WQMM_ERR_PARAM_NULLPTR), NULL for f16 / bf16 weights (a scale there is
 *                    WQMM_ERR_PARAM_INVALID); dtype of x1: per-tensor (1); per-channel (n) or (1, n);
 *                    per-group (ceil(k / G), n) -- contiguous, or transposed (strides
 *                    (1, ceil(k/G))) exactly when x2 is transposed ("约束说明").
 *  antiquant_offset  optional, same shape, dtype and strides as the scale; ADDED to the
 *                    weight before the scale multiplies it.  Must be NULL for fp8 weights,
 *                    which also only support per-channel.
 *  x3                optional, output shape, dtype of x1, contiguous.
 *  group             communication domain name; unused for one rank, may be NULL.
 *  reduce_op         must be "sum".
 *  comm_turn         must be 0.            stream_mode  must be 1.
 *  antiquant_group_size  G: 0 = not per-group; otherwise G % 32 == 0 and
 *                    32 <= G <= min(k - 1, INT32_MAX) (the G check is skipped when k == 0).
 *  output            (m, n) or (b, s, n), dtype of x1, contiguous.
 *  workspace_size    out: bytes of device workspace phase 2 needs (0 = none).
 *  executor          out: the one-shot plan.
 *
 * Shape rules ("形状与范围约束"): 1 <= m <= 2^31-1, 0 <= k <= 65535, 1 <= n <= 65535;
 * m == 0 or n == 0 is rejected; k == 0 is accepted and yields bias + x3 (or zeros).
 * Alignment (the int8/int4 rule of the "产品相关的格式与对齐约束" section, adopted
 * for this device): int8 / fp8 / f16 / bf16 weights need k % 32 == 0 and n % 32 == 0,
 * int4 weights k % 64 == 0 and n % 64 == 0.  All data pointers must be 16-byte aligned.
 */
WQMM_API wqmm_status wqmm_get_workspace_size(const wqmm_tensor* x1, const wqmm_tensor* x2, const wqmm_tensor* bias,
                                    const wqmm_tensor* antiquant_scale, const wqmm_tensor* antiquant_offset,
                                    const wqmm_tensor* x3, const char* group, const char* reduce_op,
                                    int64_t comm_turn, int64_t stream_mode, int64_t antiquant_group_size,
                                    const wqmm_tensor* output, uint64_t* workspace_size,
                                    wqmm_executor** executor);

/* wqmm_run -- phase 2 (aclnnWeightQuantMatmulAllReduce): enqueue the GEMM on
 * `stream`.  `workspace` must hold at least the size phase 1 reported (it may
 * be NULL when that size is 0).  Consumes the executor. */
WQMM_API wqmm_status wqmm_run(void* workspace, uint64_t workspace_size, wqmm_executor* executor, wqmm_stream stream);

/* ================================================================ int8 GEMM
 *
 * qmm_get_workspace_size -- phase 1 (aclnnQuantMatmulAllReduceV2GetWorkspaceSize).
 *
 *  x1               (m, k) or (b, s, k) int8, contiguous.
 *  x2               (k, n) int8: ND, ND transposed (strides (1, k)), or PACKED.
 *  bias             optional (n) int32.
 *  x3               optional, output shape and dtype, contiguous.
 *  dequant_scale    required: per-tensor (1) or per-channel (n) / (1, n).  bf16 when the
 *                   output is bf16; fp32 when the output is fp16.  (The pages require an
 *                   INT64/UINT64 TransQuantParamV2 encoding for fp16 output without
 *                   pertoken; that encoding is not published, so INT64/UINT64 are rejected
 *                   and fp32 is accepted in its place.)
 *  pertoken_scale   optional fp32 (m) -- (b*s) for 3-D x1.
 *  group, reduce_op, comm_turn, stream_mode  as for wqmm.
 *  output           (m, n) / (b, s, n), fp16 or bf16, contiguous.
 *
 * No empty tensors ("Empty tensor support"): m, k, n >= 1.  k, n <= 65535,
 * m <= 2^31-1; k % 32 == 0 and n % 32 == 0 (int8 alignment rule).
 */
WQMM_API wqmm_status qmm_get_workspace_size(const wqmm_tensor* x1, const wqmm_tensor* x2, const wqmm_tensor* bias,
                                   const wqmm_tensor* x3, const wqmm_tensor* dequant_scale,
                                   const wqmm_tensor* pertoken_scale, const char* group,
                                   const char* reduce_op, int64_t comm_turn, int64_t stream_mode,
                                   const wqmm_tensor* output, uint64_t* workspace_size,
                                   wqmm_executor** executor);

/* qmm_run -- phase 2 (aclnnQuantMatmulAllReduceV2).  Consumes the executor. */
WQMM_API wqmm_status qmm_run(void* workspace, uint64_t workspace_size, wqmm_executor* executor, wqmm_stream stream);

/* ================================================================ weight preparation
 *
 * The B200 counterpart of aclnnCalculateMatmulWeightSizeV2 + aclnnTransMatmulWeight
 * (the weight-format conversion in the QuantMatmulAllReduceV2 sample): re-lays a
 * (k, n) weight (ND or ND-transposed; int8, int4 or fp8-e4m3, or f16 / bf16 for
 * the non-quantised scenario) into the K-major
 * tiles the GEMM kernels stream (128 n-rows x 64 k per tile for wqmm, 256 x 128
 * for qmm).  The packed weight is then passed with format WQMM_FORMAT_PACKED and
 * the same logical shape (k, n); packing is done once, outside the timed path.
 *
 * wqmm_pack_weight_size: bytes of the packed buffer for x2 (a host-only query).
 *   `for_int8_gemm` selects the qmm tiling (1) or the wqmm tiling (0).
 * wqmm_pack_weight: enqueue the packing kernel on `stream`; `packed` is a device
 *   buffer of at least that size (16-byte aligned).  x2 is read, not modified.
 */
WQMM_API wqmm_status wqmm_pack_weight_size(const wqmm_tensor* x2, int32_t for_int8_gemm, uint64_t* packed_bytes);
WQMM_API wqmm_status wqmm_pack_weight(const wqmm_tensor* x2, int32_t for_int8_gemm, void* packed, wqmm_stream stream);

/* ================================================================ no-allocation variant
 *
 * wqmm_matmul_no_alloc -- both phases of the anti-quant GEMM in one call, for
 * callers that cannot allocate device memory (a region being captured into a
 * CUDA graph, a component with a fixed memory budget, a foreign ABI that passes
 * tensors but no allocator).  The operator pages have no counterpart: it exists
 * for this library's callers only.  Arguments are those of
 * wqmm_get_workspace_size minus the workspace outputs, plus the stream.
 *
 * The workspace is a fixed 16 MiB array in device memory owned by the library
 * (every GPU that loads the library keeps it until the process exits).
 * Problems that need more are rejected with WQMM_ERR_WORKSPACE before any
 * launch; pre-packing the weight keeps the need small.  No device memory is
 * allocated or freed.  All calls on a device share the array: calls that
 * overlap on the GPU race, so serialise them.  The first call on a device
 * looks up the array's address (with that device current); make it before any
 * stream capture begins.
 */
WQMM_API wqmm_status wqmm_matmul_no_alloc(const wqmm_tensor* x1, const wqmm_tensor* x2, const wqmm_tensor* bias,
                                          const wqmm_tensor* antiquant_scale, const wqmm_tensor* antiquant_offset,
                                          const wqmm_tensor* x3, const char* group, const char* reduce_op,
                                          int64_t comm_turn, int64_t stream_mode, int64_t antiquant_group_size,
                                          const wqmm_tensor* output, wqmm_stream stream);

/* ================================================================ utilities */

/* Release an executor that was never passed to a *_run call (NULL is ignored). */
WQMM_API void wqmm_executor_destroy(wqmm_executor* executor);

/* Message for the last non-zero status returned in the calling thread ("" if none). */
WQMM_API const char* wqmm_last_error(void);

/* Host wait with a deadline, the analogue of aclrtSynchronizeStreamWithTimeout in
 * the pages' samples: polls the stream until it is idle or `timeout_ms` passes
 * (WQMM_ERR_TIMEOUT; the work keeps running).  Returns WQMM_ERR_CUDA if the
 * stream reported an error. */
WQMM_API wqmm_status wqmm_stream_wait(wqmm_stream stream, int32_t timeout_ms);

/* Read the library's device error word: 0, or the code of the first bounded
 * in-kernel wait that gave up (the kernel then ended early and its output is
 * invalid).  Synchronous with respect to the device; `reset` != 0 clears it.
 * Codes: 1 a copy producer, 2 the MMA issuer, 3 a dequantiser, 4 the epilogue
 * (including the wait of a split tile's first owner for the other owners'
 * partials), 5 the final drain of outstanding copies.
 * After a timeout, owners that finished late may have left "partial written"
 * flags set in the workspace.  A new wqmm_run call never matches them (each
 * launch waits for a token of its own), but a CUDA graph replays a captured
 * launch with its captured token: zero the graph's workspace before replaying
 * it once a timeout has been reported. */
WQMM_API wqmm_status wqmm_device_error(uint32_t* code, int32_t reset);

/* Library version string, e.g. "wqmm 0.1 sm_100a". */
WQMM_API const char* wqmm_version(void);

/* Test-only: make qmm_run also write the raw int32 accumulator
 * (x1 @ x2 + bias, wrapped to 32 bits) into `acc_i32_out`, a device buffer of
 * m * n int32 (row-major).  Call between phase 1 and phase 2. */
WQMM_API wqmm_status qmm_debug_set_raw_accumulator(wqmm_executor* executor, void* acc_i32_out);

/* Test-only: make the bounded device wait of a split tile's first owner (the
 * wait for the other owners' fp32 partials of a stream-K plan) give up after
 * `wait_ns` nanoseconds instead of 2 s (0 keeps 2 s), and, when `mismatch` is
 * non-zero, wait for a flag value that no owner of the launch writes -- so the
 * wait runs out, the kernel records error code 4 in the device error word
 * (wqmm_device_error), ends early and leaves its output invalid.  No GPU fault
 * is involved.  Call between phase 1 and phase 2 of wqmm; it has no effect on
 * a plan without split tiles. */
WQMM_API wqmm_status wqmm_debug_set_flag_wait(wqmm_executor* executor, uint64_t wait_ns, int32_t mismatch);

#ifdef __cplusplus
}
#endif

#endif /* WQMM_H_ */
