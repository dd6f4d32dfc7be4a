// noalloc.cu -- the anti-quant GEMM for callers that cannot allocate device memory.
//
// wqmm_run needs a device workspace for three things: the fp32 partial tiles of
// its small-m (stream-K) schedule, a re-laid copy of an unpacked weight, and a
// transposed copy of a transposed per-group scale/offset.  Some callers have no
// way to provide one: code that runs where a device allocation is not allowed
// or not possible -- inside a region being recorded into a CUDA graph, in a
// real-time or driver-like component with a fixed memory budget, or behind a
// foreign ABI that hands over tensors but no allocator.  This file gives them
// wqmm_matmul_no_alloc: both phases in one call, with the workspace taken from
// a fixed array in device memory that the library reserves for itself.
//
// Properties a caller must know:
//  * the array holds kScratchBytes (16 MiB) and every GPU that loads the library
//    keeps it until the process exits; problems whose workspace is larger are
//    rejected with WQMM_ERR_WORKSPACE before anything is launched;
//  * all calls on a device share the one array, so calls whose work overlaps on
//    the GPU (different streams, or other threads) race on it -- serialise them;
//  * the array keeps whatever the previous call left in it.  Stale fp32
//    partial tiles are never read: a tile's partials are read only after the
//    owners of this launch have written them and raised their flags.  Stale
//    "partial written" flags cannot match either: every launch waits for its
//    own 64-bit token, which no earlier launch wrote, and the CTA that consumes
//    a tile's flags clears them;
//  * the first call on a device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture begins.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/wqmm.h"
#include "internal.h"

namespace {

constexpr uint64_t kScratchBytes = 16ull << 20;
constexpr int kMaxDevices = 64;

// The fixed workspace.  In host code this name is only a handle for the symbol
// lookup below, never a device address; kernels get the looked-up pointer.
static __device__ __align__(256) unsigned char g_wqmm_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
wqmm_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return wqmm::report_error(WQMM_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return wqmm::report_error(WQMM_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_wqmm_scratch);
    if (e != cudaSuccess || p == nullptr)
      return wqmm::report_error(WQMM_ERR_CUDA, "cudaGetSymbolAddress of the fixed workspace failed");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return WQMM_SUCCESS;
}

}  // namespace

extern "C" wqmm_status wqmm_matmul_no_alloc(const wqmm_tensor* x1, const wqmm_tensor* x2, const wqmm_tensor* bias,
                                            const wqmm_tensor* antiquant_scale,
                                            const wqmm_tensor* antiquant_offset, const wqmm_tensor* x3,
                                            const char* group, const char* reduce_op, int64_t comm_turn,
                                            int64_t stream_mode, int64_t antiquant_group_size,
                                            const wqmm_tensor* output, wqmm_stream stream) {
  uint64_t need = 0;
  wqmm_executor* ex = nullptr;
  wqmm::g_plan_ws_cap = kScratchBytes;  // plan within the fixed array where a plan can
  wqmm_status st = wqmm_get_workspace_size(x1, x2, bias, antiquant_scale, antiquant_offset, x3, group, reduce_op,
                                           comm_turn, stream_mode, antiquant_group_size, output, &need, &ex);
  wqmm::g_plan_ws_cap = 0;
  if (st != WQMM_SUCCESS) return st;
  if (need > kScratchBytes) {
    wqmm_executor_destroy(ex);
    return wqmm::report_error(WQMM_ERR_WORKSPACE,
                              "problem needs a larger workspace than the 16 MiB fixed array of "
                              "wqmm_matmul_no_alloc (pre-pack the weight, or call wqmm_run with a workspace)");
  }
  void* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st != WQMM_SUCCESS) {
    wqmm_executor_destroy(ex);
    return st;
  }
  return wqmm_run(scratch, kScratchBytes, ex, stream);
}
