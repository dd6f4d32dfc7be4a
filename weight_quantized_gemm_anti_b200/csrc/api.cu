// api.cu -- the C ABI of libwqmm (include/wqmm.h): argument validation in the
// order the anti-quant page gives (CheckNotNull -> CheckDtypeValid -> CheckAttr
// -> CheckShape, "返回值与错误码"), launch planning, one-shot executors, and
// phase-2 launches on the caller's stream.  Phase 1 is host-only: it makes no
// CUDA call except an optional SM-count query used to size split-K.
#include <atomic>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <new>
#include <string>
#include <thread>
#include <unordered_set>

#include <cuda.h>
#include <cuda_runtime.h>
#include <unistd.h>

#include "../../include/wqmm.h"
#include "internal.h"

using namespace wqmm;

namespace wqmm {
thread_local uint64_t g_plan_ws_cap = 0;
}  // namespace wqmm

namespace {

thread_local std::string g_last_error;

wqmm_status fail(wqmm_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

wqmm_status ok() {
  g_last_error.clear();
  return WQMM_SUCCESS;
}

constexpr uint64_t kFlagWaitNs = 2000000000ull;  // a split tile's flag wait gives up after 2 s
constexpr uint32_t kMagicLive = 0x57514D4Du;  // "WQMM"
constexpr uint32_t kMagicDead = 0xDEADBEEFu;

enum class OpKind { kWqmm, kQmm };

struct Region {
  uint64_t offset = 0, bytes = 0;
};

}  // namespace

struct wqmm_executor {
  uint32_t magic = kMagicLive;
  OpKind op = OpKind::kWqmm;
  // common
  int64_t m = 0;
  int k = 0, n = 0;
  int act_dtype = WQMM_DT_BF16;  // wqmm activations / qmm output
  const void* x1 = nullptr;
  const void* x2 = nullptr;
  int x2_dtype = 0;
  bool x2_packed = false;
  int64_t x2_s0 = 0, x2_s1 = 0;
  void* out = nullptr;
  const void* bias = nullptr;
  const void* x3 = nullptr;
  uint64_t workspace = 0;
  Region ws_pack, ws_scale, ws_offset, ws_partial, ws_flags;
  // wqmm
  const void* scale = nullptr;
  const void* offset = nullptr;
  bool scale_transposed = false;
  int mode = kPerChannel;
  int group_size = 0;
  int num_groups = 0;
  int bn = 256;
  int grid = 1;        // persistent CTAs of the GEMM
  int stream_k = 0;    // 1: stream-K -- the k steps of tiles dp_tiles.. split evenly over the grid, partials + fix-up
  int dp_tiles = 0;    // stream-K: tiles run whole before the split ones (a multiple of the grid)
  int sk_unit = 1;     // stream-K: split granularity in k steps
  int sk_grid = 0;     // stream-K: CTAs sharing the split tiles
  int sk_inline = 0;   // stream-K: the first owner of a split tile reduces it (no fix-up kernel)
  int pair = 0;        // 1: clusters of two CTAs share each MMA (256 weight columns per pair tile)
  int smallm = 0;      // 1: the small-m kernel (m tile 16 or 32, DG MMA-issuing dequantisation groups)
  int num_pnb = 0;     // pair: 256-column blocks
  int num_tiles = 0;
  int max_slots = 0;
  // qmm
  const void* dq = nullptr;
  int dq_dtype = 0;
  bool dq_per_tensor = false;
  const float* pertoken = nullptr;
  int32_t* raw_acc = nullptr;
  // test hook (wqmm_debug_set_flag_wait): bound of a split tile's flag wait,
  // and whether its first owner waits for a value no owner writes
  uint64_t debug_wait_ns = 0;
  bool debug_flag_mismatch = false;
};

namespace {

// Executors handed out and not yet consumed.  Phase 2 and destroy look a
// handle up here first, so a consumed or foreign handle is reported as an
// error instead of being dereferenced.
std::mutex g_live_mu;
std::unordered_set<const wqmm_executor*> g_live;

wqmm_executor* register_executor(wqmm_executor* ex) {
  std::lock_guard<std::mutex> lk(g_live_mu);
  g_live.insert(ex);
  return ex;
}

bool is_live(const wqmm_executor* ex) {
  std::lock_guard<std::mutex> lk(g_live_mu);
  return g_live.count(ex) != 0;
}

// ------------------------------------------------------------------ tensor helpers
int64_t numel(const wqmm_tensor* t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
  return n;
}

bool contiguous(const wqmm_tensor* t) {
  if (numel(t) == 0) return true;  // an empty tensor has no layout to check
  int64_t expect = 1;
  for (int i = t->ndim - 1; i >= 0; --i) {
    if (t->shape[i] != 1 && t->strides[i] != expect) return false;
    expect *= t->shape[i];
  }
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool act_dtype_ok(int dt) { return dt == WQMM_DT_F16 || dt == WQMM_DT_BF16; }

// The anti-quant GEMM's weight kind for an x2 dtype (float16 / bfloat16: the
// non-quantised scenario, x2 of the x1 dtype).
int weight_kind(int x2_dtype) {
  switch (x2_dtype) {
    case WQMM_DT_I4: return kW4;
    case WQMM_DT_I8: return kW8;
    case WQMM_DT_FP8E4M3: return kWFp8;
    default: return kWH;
  }
}

const char* dt_name(int dt) {
  switch (dt) {
    case WQMM_DT_F16: return "float16";
    case WQMM_DT_BF16: return "bfloat16";
    case WQMM_DT_F32: return "float32";
    case WQMM_DT_I8: return "int8";
    case WQMM_DT_I4: return "int4";
    case WQMM_DT_I32: return "int32";
    case WQMM_DT_FP8E4M3: return "float8_e4m3fn";
    case WQMM_DT_I64: return "int64";
    case WQMM_DT_U64: return "uint64";
    default: return "unknown";
  }
}

wqmm_status check_descriptor(const wqmm_tensor* t, const char* name) {
  if (t->ndim < 1 || t->ndim > 3) return fail(WQMM_ERR_PARAM_INVALID, "%s: ndim %d not in [1, 3]", name, t->ndim);
  if (t->reserved != 0) return fail(WQMM_ERR_PARAM_INVALID, "%s: reserved field must be 0", name);
  for (int i = 0; i < t->ndim; ++i)
    if (t->shape[i] < 0) return fail(WQMM_ERR_PARAM_INVALID, "%s: negative extent", name);
  if (t->format != WQMM_FORMAT_ND && t->format != WQMM_FORMAT_PACKED)
    return fail(WQMM_ERR_PARAM_INVALID, "%s: unknown format %d", name, t->format);
  return WQMM_SUCCESS;
}

// A value no earlier launch has written into a stream-K flag: a process-wide
// counter (odd values, step 2) started at a value mixed from the clocks and the
// process id, so that flags left in reused memory (by this or an earlier
// process) do not match.
uint64_t next_launch_token() {
  static std::atomic<uint64_t> counter{[] {
    uint64_t x = static_cast<uint64_t>(std::chrono::steady_clock::now().time_since_epoch().count());
    x ^= static_cast<uint64_t>(std::chrono::system_clock::now().time_since_epoch().count()) << 21;
    x ^= static_cast<uint64_t>(getpid()) << 40;
    x ^= x >> 33;
    x *= 0xff51afd7ed558ccdULL;
    x ^= x >> 33;
    return x | 1ULL;
  }()};
  return counter.fetch_add(2, std::memory_order_relaxed);  // odd, never zero, never repeated
}

int sm_count() {
  static std::once_flag once;
  static int sms = 148;
  std::call_once(once, [] {
    int n = 0, dev = 0;
    if (cudaGetDeviceCount(&n) == cudaSuccess && n > 0 && cudaGetDevice(&dev) == cudaSuccess) {
      int v = 0;
      if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    } else {
      cudaGetLastError();  // clear the sticky "no device" error of a CPU-only host
    }
  });
  return sms;
}

uint64_t round_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

// Resident CTA pairs of the pair-mode int8 GEMM per (device, output type).
int qmm_pair_slots_cached(bool out_bf16) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const auto key = std::make_pair(dev, out_bf16 ? 1 : 0);
  std::lock_guard<std::mutex> lock(mu);
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  const int v = qmm_pair_slots(out_bf16);
  cache[key] = v;
  return v;
}

// Resident CTA pairs of the pair-mode GEMM, per (device, m tile, weight kind,
// activation type); 0 when there is no pair mode or no device.
int pair_slots(int bn, int wk, bool bf16) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const auto key = std::make_tuple(dev, bn, wk, bf16 ? 1 : 0);
  std::lock_guard<std::mutex> lock(mu);
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  const int v = wqmm_pair_slots(bn, wk, bf16);
  cache[key] = v;
  return v;
}

uint64_t packed_bytes_for(int x2_dtype, int64_t k, int64_t n, bool for_qmm) {
  if (for_qmm) {
    const uint64_t nb = (n + kQNBlock - 1) / kQNBlock, kt = (k + kQKTile - 1) / kQKTile;
    return nb * kt * kQTileBytes;
  }
  const int wk = weight_kind(x2_dtype);
  const uint64_t nb = (n + kWqNBlock - 1) / kWqNBlock, kt = (k + kWqKTile - 1) / kWqKTile;
  return nb * kt * wq_tile_bytes(wk);
}

// x2 (k, n): ND (strides (n, 1)), ND transposed (strides (1, k)) or PACKED.
wqmm_status check_x2_layout(const wqmm_tensor* x2, int64_t k, int64_t n, bool* transposed) {
  *transposed = false;
  if (x2->format == WQMM_FORMAT_PACKED) return WQMM_SUCCESS;
  if (x2->strides[0] == n && x2->strides[1] == 1) return WQMM_SUCCESS;
  if (x2->strides[0] == 1 && x2->strides[1] == k) {
    *transposed = true;
    return WQMM_SUCCESS;
  }
  if (k <= 1 || n <= 1) return WQMM_SUCCESS;  // degenerate: every layout is contiguous
  return fail(WQMM_ERR_PARAM_INVALID,
              "x2: only contiguous (strides (n,1)) or last-two-axes-transposed (strides (1,k)) layouts are "
              "supported, got strides (%lld, %lld)",
              (long long)x2->strides[0], (long long)x2->strides[1]);
}

wqmm_status common_attr_checks(const char* reduce_op, int64_t comm_turn, int64_t stream_mode) {
  if (std::strcmp(reduce_op, "sum") != 0)
    return fail(WQMM_ERR_PARAM_INVALID, "reduceOp must be \"sum\", got \"%s\"", reduce_op);
  if (stream_mode != 1) return fail(WQMM_ERR_PARAM_INVALID, "streamMode must be 1, got %lld", (long long)stream_mode);
  if (comm_turn != 0) return fail(WQMM_ERR_PARAM_INVALID, "commTurn must be 0, got %lld", (long long)comm_turn);
  return WQMM_SUCCESS;
}

// x1 (m,k)/(b,s,k) and output (m,n)/(b,s,n) shapes; fills m, k.
wqmm_status check_x1_out(const wqmm_tensor* x1, const wqmm_tensor* out, int64_t n, int64_t* m_out) {
  if (x1->ndim != 2 && x1->ndim != 3)
    return fail(WQMM_ERR_PARAM_INVALID, "x1 must be 2-D (m,k) or 3-D (b,s,k), got %d-D", x1->ndim);
  int64_t m = 1;
  for (int i = 0; i < x1->ndim - 1; ++i) m *= x1->shape[i];
  if (out->ndim != x1->ndim) return fail(WQMM_ERR_PARAM_INVALID, "output must have the rank of x1");
  for (int i = 0; i < x1->ndim - 1; ++i)
    if (out->shape[i] != x1->shape[i]) return fail(WQMM_ERR_PARAM_INVALID, "output leading dims must match x1");
  if (out->shape[out->ndim - 1] != n) return fail(WQMM_ERR_PARAM_INVALID, "output last dim must be n = %lld", (long long)n);
  if (m < 1 || m > 2147483647LL)
    return fail(WQMM_ERR_PARAM_INVALID, "m = %lld out of range [1, 2147483647] (empty m is not supported)",
                (long long)m);
  if (!contiguous(x1)) return fail(WQMM_ERR_PARAM_INVALID, "x1 must be contiguous (non-transposed)");
  if (!contiguous(out)) return fail(WQMM_ERR_PARAM_INVALID, "output must be contiguous");
  *m_out = m;
  return WQMM_SUCCESS;
}

bool same_shape(const wqmm_tensor* a, const wqmm_tensor* b) {
  if (a->ndim != b->ndim) return false;
  for (int i = 0; i < a->ndim; ++i)
    if (a->shape[i] != b->shape[i]) return false;
  return true;
}

}  // namespace

// ===================================================================== wqmm phase 1
extern "C" wqmm_status wqmm_get_workspace_size(const wqmm_tensor* x1, const wqmm_tensor* x2,
                                               const wqmm_tensor* bias, const wqmm_tensor* scale,
                                               const wqmm_tensor* offset, const wqmm_tensor* x3,
                                               const char* group, const char* reduce_op, int64_t comm_turn,
                                               int64_t stream_mode, int64_t group_size,
                                               const wqmm_tensor* output, uint64_t* workspace_size,
                                               wqmm_executor** executor) {
  (void)group;  // communication domain: unused for one rank
  // ---- CheckNotNull (antiquantScale may be null only in the non-quantised
  // scenario, x2 of the x1 dtype)
  if (!x1 || !x2 || !output) return fail(WQMM_ERR_PARAM_NULLPTR, "x1, x2 and output must not be null");
  const bool nonquant = act_dtype_ok(x1->dtype) && x2->dtype == x1->dtype;
  if (!scale && !nonquant)
    return fail(WQMM_ERR_PARAM_NULLPTR, "antiquantScale must not be null for int8, int4 or float8_e4m3fn weights");
  if (!reduce_op) return fail(WQMM_ERR_PARAM_NULLPTR, "reduceOp must not be null");
  if (!workspace_size || !executor) return fail(WQMM_ERR_PARAM_NULLPTR, "workspaceSize and executor must not be null");
  *executor = nullptr;
  *workspace_size = 0;
  const wqmm_tensor* all[] = {x1, x2, bias, scale, offset, x3, output};
  const char* names[] = {"x1", "x2", "bias", "antiquantScale", "antiquantOffset", "x3", "output"};
  for (int i = 0; i < 7; ++i) {
    if (!all[i]) continue;
    wqmm_status st = check_descriptor(all[i], names[i]);
    if (st) return st;
    if (i != 1 && all[i]->format != WQMM_FORMAT_ND)
      return fail(WQMM_ERR_PARAM_INVALID, "%s: only x2 may use the packed format", names[i]);
  }

  // ---- CheckDtypeValid
  const int adt = x1->dtype;
  if (!act_dtype_ok(adt))
    return fail(WQMM_ERR_PARAM_INVALID, "x1 dtype %s not supported (float16, bfloat16)", dt_name(adt));
  if (x2->dtype != WQMM_DT_I8 && x2->dtype != WQMM_DT_I4 && x2->dtype != WQMM_DT_FP8E4M3 && !nonquant)
    return fail(WQMM_ERR_PARAM_INVALID, "x2 dtype %s not supported (int8, int4, float8_e4m3fn, or the x1 dtype)",
                dt_name(x2->dtype));
  if (nonquant && (scale || offset))
    return fail(WQMM_ERR_PARAM_INVALID,
                "x2 of the x1 dtype (non-quantised) takes no antiquantScale or antiquantOffset");
  const wqmm_tensor* same[] = {scale, offset, bias, x3, output};
  const char* same_names[] = {"antiquantScale", "antiquantOffset", "bias", "x3", "output"};
  for (int i = 0; i < 5; ++i)
    if (same[i] && same[i]->dtype != adt)
      return fail(WQMM_ERR_PARAM_INVALID, "%s dtype %s must equal the x1 dtype %s", same_names[i],
                  dt_name(same[i]->dtype), dt_name(adt));

  // ---- CheckAttr
  wqmm_status st = common_attr_checks(reduce_op, comm_turn, stream_mode);
  if (st) return st;
  const int64_t k_attr = x1->ndim >= 2 ? x1->shape[x1->ndim - 1] : 0;
  if (k_attr != 0 && group_size != 0) {
    const int64_t hi = (k_attr - 1) < 2147483647LL ? (k_attr - 1) : 2147483647LL;
    if (group_size % 32 != 0 || group_size < 32 || group_size > hi)
      return fail(WQMM_ERR_PARAM_INVALID,
                  "antiquantGroupSize %lld must be 0 or a multiple of 32 in [32, min(k-1, INT32_MAX)] = [32, %lld]",
                  (long long)group_size, (long long)hi);
  }
  if (group_size < 0) return fail(WQMM_ERR_PARAM_INVALID, "antiquantGroupSize must not be negative");
  if (nonquant && group_size != 0)
    return fail(WQMM_ERR_PARAM_INVALID, "antiquantGroupSize must be 0 for x2 of the x1 dtype (non-quantised)");
  if (x2->dtype == WQMM_DT_FP8E4M3 && offset)
    return fail(WQMM_ERR_PARAM_INVALID, "antiquantOffset must be null for float8_e4m3fn weights");

  // ---- CheckShape
  if (x2->ndim != 2) return fail(WQMM_ERR_PARAM_INVALID, "x2 must be 2-D (k, n), got %d-D", x2->ndim);
  const int64_t k = x2->shape[0], n = x2->shape[1];
  if (x1->ndim < 2 || x1->shape[x1->ndim - 1] != k)
    return fail(WQMM_ERR_PARAM_INVALID, "k of x1 and x2 must be equal");
  if (k > 65535 || n > 65535 || n < 1)
    return fail(WQMM_ERR_PARAM_INVALID, "k = %lld, n = %lld: k must be in [0, 65535], n in [1, 65535]",
                (long long)k, (long long)n);
  int64_t m = 0;
  st = check_x1_out(x1, output, n, &m);
  if (st) return st;
  if (bias && (bias->ndim != 1 || bias->shape[0] != n || !contiguous(bias)))
    return fail(WQMM_ERR_PARAM_INVALID, "bias must be contiguous with shape (n) = (%lld)", (long long)n);
  if (x3 && (!same_shape(x3, output) || !contiguous(x3)))
    return fail(WQMM_ERR_PARAM_INVALID, "x3 must be contiguous with the output shape");
  // quantisation mode from the scale shape (per-group when G != 0)
  int mode;
  int64_t ng = 0;
  bool scale_t = false;
  if (nonquant) {
    mode = kNoQuant;
  } else if (group_size != 0 && k != 0) {
    mode = kPerGroup;
    ng = (k + group_size - 1) / group_size;
    if (scale->ndim != 2 || scale->shape[0] != ng || scale->shape[1] != n)
      return fail(WQMM_ERR_PARAM_INVALID, "per-group antiquantScale must have shape (ceil(k/G), n) = (%lld, %lld)",
                  (long long)ng, (long long)n);
    if (scale->strides[0] == n && scale->strides[1] == 1) {
      scale_t = false;
    } else if (scale->strides[0] == 1 && scale->strides[1] == ng) {
      scale_t = true;
    } else if (ng == 1) {
      scale_t = false;
    } else {
      return fail(WQMM_ERR_PARAM_INVALID, "per-group antiquantScale must be contiguous or transposed");
    }
  } else {
    const int64_t sn = numel(scale);
    if (scale->ndim == 1 && scale->shape[0] == 1) {
      mode = kPerTensor;
    } else if ((scale->ndim == 1 && scale->shape[0] == n) ||
               (scale->ndim == 2 && scale->shape[0] == 1 && scale->shape[1] == n)) {
      mode = kPerChannel;
    } else if (k == 0) {
      mode = (sn == 1) ? kPerTensor : kPerChannel;  // shape checks of the scale are moot when k == 0
    } else {
      return fail(WQMM_ERR_PARAM_INVALID, "antiquantScale must be (1) per-tensor or (n)/(1,n) per-channel");
    }
    if (!contiguous(scale)) return fail(WQMM_ERR_PARAM_INVALID, "antiquantScale must be contiguous");
  }
  if (offset) {
    if (!same_shape(offset, scale)) return fail(WQMM_ERR_PARAM_INVALID, "antiquantOffset shape must equal antiquantScale shape");
    for (int i = 0; i < scale->ndim; ++i)
      if (offset->shape[i] != 1 && offset->strides[i] != scale->strides[i])
        return fail(WQMM_ERR_PARAM_INVALID, "antiquantOffset must have the layout of antiquantScale");
  }
  if (x2->dtype == WQMM_DT_FP8E4M3 && mode != kPerChannel && k != 0)
    return fail(WQMM_ERR_PARAM_INVALID, "float8_e4m3fn weights support per-channel scales only");
  bool x2_t = false;
  st = check_x2_layout(x2, k, n, &x2_t);
  if (st) return st;
  if (mode == kPerGroup && x2->format != WQMM_FORMAT_PACKED && scale_t != x2_t && ng > 1)
    return fail(WQMM_ERR_PARAM_INVALID,
                "per-group: antiquantScale/antiquantOffset must be transposed together with x2");
  const int align = (x2->dtype == WQMM_DT_I4) ? 64 : 32;
  if (k % align != 0 || n % align != 0)
    return fail(WQMM_ERR_PARAM_INVALID, "%s weights need k and n to be multiples of %d (k = %lld, n = %lld)",
                dt_name(x2->dtype), align, (long long)k, (long long)n);
  for (int i = 0; i < 7; ++i) {
    if (!all[i]) continue;
    if (numel(all[i]) > 0 && all[i]->data == nullptr)
      return fail(WQMM_ERR_PARAM_NULLPTR, "%s: data pointer is null", names[i]);
    if (all[i]->data && !aligned16(all[i]->data))
      return fail(WQMM_ERR_PARAM_INVALID, "%s: data must be 16-byte aligned", names[i]);
  }

  // ---- plan
  wqmm_executor* ex = new (std::nothrow) wqmm_executor();
  if (!ex) return fail(WQMM_ERR_INNER_TILING, "out of host memory");
  ex->op = OpKind::kWqmm;
  ex->m = m;
  ex->k = static_cast<int>(k);
  ex->n = static_cast<int>(n);
  ex->act_dtype = adt;
  ex->x1 = x1->data;
  ex->x2 = x2->data;
  ex->x2_dtype = x2->dtype;
  ex->x2_packed = x2->format == WQMM_FORMAT_PACKED;
  ex->x2_s0 = x2_t ? 1 : n;
  ex->x2_s1 = x2_t ? k : 1;
  ex->out = output->data;
  ex->bias = bias ? bias->data : nullptr;
  ex->x3 = x3 ? x3->data : nullptr;
  ex->scale = scale ? scale->data : nullptr;
  ex->offset = offset ? offset->data : nullptr;
  ex->scale_transposed = scale_t;
  ex->mode = mode;
  ex->group_size = static_cast<int>(group_size);
  ex->num_groups = static_cast<int>(ng);
  uint64_t ws = 0;
  if (k > 0) {
    // m tile: the smallest supported width that covers m; larger m uses 256,
    // the widest MMA (the most MMA work per dequantised weight step)
    ex->bn = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256;
    {
      // 256 < m <= 512 with fewer tiles than SMs at both 256 and 128 rows: every
      // tile is split over the SMs either way, and the 128-row split is cheaper
      // than the 256-row one (measured on B200, W4A16 g128, k = n = 4096:
      // m = 384 43.0 vs 55.2 us, m = 512 47.1 vs 55.3 us)
      const int64_t nb = (n + kWqNBlock - 1) / kWqNBlock;
      const int64_t sl = sm_count();
      if (m > 256 && m <= 512 && ((m + 255) / 256) * nb < sl && ((m + 127) / 128) * nb <= sl) ex->bn = 128;
    }
    if (const char* env = std::getenv("WQMM_BN")) {  // tuning override
      const int v = std::atoi(env);
      if (v == 16 || v == 32 || v == 64 || v == 128 || v == 192 || v == 256) ex->bn = v;
    }
    const int64_t num_mb = (m + ex->bn - 1) / ex->bn;
    const int64_t num_nb = (n + kWqNBlock - 1) / kWqNBlock;
    const int64_t kt = (k + kWqKTile - 1) / kWqKTile;
    const int64_t tiles = num_mb * num_nb;
    if (tiles > 0x7FFFFFFFLL) {
      delete ex;
      return fail(WQMM_ERR_INNER_TILING, "too many output tiles");
    }
    int64_t slots = static_cast<int64_t>(sm_count()) * wqmm_ctas_per_sm(ex->bn, 0);
    if (const char* env = std::getenv("WQMM_GRID")) {  // testing override: fewer persistent CTAs
      const int64_t v = std::atoll(env);
      if (v >= 1 && v < slots) slots = v;
    }
    ex->num_tiles = static_cast<int>(tiles);
    ex->stream_k = 0;
    ex->dp_tiles = 0;
    ex->grid = static_cast<int>(tiles < slots ? tiles : slots);
    const char* sk_env = std::getenv("WQMM_STREAMK");
    const bool force_sk = sk_env && std::atoi(sk_env) == 1;
    const bool forbid_sk = sk_env && std::atoi(sk_env) == 0;
    // m <= 32: the small-m kernel (WQMM_SMALLM=0 selects the general kernel).
    // Its CTAs share the k steps of all tiles evenly (stream-K over every tile,
    // at least 16 k steps per CTA, so that its four dequantisation groups each
    // get several), unless WQMM_STREAMK=0 asks for whole tiles.
    {
      const char* sm_env = std::getenv("WQMM_SMALLM");
      // (16-bit weights, the non-quantised scenario, run on the general kernel)
      ex->smallm = (ex->bn == 16 || ex->bn == 32) && !nonquant && !(sm_env && std::atoi(sm_env) == 0) ? 1 : 0;
    }
    if (ex->smallm && !forbid_sk) {
      // units of two k steps when the step count is even: the kernel then takes
      // two-step turns, and every split point falls on a turn boundary
      const int unit = kt % 2 == 0 ? 2 : 1;
      const int64_t T = tiles * kt / unit;
      int64_t grid = (T * unit + 15) / 16;
      grid = grid < 1 ? 1 : (grid > slots ? slots : grid);
      int ms = 1;
      for (int64_t r = 0; r < tiles; ++r) {
        const SkOwners o = sk_tile_owners(r, static_cast<int>(kt), unit, T, grid);
        if (o.last - o.first + 1 > ms) ms = static_cast<int>(o.last - o.first + 1);
      }
      const uint64_t partial_bytes = ms > 1 ? static_cast<uint64_t>(tiles) * ms * ex->bn * kWqNBlock * 4 : 0;
      uint64_t other = 0;
      if (!(x2->format == WQMM_FORMAT_PACKED)) other = round_up(packed_bytes_for(x2->dtype, k, n, false), 256);
      if (mode == kPerGroup && scale_t) other += (offset ? 2 : 1) * round_up(static_cast<uint64_t>(ng) * n * 2, 256);
      const uint64_t sk_bytes = round_up(partial_bytes, 256) + round_up(static_cast<uint64_t>(tiles) * ms * 8, 256);
      if (!(g_plan_ws_cap > 0 && ms > 1 && other + sk_bytes > g_plan_ws_cap)) {
        ex->stream_k = 1;
        ex->dp_tiles = 0;
        ex->sk_unit = unit;
        ex->sk_grid = static_cast<int>(grid);
        ex->grid = static_cast<int>(grid);
        ex->max_slots = ms;
        ex->sk_inline = ms <= 4 ? 1 : 0;
        if (const char* env = std::getenv("WQMM_SK_INLINE")) ex->sk_inline = (std::atoi(env) == 1 && ms <= 4) ? 1 : 0;
      }
    }
    // Stream-K: with fewer tiles than CTAs, the k steps of all tiles are spread
    // evenly over the CTAs.  With more, narrow m tiles (< 128 rows) run the whole
    // waves as whole tiles and split a last, partly filled wave (at most 85%
    // full) the same way over every CTA, so that no SM idles while others finish
    // it.  (Measured on B200, wide tiles gain less from the split than its
    // partial tiles cost.)  Splits fall on pairs of k steps when the
    // dequantisers take two-step turns.
    const int64_t rem = tiles % slots;
    int64_t dp = -1;  // tiles run whole before the split ones; -1: no stream-K
    if (!ex->smallm && !forbid_sk && kt >= 2) {
      if (force_sk || tiles < slots)
        dp = 0;
      else if (ex->bn < 128 && rem > 0 && rem * 100 <= 85 * slots)
        dp = tiles - rem;
    }
    if (dp >= 0) {
      const int unit = (ex->bn >= 128 && kt % 2 == 0) ? 2 : 1;
      const int64_t split = tiles - dp;
      const int64_t T = split * kt / unit;
      const int64_t grid = dp > 0 ? slots : (T < slots ? T : slots);
      const int64_t sk_grid = T < grid ? T : grid;  // every sharing CTA gets at least one unit
      int ms = 1;
      for (int64_t r = 0; r < split; ++r) {
        const SkOwners o = sk_tile_owners(r, static_cast<int>(kt), unit, T, sk_grid);
        if (o.last - o.first + 1 > ms) ms = static_cast<int>(o.last - o.first + 1);
      }
      const uint64_t partial_bytes = static_cast<uint64_t>(split) * ms * ex->bn * kWqNBlock * 4;
      // A caller with a fixed workspace (g_plan_ws_cap) gets a schedule without
      // split tiles when their partials and flags would not fit beside the
      // other workspace regions: whole tiles are slower for these shapes but
      // need no workspace of their own.
      uint64_t other = 0;
      if (!(x2->format == WQMM_FORMAT_PACKED)) other = round_up(packed_bytes_for(x2->dtype, k, n, false), 256);
      if (mode == kPerGroup && scale_t) other += (offset ? 2 : 1) * round_up(static_cast<uint64_t>(ng) * n * 2, 256);
      const uint64_t sk_bytes = round_up(partial_bytes, 256) + round_up(static_cast<uint64_t>(split) * ms * 8, 256);
      if (!(g_plan_ws_cap > 0 && other + sk_bytes > g_plan_ws_cap)) {
        ex->stream_k = 1;
        ex->dp_tiles = static_cast<int>(dp);
        ex->sk_unit = unit;
        ex->sk_grid = static_cast<int>(sk_grid);
        ex->grid = static_cast<int>(grid);
        ex->max_slots = ms;
        // a few owners per tile: the first owner, which reaches its part last,
        // adds the others' partials itself; many: a fix-up kernel spreads the sums
        ex->sk_inline = ms <= 4 ? 1 : 0;
        if (const char* env = std::getenv("WQMM_SK_INLINE")) ex->sk_inline = (std::atoi(env) == 1 && ms <= 4) ? 1 : 0;
      }
    }
    // 192- and 256-row m tiles over whole tiles can run as clusters of two CTAs
    // that share each MMA (each CTA holds half of the x1 slab, so the x1 ring
    // and the MMA issuer's batches are twice as deep).  Measured on B200 the
    // 256-row pairs are faster for int4 weights (W4A16 g128 4096^3: 137.7 vs
    // 141.3 us) and not for int8 (W8A16 2048x4096x4096: 94.3 vs 92.2 us): the
    // default for int4 at 256 rows; WQMM_PAIR=1 / 0 forces them on / off.
    const char* pair_env = std::getenv("WQMM_PAIR");
    const int wk = weight_kind(x2->dtype);
    const bool want_pair = pair_env ? std::atoi(pair_env) == 1 : (ex->bn == 256 && wk == kW4);
    if (!ex->smallm && !ex->stream_k && want_pair && (ex->bn == 192 || ex->bn == 256) && num_nb >= 2) {
      const int ps = pair_slots(ex->bn, wk, adt == WQMM_DT_BF16);
      if (ps > 0) {
        const int64_t pnb = (num_nb + 1) / 2;
        const int64_t ptiles = num_mb * pnb;
        ex->pair = 1;
        ex->num_pnb = static_cast<int>(pnb);
        ex->num_tiles = static_cast<int>(ptiles);
        ex->grid = static_cast<int>(2 * (ptiles < ps ? ptiles : ps));
      }
    }
    if (!ex->x2_packed) {
      ex->ws_pack = {ws, packed_bytes_for(x2->dtype, k, n, false)};
      ws = round_up(ws + ex->ws_pack.bytes, 256);
    }
    if (mode == kPerGroup && scale_t) {
      ex->ws_scale = {ws, static_cast<uint64_t>(ng) * n * 2};
      ws = round_up(ws + ex->ws_scale.bytes, 256);
      if (offset) {
        ex->ws_offset = {ws, static_cast<uint64_t>(ng) * n * 2};
        ws = round_up(ws + ex->ws_offset.bytes, 256);
      }
    }
    if (ex->stream_k && ex->max_slots > 1) {  // one owner per tile: no partials
      ex->ws_partial = {ws, static_cast<uint64_t>(tiles - ex->dp_tiles) * ex->max_slots * ex->bn * kWqNBlock * 4};
      ws = round_up(ws + ex->ws_partial.bytes, 256);
      if (ex->sk_inline) {
        ex->ws_flags = {ws, static_cast<uint64_t>(tiles - ex->dp_tiles) * ex->max_slots * 8};
        ws = round_up(ws + ex->ws_flags.bytes, 256);
      }
    }
  }
  ex->workspace = ws;
  *workspace_size = ws;
  *executor = register_executor(ex);
  return ok();
}

// ===================================================================== qmm phase 1
extern "C" wqmm_status qmm_get_workspace_size(const wqmm_tensor* x1, const wqmm_tensor* x2, const wqmm_tensor* bias,
                                              const wqmm_tensor* x3, const wqmm_tensor* dq,
                                              const wqmm_tensor* pertoken, const char* group,
                                              const char* reduce_op, int64_t comm_turn, int64_t stream_mode,
                                              const wqmm_tensor* output, uint64_t* workspace_size,
                                              wqmm_executor** executor) {
  (void)group;
  // ---- CheckNotNull
  if (!x1 || !x2 || !dq || !output)
    return fail(WQMM_ERR_PARAM_NULLPTR, "x1, x2, dequantScale and output must not be null");
  if (!reduce_op) return fail(WQMM_ERR_PARAM_NULLPTR, "reduceOp must not be null");
  if (!workspace_size || !executor) return fail(WQMM_ERR_PARAM_NULLPTR, "workspaceSize and executor must not be null");
  *executor = nullptr;
  *workspace_size = 0;
  const wqmm_tensor* all[] = {x1, x2, bias, x3, dq, pertoken, output};
  const char* names[] = {"x1", "x2", "bias", "x3", "dequantScale", "pertokenScale", "output"};
  for (int i = 0; i < 7; ++i) {
    if (!all[i]) continue;
    wqmm_status st = check_descriptor(all[i], names[i]);
    if (st) return st;
    if (i != 1 && all[i]->format != WQMM_FORMAT_ND)
      return fail(WQMM_ERR_PARAM_INVALID, "%s: only x2 may use the packed format", names[i]);
  }
  // ---- dtypes (parameter table of aclnnQuantMatmulAllReduceV2)
  if (x1->dtype != WQMM_DT_I8) return fail(WQMM_ERR_PARAM_INVALID, "x1 must be int8, got %s", dt_name(x1->dtype));
  if (x2->dtype != WQMM_DT_I8) return fail(WQMM_ERR_PARAM_INVALID, "x2 must be int8, got %s", dt_name(x2->dtype));
  if (bias && bias->dtype != WQMM_DT_I32) return fail(WQMM_ERR_PARAM_INVALID, "bias must be int32");
  if (!act_dtype_ok(output->dtype)) return fail(WQMM_ERR_PARAM_INVALID, "output must be float16 or bfloat16");
  if (x3 && x3->dtype != output->dtype) return fail(WQMM_ERR_PARAM_INVALID, "x3 dtype must equal the output dtype");
  if (pertoken && pertoken->dtype != WQMM_DT_F32) return fail(WQMM_ERR_PARAM_INVALID, "pertokenScale must be float32");
  if (output->dtype == WQMM_DT_BF16 && dq->dtype != WQMM_DT_BF16)
    return fail(WQMM_ERR_PARAM_INVALID, "bfloat16 output needs a bfloat16 dequantScale, got %s", dt_name(dq->dtype));
  if (output->dtype == WQMM_DT_F16) {
    if (dq->dtype == WQMM_DT_I64 || dq->dtype == WQMM_DT_U64)
      return fail(WQMM_ERR_PARAM_INVALID,
                  "int64/uint64 (TransQuantParamV2-encoded) dequantScale is not supported; pass float32");
    if (dq->dtype != WQMM_DT_F32)
      return fail(WQMM_ERR_PARAM_INVALID, "float16 output needs a float32 dequantScale, got %s", dt_name(dq->dtype));
  }
  // ---- attributes
  wqmm_status st = common_attr_checks(reduce_op, comm_turn, stream_mode);
  if (st) return st;
  // ---- shapes
  if (x2->ndim != 2) return fail(WQMM_ERR_PARAM_INVALID, "x2 must be 2-D (k, n)");
  const int64_t k = x2->shape[0], n = x2->shape[1];
  if (x1->ndim < 2 || x1->shape[x1->ndim - 1] != k) return fail(WQMM_ERR_PARAM_INVALID, "k of x1 and x2 must be equal");
  if (k < 1 || n < 1) return fail(WQMM_ERR_PARAM_INVALID, "empty tensors are not supported");
  if (k > 65535 || n > 65535) return fail(WQMM_ERR_PARAM_INVALID, "k and n must be <= 65535");
  int64_t m = 0;
  st = check_x1_out(x1, output, n, &m);
  if (st) return st;
  if (bias && (bias->ndim != 1 || bias->shape[0] != n || !contiguous(bias)))
    return fail(WQMM_ERR_PARAM_INVALID, "bias must have shape (n)");
  if (x3 && (!same_shape(x3, output) || !contiguous(x3)))
    return fail(WQMM_ERR_PARAM_INVALID, "x3 must have the output shape");
  const int64_t dqn = numel(dq);
  bool dq_tensor;
  if (dq->ndim == 1 && dq->shape[0] == 1)
    dq_tensor = true;
  else if ((dq->ndim == 1 && dq->shape[0] == n) || (dq->ndim == 2 && dq->shape[0] == 1 && dq->shape[1] == n))
    dq_tensor = false;
  else
    return fail(WQMM_ERR_PARAM_INVALID, "dequantScale must be (1), (n) or (1, n)");
  (void)dqn;
  if (!contiguous(dq)) return fail(WQMM_ERR_PARAM_INVALID, "dequantScale must be contiguous");
  if (pertoken && (pertoken->ndim != 1 || pertoken->shape[0] != m || !contiguous(pertoken)))
    return fail(WQMM_ERR_PARAM_INVALID, "pertokenScale must have shape (m) = (%lld)", (long long)m);
  bool x2_t = false;
  st = check_x2_layout(x2, k, n, &x2_t);
  if (st) return st;
  if (k % 32 != 0 || n % 32 != 0)
    return fail(WQMM_ERR_PARAM_INVALID, "int8 weights need k and n to be multiples of 32 (k = %lld, n = %lld)",
                (long long)k, (long long)n);
  for (int i = 0; i < 7; ++i) {
    if (!all[i]) continue;
    if (all[i]->data == nullptr) return fail(WQMM_ERR_PARAM_NULLPTR, "%s: data pointer is null", names[i]);
    if (!aligned16(all[i]->data)) return fail(WQMM_ERR_PARAM_INVALID, "%s: data must be 16-byte aligned", names[i]);
  }
  // ---- plan
  wqmm_executor* ex = new (std::nothrow) wqmm_executor();
  if (!ex) return fail(WQMM_ERR_INNER_TILING, "out of host memory");
  ex->op = OpKind::kQmm;
  ex->m = m;
  ex->k = static_cast<int>(k);
  ex->n = static_cast<int>(n);
  ex->act_dtype = output->dtype;
  ex->x1 = x1->data;
  ex->x2 = x2->data;
  ex->x2_dtype = WQMM_DT_I8;
  ex->x2_packed = x2->format == WQMM_FORMAT_PACKED;
  ex->x2_s0 = x2_t ? 1 : n;
  ex->x2_s1 = x2_t ? k : 1;
  ex->out = output->data;
  ex->bias = bias ? bias->data : nullptr;
  ex->x3 = x3 ? x3->data : nullptr;
  ex->dq = dq->data;
  ex->dq_dtype = dq->dtype;
  ex->dq_per_tensor = dq_tensor;
  ex->pertoken = pertoken ? static_cast<const float*>(pertoken->data) : nullptr;
  uint64_t ws = 0;
  if (!ex->x2_packed) {
    ex->ws_pack = {0, packed_bytes_for(WQMM_DT_I8, k, n, true)};
    ws = round_up(ex->ws_pack.bytes, 256);
  }
  ex->workspace = ws;
  *workspace_size = ws;
  *executor = register_executor(ex);
  return ok();
}

// ===================================================================== phase 2
namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static std::once_flag once;
  static EncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// 2-D row-major matrix (rows x cols elements of `esize` bytes), box (box_cols x
// box_rows), 128-byte swizzle unless told otherwise, out-of-bounds elements
// read as zero.
wqmm_status make_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, int64_t rows,
                      int64_t cols, int box_cols, int box_rows,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeFn fn = encode_fn();
  if (!fn) return fail(WQMM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WQMM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return WQMM_SUCCESS;
}

wqmm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(WQMM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

wqmm_status take_executor(wqmm_executor* ex, OpKind op) {
  if (!ex) return fail(WQMM_ERR_EXECUTOR, "executor is null");
  if (!is_live(ex) || ex->magic != kMagicLive)
    return fail(WQMM_ERR_EXECUTOR, "executor was already consumed or destroyed");
  if (ex->op != op) return fail(WQMM_ERR_EXECUTOR, "executor belongs to the other operator");
  return WQMM_SUCCESS;
}

void release(wqmm_executor* ex) {
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    if (g_live.erase(ex) == 0) return;
  }
  ex->magic = kMagicDead;
  delete ex;
}

wqmm_status check_workspace(const wqmm_executor* ex, void* ws, uint64_t size) {
  if (size < ex->workspace)
    return fail(WQMM_ERR_WORKSPACE, "workspace of %llu bytes is smaller than the %llu bytes phase 1 reported",
                (unsigned long long)size, (unsigned long long)ex->workspace);
  if (ex->workspace > 0 && ws == nullptr) return fail(WQMM_ERR_WORKSPACE, "workspace is null but %llu bytes are needed",
                                                     (unsigned long long)ex->workspace);
  if (ws && !aligned16(ws)) return fail(WQMM_ERR_WORKSPACE, "workspace must be 16-byte aligned");
  return WQMM_SUCCESS;
}

wqmm_status run_wqmm(void* ws, wqmm_executor* ex, cudaStream_t s) {
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const bool bf16 = ex->act_dtype == WQMM_DT_BF16;
  const int wk = weight_kind(ex->x2_dtype);
  cudaError_t e;
  if (ex->k == 0) {
    EpiParams ep{};
    ep.scale = static_cast<const uint16_t*>(ex->scale);
    ep.bias = static_cast<const uint16_t*>(ex->bias);
    ep.x3 = static_cast<const uint16_t*>(ex->x3);
    ep.out = static_cast<uint16_t*>(ex->out);
    ep.m = ex->m;
    ep.n = ex->n;
    ep.splits = 0;
    ep.mode = ex->mode;
    ep.wk = wk;
    ep.act_bf16 = bf16;
    e = launch_wqmm_epilogue(ep, s);
    return e == cudaSuccess ? WQMM_SUCCESS : cuda_fail(e, "epilogue launch");
  }
  const uint8_t* wpack = static_cast<const uint8_t*>(ex->x2);
  if (!ex->x2_packed) {
    PackParams pp{};
    pp.src = static_cast<const uint8_t*>(ex->x2);
    pp.dst = wsb + ex->ws_pack.offset;
    pp.s0 = ex->x2_s0;
    pp.s1 = ex->x2_s1;
    pp.k = ex->k;
    pp.n = ex->n;
    pp.wk = wk;
    pp.for_qmm = 0;
    e = launch_pack(pp, s);
    if (e != cudaSuccess) return cuda_fail(e, "weight pack launch");
    wpack = pp.dst;
  }
  const uint16_t* scale = static_cast<const uint16_t*>(ex->scale);
  const uint16_t* offset = static_cast<const uint16_t*>(ex->offset);
  if (ex->mode == kPerGroup && ex->scale_transposed) {
    uint16_t* st = reinterpret_cast<uint16_t*>(wsb + ex->ws_scale.offset);
    e = launch_transpose_u16(scale, st, ex->num_groups, ex->n, s);
    if (e != cudaSuccess) return cuda_fail(e, "scale transpose launch");
    scale = st;
    if (offset) {
      uint16_t* ot = reinterpret_cast<uint16_t*>(wsb + ex->ws_offset.offset);
      e = launch_transpose_u16(offset, ot, ex->num_groups, ex->n, s);
      if (e != cudaSuccess) return cuda_fail(e, "offset transpose launch");
      offset = ot;
    }
  }
  CUtensorMap tmap;
  if (!ex->smallm) {  // the small-m kernel reads x1 with plain 16-byte copies
    const CUtensorMapDataType dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    wqmm_status st = make_tmap(&tmap, ex->x1, dt, 2, ex->m, ex->k, kWqKTile, ex->pair ? ex->bn / 2 : ex->bn);
    if (st) return st;
  }
  WqParams p{};
  p.x1 = static_cast<const uint16_t*>(ex->x1);
  p.wpack = wpack;
  p.scale = scale;
  p.offset = offset;
  p.bias = static_cast<const uint16_t*>(ex->bias);
  p.x3 = static_cast<const uint16_t*>(ex->x3);
  p.out = static_cast<uint16_t*>(ex->out);
  p.partial = (ex->stream_k && ex->max_slots > 1) ? reinterpret_cast<float*>(wsb + ex->ws_partial.offset) : nullptr;
  p.err = device_error_word();
  p.m = ex->m;
  p.n = ex->n;
  p.k = ex->k;
  p.kt_total = (ex->k + kWqKTile - 1) / kWqKTile;
  p.num_nb = (ex->n + kWqNBlock - 1) / kWqNBlock;
  p.num_mb = static_cast<int>((ex->m + ex->bn - 1) / ex->bn);
  p.num_tiles = ex->num_tiles;
  p.pair = ex->pair;
  p.num_pnb = ex->num_pnb;
  p.stream_k = ex->stream_k;
  p.dp_tiles = ex->dp_tiles;
  p.sk_unit = ex->sk_unit;
  p.sk_grid = ex->sk_grid;
  p.sk_inline = ex->sk_inline;
  p.sk_flags = (ex->sk_inline && ex->max_slots > 1) ? reinterpret_cast<uint64_t*>(wsb + ex->ws_flags.offset) : nullptr;
  p.sk_token = ex->sk_inline ? next_launch_token() : 0;
  p.sk_expect = p.sk_token + (ex->debug_flag_mismatch ? 2 : 0);
  p.sk_wait_ns = ex->debug_wait_ns > 0 ? ex->debug_wait_ns : kFlagWaitNs;
  p.max_slots = ex->max_slots;
  p.mode = ex->mode;
  p.group_size = ex->group_size;
  p.num_groups = ex->num_groups;
  e = ex->smallm ? launch_wqmm_smallm(p, ex->bn, wk, bf16, ex->grid, s)
                 : launch_wqmm_gemm(tmap, p, ex->bn, wk, bf16, ex->grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "anti-quant GEMM launch");
  if (ex->stream_k && !ex->sk_inline && ex->max_slots > 1) {
    FixupParams fp{};
    fp.partial = p.partial;
    fp.scale = scale;
    fp.offset = offset;
    fp.bias = p.bias;
    fp.x3 = p.x3;
    fp.out = p.out;
    fp.m = ex->m;
    fp.n = ex->n;
    fp.bn = ex->bn;
    fp.num_nb = p.num_nb;
    fp.num_tiles = ex->num_tiles;
    fp.dp_tiles = ex->dp_tiles;
    fp.kt_total = p.kt_total;
    fp.sk_unit = ex->sk_unit;
    fp.sk_grid = ex->sk_grid;
    fp.max_slots = ex->max_slots;
    fp.mode = ex->mode;
    fp.act_bf16 = bf16;
    e = launch_wqmm_fixup(fp, s);
    if (e != cudaSuccess) return cuda_fail(e, "stream-K fix-up launch");
  }
  return WQMM_SUCCESS;
}

wqmm_status run_qmm(void* ws, wqmm_executor* ex, cudaStream_t s) {
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const uint8_t* wpack = static_cast<const uint8_t*>(ex->x2);
  cudaError_t e;
  if (!ex->x2_packed) {
    PackParams pp{};
    pp.src = static_cast<const uint8_t*>(ex->x2);
    pp.dst = wsb + ex->ws_pack.offset;
    pp.s0 = ex->x2_s0;
    pp.s1 = ex->x2_s1;
    pp.k = ex->k;
    pp.n = ex->n;
    pp.wk = kW8;
    pp.for_qmm = 1;
    e = launch_pack(pp, s);
    if (e != cudaSuccess) return cuda_fail(e, "weight pack launch");
    wpack = pp.dst;
  }
  CUtensorMap tmap;
  wqmm_status st = make_tmap(&tmap, ex->x1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ex->m, ex->k, kQKTile, 128);
  if (st) return st;
  QParams p{};
  p.wpack = wpack;
  p.bias = static_cast<const int32_t*>(ex->bias);
  p.dq = ex->dq;
  p.pertoken = ex->pertoken;
  p.x3 = static_cast<const uint16_t*>(ex->x3);
  p.out = static_cast<uint16_t*>(ex->out);
  p.raw_acc = ex->raw_acc;
  p.err = device_error_word();
  p.m = ex->m;
  p.n = ex->n;
  p.k = ex->k;
  p.kt_total = (ex->k + kQKTile - 1) / kQKTile;
  p.num_nb = (ex->n + kQNBlock - 1) / kQNBlock;
  p.num_mb = static_cast<int>((ex->m + 127) / 128);
  p.dq_bf16 = ex->dq_dtype == WQMM_DT_BF16;
  p.dq_per_tensor = ex->dq_per_tensor;
  p.out_bf16 = ex->act_dtype == WQMM_DT_BF16;
  // enough 256-row tiles for every pair of SMs: clusters of two CTAs share
  // each MMA, so each SM loads half of the weight tile (WQMM_PAIR=0 turns it off)
  p.pair_grid = 0;
  {
    const char* pair_env = std::getenv("WQMM_PAIR");
    const bool forbid_pair = pair_env && std::atoi(pair_env) == 0;
    const bool force_pair = pair_env && std::atoi(pair_env) == 1;  // tests: pairs at any size
    const int64_t ptiles = static_cast<int64_t>((p.num_mb + 1) / 2) * p.num_nb;
    const int slots = forbid_pair ? 0 : qmm_pair_slots_cached(p.out_bf16 != 0);
    if (slots > 0 && (ptiles >= slots || force_pair)) p.pair_grid = static_cast<int>(2 * (ptiles < slots ? ptiles : slots));
  }
  CUtensorMap tmap_w = tmap;
  if (p.pair_grid > 0) {
    // the packed weight is already in the shared-memory (swizzled) order: a
    // plain 2-D view, 128-byte rows, each CTA of a pair copying 128 of them
    const int64_t rows = static_cast<int64_t>(p.num_nb) * p.kt_total * kQNBlock;
    st = make_tmap(&tmap_w, wpack, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, kQKTile, kQKTile, kQNBlock / 2,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st) return st;
  }
  e = launch_qmm_gemm(tmap, tmap_w, p, s);
  if (e != cudaSuccess) return cuda_fail(e, "int8 GEMM launch");
  return WQMM_SUCCESS;
}

}  // namespace

extern "C" wqmm_status wqmm_run(void* workspace, uint64_t workspace_size, wqmm_executor* executor,
                                wqmm_stream stream) {
  wqmm_status st = take_executor(executor, OpKind::kWqmm);
  if (st) return st;
  st = check_workspace(executor, workspace, workspace_size);
  if (st == WQMM_SUCCESS) st = run_wqmm(workspace, executor, reinterpret_cast<cudaStream_t>(stream));
  release(executor);
  return st == WQMM_SUCCESS ? ok() : st;
}

extern "C" wqmm_status qmm_run(void* workspace, uint64_t workspace_size, wqmm_executor* executor,
                               wqmm_stream stream) {
  wqmm_status st = take_executor(executor, OpKind::kQmm);
  if (st) return st;
  st = check_workspace(executor, workspace, workspace_size);
  if (st == WQMM_SUCCESS) st = run_qmm(workspace, executor, reinterpret_cast<cudaStream_t>(stream));
  release(executor);
  return st == WQMM_SUCCESS ? ok() : st;
}

// ===================================================================== weight packing
namespace {
wqmm_status check_pack_args(const wqmm_tensor* x2, int32_t for_qmm, bool* transposed) {
  if (!x2) return fail(WQMM_ERR_PARAM_NULLPTR, "x2 must not be null");
  wqmm_status st = check_descriptor(x2, "x2");
  if (st) return st;
  if (x2->format != WQMM_FORMAT_ND) return fail(WQMM_ERR_PARAM_INVALID, "x2 to pack must be in the ND format");
  if (x2->ndim != 2) return fail(WQMM_ERR_PARAM_INVALID, "x2 must be 2-D (k, n)");
  if (for_qmm) {
    if (x2->dtype != WQMM_DT_I8) return fail(WQMM_ERR_PARAM_INVALID, "the int8 GEMM packs int8 weights only");
  } else if (x2->dtype != WQMM_DT_I8 && x2->dtype != WQMM_DT_I4 && x2->dtype != WQMM_DT_FP8E4M3 &&
             !act_dtype_ok(x2->dtype)) {
    return fail(WQMM_ERR_PARAM_INVALID, "x2 dtype %s cannot be packed", dt_name(x2->dtype));
  }
  const int64_t k = x2->shape[0], n = x2->shape[1];
  if (k < 1 || n < 1 || k > 65535 || n > 65535) return fail(WQMM_ERR_PARAM_INVALID, "k and n must be in [1, 65535]");
  const int align = (x2->dtype == WQMM_DT_I4) ? 64 : 32;
  if (k % align || n % align)
    return fail(WQMM_ERR_PARAM_INVALID, "k and n must be multiples of %d for %s weights", align, dt_name(x2->dtype));
  return check_x2_layout(x2, k, n, transposed);
}
}  // namespace

extern "C" wqmm_status wqmm_pack_weight_size(const wqmm_tensor* x2, int32_t for_int8_gemm, uint64_t* packed_bytes) {
  if (!packed_bytes) return fail(WQMM_ERR_PARAM_NULLPTR, "packed_bytes must not be null");
  bool t = false;
  wqmm_status st = check_pack_args(x2, for_int8_gemm, &t);
  if (st) return st;
  *packed_bytes = packed_bytes_for(x2->dtype, x2->shape[0], x2->shape[1], for_int8_gemm != 0);
  return ok();
}

extern "C" wqmm_status wqmm_pack_weight(const wqmm_tensor* x2, int32_t for_int8_gemm, void* packed,
                                        wqmm_stream stream) {
  bool t = false;
  wqmm_status st = check_pack_args(x2, for_int8_gemm, &t);
  if (st) return st;
  if (!packed || !x2->data) return fail(WQMM_ERR_PARAM_NULLPTR, "x2 data and the packed buffer must not be null");
  if (!aligned16(packed)) return fail(WQMM_ERR_PARAM_INVALID, "packed buffer must be 16-byte aligned");
  PackParams pp{};
  pp.src = static_cast<const uint8_t*>(x2->data);
  pp.dst = static_cast<uint8_t*>(packed);
  pp.k = static_cast<int>(x2->shape[0]);
  pp.n = static_cast<int>(x2->shape[1]);
  pp.s0 = t ? 1 : pp.n;
  pp.s1 = t ? pp.k : 1;
  pp.wk = weight_kind(x2->dtype);
  pp.for_qmm = for_int8_gemm != 0;
  cudaError_t e = launch_pack(pp, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight pack launch");
  return ok();
}

// ===================================================================== utilities
extern "C" void wqmm_executor_destroy(wqmm_executor* executor) {
  if (executor) release(executor);
}

extern "C" const char* wqmm_last_error(void) { return g_last_error.c_str(); }

extern "C" wqmm_status wqmm_stream_wait(wqmm_stream stream, int32_t timeout_ms) {
  const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms < 0 ? 0 : timeout_ms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  while (true) {
    cudaError_t e = cudaStreamQuery(s);
    if (e == cudaSuccess) return ok();
    if (e != cudaErrorNotReady) return cuda_fail(e, "stream query");
    if (std::chrono::steady_clock::now() >= deadline)
      return fail(WQMM_ERR_TIMEOUT, "stream still busy after %d ms", static_cast<int>(timeout_ms));
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

extern "C" const char* wqmm_version(void) { return "wqmm 0.1 sm_100a"; }

extern "C" wqmm_status qmm_debug_set_raw_accumulator(wqmm_executor* executor, void* acc_i32_out) {
  wqmm_status st = take_executor(executor, OpKind::kQmm);
  if (st) return st;
  if (acc_i32_out && !aligned16(acc_i32_out)) return fail(WQMM_ERR_PARAM_INVALID, "accumulator buffer must be 16-byte aligned");
  executor->raw_acc = static_cast<int32_t*>(acc_i32_out);
  return ok();
}

extern "C" wqmm_status wqmm_debug_set_flag_wait(wqmm_executor* executor, uint64_t wait_ns, int32_t mismatch) {
  wqmm_status st = take_executor(executor, OpKind::kWqmm);
  if (st) return st;
  executor->debug_wait_ns = wait_ns;
  executor->debug_flag_mismatch = mismatch != 0;
  return ok();
}

extern "C" wqmm_status wqmm_device_error(uint32_t* code, int32_t reset) {
  if (!code) return fail(WQMM_ERR_PARAM_NULLPTR, "code must not be null");
  uint32_t* w = device_error_word();
  if (!w) return fail(WQMM_ERR_CUDA, "device error word unavailable");
  cudaError_t e = cudaMemcpy(code, w, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpy(w, &zero, sizeof(uint32_t), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "reset device error word");
  }
  return ok();
}

namespace wqmm {
// Record a message for wqmm_last_error() from another translation unit of the library.
wqmm_status report_error(wqmm_status code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace wqmm
