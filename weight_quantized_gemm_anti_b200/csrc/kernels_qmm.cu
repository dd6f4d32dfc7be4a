// kernels_qmm.cu -- int8 x int8 GEMM on the sm_100a tensor cores, after
// aclnnQuantMatmulAllReduceV2 ("Function", cases 1 and 2):
//     out = dequantScale * pertokenScale * (x1_int8 @ x2_int8 + bias_int32) + x3
//
//   * one CTA owns a 128 (m) x 256 (n) output tile; its int32 accumulator
//     (128 lanes x 256 columns) lives in TMEM;
//   * warp 0 (one thread) stages, per 128-byte k step, the x1 tile with a 2-D
//     tensor copy (128-byte swizzle) and the packed weight tile -- already
//     stored in that swizzled order by the packing kernel -- with one 32 KB
//     1-D bulk copy, into a 4-deep shared-memory ring;
//   * warp 1 (one thread) issues four tcgen05.mma kind::i8 (M=128, N=256,
//     K=32) per k step, both operands from shared memory;
//   * warps 2..5 read the accumulator with tcgen05.ld (thread = output row) and
//     apply the epilogue in fp32: (acc + bias) * dq[n] * pt[m] + x3, one
//     rounding to bf16/f16, 16-byte vector stores; optionally they also store
//     the raw int32 accumulator (+ bias) for bit-exact testing.
// The int32 sum of x1*x2 products is exact (|sum| < 2^31 for k <= 65535 with
// the bias added in two's complement, as a 32-bit accumulator does).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace wqmm {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kBM = 128;
constexpr int kBN = kQNBlock;       // 256
constexpr int kABytes = kBM * 128;  // 16 KB
constexpr int kBBytes = kQTileBytes;
constexpr int kTmemCols = 256;
constexpr int kSmemBytes = kStages * (kABytes + kBBytes) + 1024;

__device__ __forceinline__ float act_f32(uint16_t v, bool bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(v) << 16) : __half2float(__ushort_as_half(v));
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  if constexpr (BF16)
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    qmm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x1, const QParams p) {
  constexpr uint32_t kIdesc = idesc_make(2u, 1u, kBM, kBN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;
  uint8_t* s_b = smem + kStages * kABytes;

  __shared__ __align__(8) uint64_t bar_full[kStages];
  __shared__ __align__(8) uint64_t bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_acc;
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = blockIdx.x % p.num_nb;
  const int mb = blockIdx.x / p.num_nb;
  const int64_t m0 = static_cast<int64_t>(mb) * kBM;
  const int n0 = nb * kBN;
  const int n_iter = p.kt_total;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_acc, 1);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmap_x1);
      int issued = 0;
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % kStages;
        if (!mbar_wait(&bar_empty[st], ((i / kStages) & 1) ^ 1, abort_flag, p.err, kDevTimeoutProducer)) break;
        mbar_arrive_expect_tx(&bar_full[st], kABytes + kBBytes);
        tma_load_2d(s_a + st * kABytes, &tmap_x1, &bar_full[st], i * kQKTile, static_cast<int32_t>(m0));
        bulk_g2s(s_b + st * kBBytes, p.wpack + (static_cast<int64_t>(nb) * p.kt_total + i) * kBBytes, kBBytes,
                 &bar_full[st]);
        ++issued;
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&bar_full[i % kStages], (i / kStages) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % kStages;
        if (!mbar_wait(&bar_full[st], (i / kStages) & 1, abort_flag, p.err, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(s_a + st * kABytes);
        const uint32_t b_base = smem_u32(s_b + st * kBBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_i8_ss(tmem, sdesc_kmajor_sw128(a_base + kk * 32), sdesc_kmajor_sw128(b_base + kk * 32), kIdesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_empty[st]);
      }
      mma_commit(&bar_acc);
      mma_commit(&bar_drain);
      volatile int no_abort = 0;
      mbar_wait(&bar_drain, 0, &no_abort, p.err, kDevTimeoutDrain);
    }
  } else {
    const int quad = warp & 3;
    const int64_t mm = m0 + quad * 32 + lane;  // output row of this thread
    const bool row_ok = mm < p.m;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const float pt = (p.pertoken && row_ok) ? p.pertoken[mm] : 1.f;
    bool ready = mbar_wait(&bar_acc, 0, abort_flag, p.err, kDevTimeoutEpilogue);
    ready = __all_sync(0xFFFFFFFFu, ready && !*abort_flag);
    if (ready) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_addr + c0, v);
        tmem_wait_ld();
        const int nc = n0 + c0;
        if (row_ok && nc < p.n) {  // n % 32 == 0, so a 32-column chunk is all in or all out
          int32_t acc[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            acc[j] = static_cast<int32_t>(v[j]);
            if (p.bias) acc[j] = static_cast<int32_t>(static_cast<uint32_t>(acc[j]) + static_cast<uint32_t>(p.bias[nc + j]));
          }
          if (p.raw_acc) {
            int4* dst = reinterpret_cast<int4*>(p.raw_acc + mm * p.n + nc);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_int4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
          }
          uint32_t x3w[16];
          if (p.x3) {
            const uint4* src = reinterpret_cast<const uint4*>(p.x3 + mm * p.n + nc);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 t = src[j];
              x3w[4 * j] = t.x;
              x3w[4 * j + 1] = t.y;
              x3w[4 * j + 2] = t.z;
              x3w[4 * j + 3] = t.w;
            }
          }
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float y[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col = nc + 2 * j + h;
              const float dq = p.dq_bf16 ? act_f32(static_cast<const uint16_t*>(p.dq)[p.dq_per_tensor ? 0 : col], true)
                                         : static_cast<const float*>(p.dq)[p.dq_per_tensor ? 0 : col];
              float t = static_cast<float>(acc[2 * j + h]) * dq * pt;
              if (p.x3) t += act_f32(static_cast<uint16_t>(x3w[j] >> (16 * h)), BF16);
              y[h] = t;
            }
            o[j] = pack2<BF16>(y[0], y[1]);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.out + mm * p.n + nc);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_qmm_gemm(const CUtensorMap& tmap_x1, const QParams& p, cudaStream_t s) {
  const int64_t grid = static_cast<int64_t>(p.num_mb) * p.num_nb;
  if (grid <= 0 || grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  if (p.out_bf16) {
    e = cudaFuncSetAttribute(qmm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    qmm_tc_kernel<true><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, s>>>(tmap_x1, p);
  } else {
    e = cudaFuncSetAttribute(qmm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    qmm_tc_kernel<false><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, s>>>(tmap_x1, p);
  }
  return cudaGetLastError();
}

}  // namespace wqmm
