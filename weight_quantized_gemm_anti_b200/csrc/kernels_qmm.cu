// kernels_qmm.cu -- int8 x int8 GEMM on the sm_100a tensor cores, after
// aclnnQuantMatmulAllReduceV2 ("Function", cases 1 and 2):
//     out = dequantScale * pertokenScale * (x1_int8 @ x2_int8 + bias_int32) + x3
//
// A persistent, warp-specialised kernel, one CTA per SM, output tiles of
// 128 (m) x 256 (n) dealt round-robin to the CTAs:
//   warp 0      x1 producer: per 128-byte k step, the x1 tile (2-D tensor copy,
//               128-byte swizzle) into a 4-deep ring;
//   warp 6      weight producer: the packed weight tile -- already stored in
//               that swizzled order by the packing kernel -- as one 32 KB bulk
//               copy into the same ring (a copy holds its issuing thread for
//               hundreds of cycles, so the two streams have their own warps);
//   warp 1      MMA issuer: four tcgen05.mma kind::i8 (M=128, N=256, K=32) per
//               k step, both operands from shared memory, int32 accumulators in
//               TMEM, two buffers of 256 columns so that the epilogue of one
//               tile overlaps the main loop of the next; the whole warp walks
//               the loop and one elected lane issues;
//   warps 2..5  epilogue (thread = output row): tcgen05.ld of the accumulator,
//               (acc + bias) * dq[n] * pt[m] + x3 in fp32, one rounding to
//               bf16/f16, 16-byte vector stores; optionally the raw int32
//               accumulator (+ bias) for bit-exact testing.
// The int32 sum of x1*x2 products is exact (|sum| < 2^31 for k <= 65535 with
// the bias added in two's complement, as a 32-bit accumulator does).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace wqmm {

namespace {

constexpr int kThreads = 224;
constexpr int kStages = 4;
constexpr int kBM = 128;
constexpr int kBN = kQNBlock;       // 256
constexpr int kABytes = kBM * 128;  // 16 KB
constexpr int kBBytes = kQTileBytes;
constexpr int kNAcc = 2;
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = kStages * (kABytes + kBBytes) + 1024;
constexpr unsigned kFullMask = 0xFFFFFFFFu;

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

  __shared__ __align__(8) uint64_t bar_afull[kStages];  // x1 tile landed
  __shared__ __align__(8) uint64_t bar_bfull[kStages];  // weight tile landed
  __shared__ __align__(8) uint64_t bar_empty[kStages];  // both read by the MMA
  __shared__ __align__(8) uint64_t bar_accfull[kNAcc];
  __shared__ __align__(8) uint64_t bar_accempty[kNAcc];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.num_mb * p.num_nb;
  const int n_iter = p.kt_total;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_afull[i], 1);
      mbar_init(&bar_bfull[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < kNAcc; ++i) {
      mbar_init(&bar_accfull[i], 1);
      mbar_init(&bar_accempty[i], 4);
    }
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

  if (warp == 0 || warp == 6) {
    // ---------------------------------------------------------------- producers
    const bool is_a = (warp == 0);
    if (is_a && elect_one()) prefetch_tensormap(&tmap_x1);
    __syncwarp();
    uint32_t g = 0;  // k step counter over this CTA's tiles
    bool live = true;
    for (int t = blockIdx.x; t < num_tiles && live; t += gridDim.x) {
      const int nb = t % p.num_nb;
      const int32_t m0 = static_cast<int32_t>(static_cast<int64_t>(t / p.num_nb) * kBM);
      for (int i = 0; i < n_iter; ++i, ++g) {
        const int st = g % kStages;
        const bool ok = mbar_wait(&bar_empty[st], ((g / kStages) & 1) ^ 1, abort_flag, p.err, kDevTimeoutProducer);
        if (!__all_sync(kFullMask, ok)) {
          live = false;
          break;
        }
        if (elect_one()) {
          if (is_a) {
            mbar_arrive_expect_tx(&bar_afull[st], kABytes);
            tma_load_2d(s_a + st * kABytes, &tmap_x1, &bar_afull[st], i * kQKTile, m0);
          } else {
            mbar_arrive_expect_tx(&bar_bfull[st], kBBytes);
            bulk_g2s(s_b + st * kBBytes, p.wpack + (static_cast<int64_t>(nb) * p.kt_total + i) * kBBytes, kBBytes,
                     &bar_bfull[st]);
          }
        }
        __syncwarp();
      }
    }
    // every copy issued has landed before the CTA may exit
    if (lane == 0) {
      uint64_t* full = is_a ? bar_afull : bar_bfull;
      for (uint32_t i = (g > kStages ? g - kStages : 0); i < g; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&full[i % kStages], (i / kStages) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint64_t adesc0 = sdesc_kmajor_sw128(smem_u32(s_a));
    const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(s_b));
    uint32_t g = 0, j = 0;
    bool live = true;
    for (int t = blockIdx.x; t < num_tiles && live; t += gridDim.x, ++j) {
      const int ab = j % kNAcc;
      if (!__all_sync(kFullMask, mbar_wait(&bar_accempty[ab], ((j / kNAcc) & 1) ^ 1, abort_flag, p.err,
                                           kDevTimeoutMma)))
        break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + ab * kBN;
      for (int i = 0; i < n_iter; ++i, ++g) {
        const int st = g % kStages;
        const uint32_t ph = (g / kStages) & 1;
        const bool ok = mbar_wait(&bar_afull[st], ph, abort_flag, p.err, kDevTimeoutMma) &&
                        mbar_wait(&bar_bfull[st], ph, abort_flag, p.err, kDevTimeoutMma);
        if (!__all_sync(kFullMask, ok)) {
          live = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = adesc0 + static_cast<uint64_t>(st) * (kABytes >> 4);
        const uint64_t bd = bdesc0 + static_cast<uint64_t>(st) * (kBBytes >> 4);
        const uint32_t acc0 = i > 0 ? 1u : 0u;
        if (elect_one()) {
          mma_i8_ss(d_tmem, ad, bd, kIdesc, acc0);
          mma_i8_ss(d_tmem, ad + 2, bd + 2, kIdesc, 1u);
          mma_i8_ss(d_tmem, ad + 4, bd + 4, kIdesc, 1u);
          mma_i8_ss(d_tmem, ad + 6, bd + 6, kIdesc, 1u);
          mma_commit(&bar_empty[st]);
        }
        __syncwarp();
      }
      if (!live) break;
      if (elect_one()) mma_commit(&bar_accfull[ab]);
      __syncwarp();
    }
    if (elect_one()) {
      mma_commit(&bar_drain);
      volatile int no_abort = 0;
      mbar_wait(&bar_drain, 0, &no_abort, p.err, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t j = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++j) {
      const int ab = j % kNAcc;
      const int nb = t % p.num_nb;
      const int64_t m0 = static_cast<int64_t>(t / p.num_nb) * kBM;
      const int n0 = nb * kBN;
      const int64_t mm = m0 + quad * 32 + lane;  // output row of this thread
      const bool row_ok = mm < p.m;
      const float pt = (p.pertoken && row_ok) ? p.pertoken[mm] : 1.f;
      bool ready = mbar_wait_sleep(&bar_accfull[ab], (j / kNAcc) & 1, abort_flag, p.err, kDevTimeoutEpilogue, 64, 512);
      if (!__all_sync(kFullMask, ready && !*abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_addr + ab * kBN + c0, v);
        tmem_wait_ld();
        if (c0 + 32 >= kBN) {
          // the whole accumulator has been read: hand it back to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_accempty[ab]);
        }
        const int nc = n0 + c0;
        if (row_ok && nc < p.n) {  // n % 32 == 0, so a 32-column chunk is all in or all out
          int32_t acc[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            acc[q] = static_cast<int32_t>(v[q]);
            if (p.bias) acc[q] = static_cast<int32_t>(static_cast<uint32_t>(acc[q]) + static_cast<uint32_t>(p.bias[nc + q]));
          }
          if (p.raw_acc) {
            int4* dst = reinterpret_cast<int4*>(p.raw_acc + mm * p.n + nc);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_int4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
          }
          uint32_t x3w[16];
          if (p.x3) {
            const uint4* src = reinterpret_cast<const uint4*>(p.x3 + mm * p.n + nc);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 u = src[q];
              x3w[4 * q] = u.x;
              x3w[4 * q + 1] = u.y;
              x3w[4 * q + 2] = u.z;
              x3w[4 * q + 3] = u.w;
            }
          }
          uint32_t o[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float y[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col = nc + 2 * q + h;
              const float dq = p.dq_bf16 ? act_f32(static_cast<const uint16_t*>(p.dq)[p.dq_per_tensor ? 0 : col], true)
                                         : static_cast<const float*>(p.dq)[p.dq_per_tensor ? 0 : col];
              float u = static_cast<float>(acc[2 * q + h]) * dq * pt;
              if (p.x3) u += act_f32(static_cast<uint16_t>(x3w[q] >> (16 * h)), BF16);
              y[h] = u;
            }
            o[q] = pack2<BF16>(y[0], y[1]);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.out + mm * p.n + nc);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
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
  const int64_t tiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
  if (tiles <= 0 || tiles > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);  // persistent: one CTA per SM
  cudaError_t e;
  if (p.out_bf16) {
    e = cudaFuncSetAttribute(qmm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    qmm_tc_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(tmap_x1, p);
  } else {
    e = cudaFuncSetAttribute(qmm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    qmm_tc_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(tmap_x1, p);
  }
  return cudaGetLastError();
}

}  // namespace wqmm
