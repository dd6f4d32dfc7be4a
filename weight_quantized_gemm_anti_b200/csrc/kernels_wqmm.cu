// kernels_wqmm.cu -- anti-quant weight GEMM on the sm_100a tensor cores.
//
// Computes, per aclnnWeightQuantMatmulAllReduce "计算公式",
//     out = x1 @ ((x2 + antiquantOffset) * antiquantScale) + bias + x3
// as the transposed product  out^T = W^T x1^T  so that the dequantised weight
// is the tcgen05 A operand held in tensor memory and x1 is the B operand in
// shared memory:
//
//   * one CTA owns a tile of 128 weight columns (n) x BN activation rows (m);
//     its accumulator D^T (128 lanes = n, BN columns = m, fp32) lives in TMEM;
//   * warp 0 (one thread) streams, per 64-wide k step, the x1 tile (2-D tensor
//     copy, 128-byte swizzle), the packed weight tile (one 1-D bulk copy) and,
//     in per-group mode, the two scale/offset rows it needs, into a STAGES-deep
//     shared-memory ring;
//   * warps 2..5 (one per TMEM lane quadrant; thread = weight column n) unpack
//     their column's 64 weights, dequantise them in registers and write them
//     with tcgen05.st into one of four TMEM A stages;
//   * warp 1 (one thread) issues four tcgen05.mma kind::f16 (M=128, N=BN, K=16)
//     per k step, A from TMEM and B from shared memory, and releases the
//     shared-memory and TMEM stages with tcgen05.commit;
//   * after the last k step warps 2..5 read the accumulator back with
//     tcgen05.ld and apply the epilogue (scale, + bias, + x3, round) -- or
//     store fp32 split-K partials that a second kernel reduces in fixed order.
//
// Dequantisation (per element pair, bf16x2 / f16x2 registers):
//   int4, integer offset:   t = 0x4300|nibble (=128+q+8, exact); v = t + (off-136)
//                            (exact); per-group w = v * s (one rounding);
//                            per-tensor/channel w = v, scale applied in fp32 later.
//   int8: built exactly in fp32 (0x4B000000|byte trick), same split.
//   fp8-e4m3: converted exactly; scale applied in fp32 in the epilogue.
//   Non-integer offsets take an fp32 path: w = round((q + off) * s).
// No cluster multicast; every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace wqmm {

namespace {

constexpr int kThreads = 192;
constexpr int kAStages = 4;
constexpr int kSoBytes = 1024;  // per stage: 2 half-steps x (scale, offset) x 128 x 2 B

template <int BN>
struct Cfg {
  static constexpr int kStages = BN >= 256 ? 5 : (BN >= 128 ? 7 : 10);
  static constexpr int kX1Bytes = BN * 128;
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr int kTmemNeed = kAccCols + kAStages * 32;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  template <int WK>
  static constexpr int smem_bytes() {
    return kStages * (kX1Bytes + wq_tile_bytes(WK) + kSoBytes) + 1024;
  }
};

__device__ __forceinline__ float act_f32(uint16_t v, bool bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(v) << 16) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint16_t f32_act(float v, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ bool small_int(float off) { return off == rintf(off) && fabsf(off) <= 112.f; }

// Pack two fp32 into a bf16x2 / f16x2 register, round to nearest even; `lo`
// lands in bits 0..15.
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
__device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (BF16)
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <bool BF16>
__device__ __forceinline__ uint32_t mul2(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (BF16)
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <bool BF16>
__device__ __forceinline__ uint32_t splat(float v) {
  return pack2<BF16>(v, v);
}

// Per-half-step dequantisation constants for one weight column.
struct DqConst {
  uint32_t c2;     // (offset - magic) splatted, exact (integer path)
  uint32_t s2;     // scale splatted (per-group integer path)
  float off, s;    // fp32 values (general path)
  bool fast;       // integer offset: exact add path
  bool apply_s;    // multiply by the scale in the operand (per-group or non-integer offset)
};

template <bool BF16, int WK>
__device__ __forceinline__ DqConst make_const(float s, float off, bool per_group) {
  DqConst c;
  c.off = off;
  c.s = s;
  c.fast = small_int(off);
  c.apply_s = per_group || !c.fast;
  // int4 magic: bf16 0x4300 = 128, f16 0x6400 = 1024; stored nibble = q + 8.
  const float magic = (WK == kW4) ? (BF16 ? 136.f : 1032.f) : (BF16 ? 0.f : 1152.f);
  c.c2 = splat<BF16>(off - magic);
  c.s2 = splat<BF16>(s);
  return c;
}

// Dequantise the 32 k values of one 16-byte int4 chunk into 16 operand registers.
template <bool BF16>
__device__ __forceinline__ void dq_int4(const uint4 chunk, const DqConst& c, uint32_t* out) {
  const uint32_t words[4] = {chunk.x, chunk.y, chunk.z, chunk.w};
  const uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t t = ((words[w] >> (4 * j)) & 0x000F000Fu) | magic;
      uint32_t v;
      if (c.fast) {
        v = add2<BF16>(t, c.c2);
        if (c.apply_s) v = mul2<BF16>(v, c.s2);
      } else {
        float lo, hi;
        if constexpr (BF16) {
          lo = __uint_as_float(t << 16) - 136.f;
          hi = __uint_as_float(t & 0xFFFF0000u) - 136.f;
        } else {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&t));
          lo = f.x - 1032.f;
          hi = f.y - 1032.f;
        }
        v = pack2<BF16>((lo + c.off) * c.s, (hi + c.off) * c.s);
      }
      out[4 * w + j] = v;
    }
  }
}

// Dequantise the 16 k values of one 16-byte int8 chunk into 8 operand registers.
template <bool BF16>
__device__ __forceinline__ void dq_int8(const uint4 chunk, const DqConst& c, uint32_t* out) {
  const uint32_t words[4] = {chunk.x, chunk.y, chunk.z, chunk.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v;
      if (!BF16 && c.fast) {
        // f16: 0x6400 | byte = 1024 + (q + 128); add (off - 1152) exactly.
        const uint32_t t = __byte_perm(words[w], 0x64646464u, h ? 0x7372 : 0x7170);
        v = add2<false>(t, c.c2);
        if (c.apply_s) v = mul2<false>(v, c.s2);
      } else {
        // fp32: 0x4B000000 | byte = 2^23 + q + 128, exact.
        const float lo = __uint_as_float(0x4B000000u | ((words[w] >> (16 * h)) & 0xFFu)) - 8388736.f;
        const float hi = __uint_as_float(0x4B000000u | ((words[w] >> (16 * h + 8)) & 0xFFu)) - 8388736.f;
        if (c.apply_s)
          v = pack2<BF16>((lo + c.off) * c.s, (hi + c.off) * c.s);
        else
          v = pack2<BF16>(lo + c.off, hi + c.off);
      }
      out[2 * w + h] = v;
    }
  }
}

// Convert the 16 fp8-e4m3 values of one chunk exactly (no offset, scale later).
template <bool BF16>
__device__ __forceinline__ void dq_fp8(const uint4 chunk, uint32_t* out) {
  const uint32_t words[4] = {chunk.x, chunk.y, chunk.z, chunk.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((words[w] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      uint32_t v;
      if constexpr (BF16) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        v = pack2<true>(f.x, f.y);
      } else {
        v = static_cast<uint32_t>(hr.x) | (static_cast<uint32_t>(hr.y) << 16);
      }
      out[2 * w + h] = v;
    }
  }
}

template <int BN, int WK, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    wqmm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x1, const WqParams p) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr int kTile = wq_tile_bytes(WK);
  constexpr uint32_t kIdesc = idesc_make(1u, BF16 ? 1u : 0u, 128u, static_cast<uint32_t>(BN));
  constexpr uint32_t kAccCol = 0;
  constexpr uint32_t kACol0 = C::kAccCols;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_x1 = smem;
  uint8_t* s_w = s_x1 + S * C::kX1Bytes;
  uint8_t* s_so = s_w + S * kTile;

  __shared__ __align__(8) uint64_t bar_full[S];
  __shared__ __align__(8) uint64_t bar_empty[S];
  __shared__ __align__(8) uint64_t bar_afull[kAStages];
  __shared__ __align__(8) uint64_t bar_aempty[kAStages];
  __shared__ __align__(8) uint64_t bar_acc;
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // tile coordinates: split fastest, then n-block, then m-block
  int bid = blockIdx.x;
  const int split = bid % p.splits;
  bid /= p.splits;
  const int nb = bid % p.num_nb;
  const int mb = bid / p.num_nb;
  const int kt_begin = static_cast<int>((static_cast<int64_t>(split) * p.kt_total) / p.splits);
  const int kt_end = static_cast<int>((static_cast<int64_t>(split + 1) * p.kt_total) / p.splits);
  const int n_iter = kt_end - kt_begin;
  const int n0 = nb * kWqNBlock;
  const int64_t m0 = static_cast<int64_t>(mb) * BN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 4 + 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&bar_afull[i], 4);
      mbar_init(&bar_aempty[i], 1);
    }
    mbar_init(&bar_acc, 1);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmap_x1);
      const bool grp = (p.mode == kPerGroup);
      int issued = 0;
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % S;
        const uint32_t ph = (i / S) & 1;
        if (!mbar_wait(&bar_empty[st], ph ^ 1, abort_flag, p.err, kDevTimeoutProducer)) break;
        const int kt = kt_begin + i;
        // scale/offset rows of the two 32-wide half-steps (per-group only)
        int grow[2] = {-1, -1};
        uint32_t so_bytes = 0;
        const int ncols = min(kWqNBlock, p.n - n0);
        if (grp) {
          for (int h = 0; h < 2; ++h) {
            const int kk = kt * kWqKTile + 32 * h;
            if (kk < p.k) grow[h] = kk / p.group_size;
          }
          for (int h = 0; h < 2; ++h)
            if (grow[h] >= 0) so_bytes += static_cast<uint32_t>(ncols) * 2u * (p.offset ? 2u : 1u);
        }
        mbar_arrive_expect_tx(&bar_full[st], static_cast<uint32_t>(C::kX1Bytes + kTile) + so_bytes);
        tma_load_2d(s_x1 + st * C::kX1Bytes, &tmap_x1, &bar_full[st], kt * kWqKTile, static_cast<int32_t>(m0));
        bulk_g2s(s_w + st * kTile,
                 p.wpack + (static_cast<int64_t>(nb) * p.kt_total + kt) * kTile, kTile, &bar_full[st]);
        if (grp) {
          uint8_t* so = s_so + st * kSoBytes;
          for (int h = 0; h < 2; ++h) {
            if (grow[h] < 0) continue;
            const uint16_t* srow = p.scale + static_cast<int64_t>(grow[h]) * p.n + n0;
            bulk_g2s(so + h * 512, srow, ncols * 2, &bar_full[st]);
            if (p.offset) {
              const uint16_t* orow = p.offset + static_cast<int64_t>(grow[h]) * p.n + n0;
              bulk_g2s(so + h * 512 + 256, orow, ncols * 2, &bar_full[st]);
            }
          }
        }
        ++issued;
      }
      // drain: wait until every copy issued into the ring has landed
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&bar_full[i % S], (i / S) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % S;
        const int as = i % kAStages;
        if (!mbar_wait(&bar_full[st], (i / S) & 1, abort_flag, p.err, kDevTimeoutMma)) break;
        if (!mbar_wait(&bar_afull[as], (i / kAStages) & 1, abort_flag, p.err, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t b_base = smem_u32(s_x1 + st * C::kX1Bytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bdesc = sdesc_kmajor_sw128(b_base + kk * 32);
          const uint32_t a_tmem = tmem + kACol0 + as * 32 + kk * 8;
          mma_f16_ts(tmem + kAccCol, a_tmem, bdesc, kIdesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_empty[st]);
        mma_commit(&bar_aempty[as]);
      }
      mma_commit(&bar_acc);
      // wait for every MMA this thread issued before the TMEM is released
      mma_commit(&bar_drain);
      volatile int no_abort = 0;
      mbar_wait(&bar_drain, 0, &no_abort, p.err, kDevTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int quad = warp & 3;                       // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;                  // row of the 128-column weight block
    const int nn = n0 + r;
    const bool col_ok = nn < p.n;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    // per-tensor / per-channel constants, fixed for the whole tile
    DqConst cst{};
    if (p.mode != kPerGroup) {
      const int idx = (p.mode == kPerTensor) ? 0 : (col_ok ? nn : 0);
      const float s = act_f32(p.scale[idx], BF16);
      const float off = p.offset ? act_f32(p.offset[idx], BF16) : 0.f;
      cst = make_const<BF16, WK>(s, off, false);
    }
    bool ok = true;
    for (int i = 0; i < n_iter && ok; ++i) {
      const int st = i % S;
      const int as = i % kAStages;
      bool got = mbar_wait(&bar_full[st], (i / S) & 1, abort_flag, p.err, kDevTimeoutDequant);
      got = got && mbar_wait(&bar_aempty[as], ((i / kAStages) & 1) ^ 1, abort_flag, p.err, kDevTimeoutDequant);
      // tcgen05.st below is warp-collective: proceed only if every lane's wait succeeded
      if (!__all_sync(0xFFFFFFFFu, got)) {
        ok = false;
        break;
      }
      const uint8_t* wt = s_w + st * kTile;
      const int kbase = (kt_begin + i) * kWqKTile;
      uint32_t a[32];
      if constexpr (WK == kW4) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          DqConst c = cst;
          if (p.mode == kPerGroup) {
            // a half-step past k has no scale/offset row staged: its weights become 0
            const bool use = col_ok && (kbase + 32 * h < p.k);
            const uint8_t* so = s_so + st * kSoBytes + h * 512;
            const float s = use ? act_f32(reinterpret_cast<const uint16_t*>(so)[r], BF16) : 0.f;
            const float off =
                (p.offset && use) ? act_f32(reinterpret_cast<const uint16_t*>(so + 256)[r], BF16) : 0.f;
            c = make_const<BF16, WK>(s, off, true);
          }
          const uint4 chunk = *reinterpret_cast<const uint4*>(wt + (h * kWqNBlock + r) * 16);
          dq_int4<BF16>(chunk, c, a + 16 * h);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 chunk = *reinterpret_cast<const uint4*>(wt + (q * kWqNBlock + r) * 16);
          if constexpr (WK == kWFp8) {
            dq_fp8<BF16>(chunk, a + 8 * q);
          } else {
            DqConst c = cst;
            if (p.mode == kPerGroup) {
              const bool use = col_ok && (kbase + 32 * (q >> 1) < p.k);
              const uint8_t* so = s_so + st * kSoBytes + (q >> 1) * 512;
              const float s = use ? act_f32(reinterpret_cast<const uint16_t*>(so)[r], BF16) : 0.f;
              const float off =
                  (p.offset && use) ? act_f32(reinterpret_cast<const uint16_t*>(so + 256)[r], BF16) : 0.f;
              c = make_const<BF16, WK>(s, off, true);
            }
            dq_int8<BF16>(chunk, c, a + 8 * q);
          }
        }
      }
      tmem_st_x32(tmem + lane_addr + kACol0 + as * 32, a);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_afull[as]);
        mbar_arrive(&bar_empty[st]);
      }
    }
    // epilogue: wait for the accumulator (warp-uniform outcome before tcgen05.ld)
    bool acc_ready = ok && n_iter > 0 && mbar_wait(&bar_acc, 0, abort_flag, p.err, kDevTimeoutEpilogue);
    acc_ready = __all_sync(0xFFFFFFFFu, acc_ready && !*abort_flag);
    if (acc_ready) {
      tc_fence_after();
      float escale = 1.f;
      if (p.mode != kPerGroup && WK != kWFp8) escale = cst.apply_s ? 1.f : cst.s;
      if (WK == kWFp8) escale = cst.s;
      const float bias_v = (p.bias && col_ok && p.splits == 1) ? act_f32(p.bias[nn], BF16) : 0.f;
      constexpr int kChunk = BN < 32 ? BN : 32;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += kChunk) {
        uint32_t v[32];
        if constexpr (kChunk == 32)
          tmem_ld_x32(tmem + lane_addr + kAccCol + c0, v);
        else
          tmem_ld_x16(tmem + lane_addr + kAccCol + c0, v);
        tmem_wait_ld();
        if (col_ok) {
#pragma unroll
          for (int j = 0; j < kChunk; ++j) {
            const int64_t mm = m0 + c0 + j;
            if (mm < p.m) {
              const float acc = __uint_as_float(v[j]);
              if (p.splits == 1) {
                float y = acc * escale + bias_v;
                if (p.x3) y += act_f32(p.x3[mm * p.n + nn], BF16);
                p.out[mm * p.n + nn] = f32_act(y, BF16);
              } else {
                p.partial[(static_cast<int64_t>(split) * p.m + mm) * p.n + nn] = acc;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int WK, bool BF16>
cudaError_t launch_one(const CUtensorMap& tmap, const WqParams& p, cudaStream_t s) {
  constexpr int smem = Cfg<BN>::template smem_bytes<WK>();
  auto kern = wqmm_tc_kernel<BN, WK, BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(p.num_mb) * p.num_nb * p.splits;
  if (grid <= 0 || grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(tmap, p);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& tmap, const WqParams& p, int wk, bool bf16, cudaStream_t s) {
  if (wk == kW4) return bf16 ? launch_one<BN, kW4, true>(tmap, p, s) : launch_one<BN, kW4, false>(tmap, p, s);
  if (wk == kW8) return bf16 ? launch_one<BN, kW8, true>(tmap, p, s) : launch_one<BN, kW8, false>(tmap, p, s);
  return bf16 ? launch_one<BN, kWFp8, true>(tmap, p, s) : launch_one<BN, kWFp8, false>(tmap, p, s);
}

}  // namespace

cudaError_t launch_wqmm_gemm(const CUtensorMap& tmap_x1, const WqParams& p, int bn, int wk, bool act_bf16,
                             cudaStream_t s) {
  switch (bn) {
    case 16: return launch_bn<16>(tmap_x1, p, wk, act_bf16, s);
    case 32: return launch_bn<32>(tmap_x1, p, wk, act_bf16, s);
    case 64: return launch_bn<64>(tmap_x1, p, wk, act_bf16, s);
    case 128: return launch_bn<128>(tmap_x1, p, wk, act_bf16, s);
    case 256: return launch_bn<256>(tmap_x1, p, wk, act_bf16, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wqmm
