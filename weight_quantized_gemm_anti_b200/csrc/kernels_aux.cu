// kernels_aux.cu -- weight packing (the device-side counterpart of the
// TransMatmulWeight weight-format conversion), the scale/offset transpose for
// transposed per-group inputs, and the split-K reduction + epilogue.
//
// These kernels are bandwidth-bound elementwise passes: one thread per 16-byte
// output chunk (pack) or per 4 output elements (epilogue), 128-bit stores,
// grids sized in multiples of the SM count by the caller's problem size.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace wqmm {

__device__ uint32_t g_device_error = 0;

// ---------------------------------------------------------------- weight pack
// Read one logical weight element (kk, nn) of x2 as its raw code: int8 / fp8
// byte, the 4-bit two's-complement nibble (even linear index in the low
// nibble), or the 16-bit float16/bfloat16 pattern.  Out-of-range elements read
// as 0.
__device__ __forceinline__ uint32_t read_code(const PackParams& p, int kk, int nn) {
  if (kk >= p.k || nn >= p.n) return 0;
  const int64_t idx = static_cast<int64_t>(kk) * p.s0 + static_cast<int64_t>(nn) * p.s1;
  if (p.wk == kW4) {
    const uint8_t b = p.src[idx >> 1];
    return (idx & 1) ? (b >> 4) : (b & 0xF);
  }
  if (p.wk == kWH) return reinterpret_cast<const uint16_t*>(p.src)[idx];
  return p.src[idx];
}

// Anti-quant GEMM tiling.  int4 chunk (32 k values k0..k0+31): word w holds
// k0+8w .. k0+8w+7, nibble j (j < 4) = k0+8w+2j, nibble j+4 = k0+8w+2j+1, each
// stored biased as (q + 8) so a nibble pair ORed into a 0x4300 (bf16 128.0) /
// 0x6400 (f16 1024.0) exponent pattern gives 128+q+8 / 1024+q+8 exactly.
// int8 chunk (16 k values): byte b = k0 + b, stored biased as (q + 128).
// fp8 chunk: byte b = k0 + b, raw e4m3 code.
// 16-bit chunk (8 k values): half-word h = k0 + h, the value's own bits.
__global__ void pack_wq_kernel(PackParams p, int64_t total_chunks) {
  const int chunks_per_row = wq_chunks_per_col(p.wk);
  const int vals_per_chunk = kWqKTile / chunks_per_row;
  const int kt_total = (p.k + kWqKTile - 1) / kWqKTile;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total_chunks;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = g / (chunks_per_row * kWqNBlock);
    const int within = static_cast<int>(g % (chunks_per_row * kWqNBlock));
    const int c = within / kWqNBlock;
    const int r = within % kWqNBlock;
    const int nb = static_cast<int>(tile / kt_total);
    const int kt = static_cast<int>(tile % kt_total);
    const int nn = nb * kWqNBlock + r;
    const int k0 = kt * kWqKTile + c * vals_per_chunk;
    uint32_t words[4];
    if (p.wk == kW4) {
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
        for (int j = 0; j < 4; ++j) {
          const uint32_t lo = (read_code(p, k0 + 8 * w + 2 * j, nn) ^ 8) & 0xF;
          const uint32_t hi = (read_code(p, k0 + 8 * w + 2 * j + 1, nn) ^ 8) & 0xF;
          word |= lo << (4 * j);
          word |= hi << (16 + 4 * j);
        }
        words[w] = word;
      }
    } else if (p.wk == kWH) {
      for (int w = 0; w < 4; ++w) words[w] = read_code(p, k0 + 2 * w, nn) | (read_code(p, k0 + 2 * w + 1, nn) << 16);
    } else {
      const uint32_t bias = (p.wk == kW8) ? 0x80u : 0u;
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
        for (int b = 0; b < 4; ++b) word |= ((read_code(p, k0 + 4 * w + b, nn) ^ bias) & 0xFF) << (8 * b);
        words[w] = word;
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(p.dst + tile * wq_tile_bytes(p.wk) + (c * kWqNBlock + r) * 16);
    *dst = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// Int8 GEMM tiling: tile (nb, kt) of 256 rows x 128 k bytes at (nb*KT+kt)*32K;
// 16-byte chunk c of row r at r*128 + ((c ^ (r & 7)) * 16): the order a
// 128-byte-swizzled tensor copy would produce, so one bulk copy stages it.
__global__ void pack_q_kernel(PackParams p, int64_t total_chunks) {
  const int kt_total = (p.k + kQKTile - 1) / kQKTile;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total_chunks;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = g / (8 * kQNBlock);
    const int within = static_cast<int>(g % (8 * kQNBlock));
    const int r = within / 8;
    const int c = within % 8;
    const int nb = static_cast<int>(tile / kt_total);
    const int kt = static_cast<int>(tile % kt_total);
    const int nn = nb * kQNBlock + r;
    const int k0 = kt * kQKTile + c * 16;
    uint32_t words[4];
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
      for (int b = 0; b < 4; ++b) word |= (read_code(p, k0 + 4 * w + b, nn) & 0xFF) << (8 * b);
      words[w] = word;
    }
    uint4* dst = reinterpret_cast<uint4*>(p.dst + tile * kQTileBytes + r * 128 + ((c ^ (r & 7)) * 16));
    *dst = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

static int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_pack(const PackParams& p, cudaStream_t s) {
  if (p.for_qmm) {
    const int64_t nb = (p.n + kQNBlock - 1) / kQNBlock, kt = (p.k + kQKTile - 1) / kQKTile;
    const int64_t total = nb * kt * 8 * kQNBlock;
    pack_q_kernel<<<grid_for(total, 256), 256, 0, s>>>(p, total);
  } else {
    const int64_t nb = (p.n + kWqNBlock - 1) / kWqNBlock, kt = (p.k + kWqKTile - 1) / kWqKTile;
    const int64_t total = nb * kt * wq_chunks_per_col(p.wk) * kWqNBlock;
    pack_wq_kernel<<<grid_for(total, 256), 256, 0, s>>>(p, total);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- transpose
// dst[r][c] = src[c][r]; src is (cols, rows) row-major.  Used to turn a
// transposed per-group scale/offset (stored (n, ng)) into (ng, n).
__global__ void transpose_u16_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int rows,
                                     int cols) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows) tile[i][threadIdx.x] = src[static_cast<int64_t>(c) * rows + r];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (c < cols && r < rows) dst[static_cast<int64_t>(r) * cols + c] = tile[threadIdx.x][i];
  }
}

cudaError_t launch_transpose_u16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  transpose_u16_kernel<<<grid, block, 0, s>>>(src, dst, rows, cols);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- epilogue
__device__ __forceinline__ float act_to_f32(uint16_t v, int bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(v) << 16) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint16_t f32_to_act(float v, int bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

// Offsets that are small integers are folded exactly into the tensor-core
// operand (q + offset is exact in bf16/f16), leaving the scale for the fp32
// epilogue; other offsets take the full dequantisation (scale applied to the
// operand) and an epilogue scale of 1.  Mirrors the choice the GEMM makes.
__device__ __forceinline__ bool small_int_offset(float off) { return off == rintf(off) && fabsf(off) <= 112.f; }

__device__ __forceinline__ float epilogue_scale(const EpiParams& p, int nn) {
  if (p.mode == kPerGroup || p.mode == kNoQuant) return 1.f;
  const int i = (p.mode == kPerTensor) ? 0 : nn;
  const float s = act_to_f32(p.scale[i], p.act_bf16);
  const float o = p.offset ? act_to_f32(p.offset[i], p.act_bf16) : 0.f;
  return small_int_offset(o) ? s : 1.f;
}

// out[m][n] = sum_s partial[s][m][n] * epi_scale[n] + bias[n] + x3[m][n];
// splits == 0 gives bias + x3 (the empty-k case).  Four columns per thread.
__global__ void epilogue_kernel(EpiParams p) {
  const int nq = p.n / 4;
  const int64_t total = p.m * nq;
  const int64_t plane = p.m * static_cast<int64_t>(p.n);
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = g / nq;
    const int c4 = static_cast<int>(g % nq) * 4;
    const int64_t base = row * p.n + c4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sp = 0; sp < p.splits; ++sp) {
      const float4 v = *reinterpret_cast<const float4*>(p.partial + sp * plane + base);
      acc[0] += v.x;
      acc[1] += v.y;
      acc[2] += v.z;
      acc[3] += v.w;
    }
    uint16_t o[4];
    for (int j = 0; j < 4; ++j) {
      float v = p.splits ? acc[j] * epilogue_scale(p, c4 + j) : 0.f;
      if (p.bias) v += act_to_f32(p.bias[c4 + j], p.act_bf16);
      if (p.x3) v += act_to_f32(p.x3[base + j], p.act_bf16);
      o[j] = f32_to_act(v, p.act_bf16);
    }
    uint2 packed;
    packed.x = static_cast<uint32_t>(o[0]) | (static_cast<uint32_t>(o[1]) << 16);
    packed.y = static_cast<uint32_t>(o[2]) | (static_cast<uint32_t>(o[3]) << 16);
    *reinterpret_cast<uint2*>(p.out + base) = packed;
  }
}

cudaError_t launch_wqmm_epilogue(const EpiParams& p, cudaStream_t s) {
  const int64_t total = p.m * (p.n / 4);
  epilogue_kernel<<<grid_for(total, 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

uint32_t* device_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(ptr);
}

}  // namespace wqmm
