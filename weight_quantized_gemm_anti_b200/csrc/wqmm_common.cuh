// wqmm_common.cuh -- device helpers shared by the anti-quant GEMM kernels:
// activation-type conversions, the exact dequantisation of int4 / int8 /
// fp8-e4m3 weight chunks into bf16x2 / f16x2 operand registers, per-group
// scale/offset row tracking, and the persistent-CTA work walk (whole tiles,
// then stream-K parts of split tiles).  Included by each kernel translation
// unit; everything here is internal to that unit.
//
// Dequantisation ("计算公式" of the aclnnWeightQuantMatmulAllReduce guide:
// w = (x2 + antiquantOffset) * antiquantScale), per element pair:
//   int4, integer offsets (warp-uniform test): t = 0x4300|nibble (= 128+q+8)
//       then v = t + (off - 136), exact; per-group w = v * s (one rounding);
//       per-tensor/per-channel w = v and the scale is applied to the fp32
//       accumulator in the epilogue.
//   int8: built exactly in fp32 from 0x4B000000|byte (bf16) or exactly in
//       f16x2 from 0x6400|byte (f16), same split of the scale.
//   fp8-e4m3: converted exactly, scale in the epilogue.
//   other offsets: fp32 path, w = round((q + off) * s), epilogue scale 1.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace wqmm {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ float act_f32(uint16_t v, bool bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(v) << 16) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint16_t f32_act(float v, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

// Offsets that are small integers fold exactly into the operand: q + off is an
// integer of magnitude < 256, exact in bf16 and f16.
__device__ __forceinline__ bool small_int(float off) { return off == rintf(off) && fabsf(off) <= 112.f; }

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

__device__ __forceinline__ uint32_t splat_bits(uint16_t b) {
  return static_cast<uint32_t>(b) | (static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------- int4
// 16-byte chunk = 32 k values -> 16 operand registers (k pairs).
// Exact integer path: v = (0x4300|nibble pair) + c2, optionally * s2.
template <bool BF16, bool MUL>
__device__ __forceinline__ void dq4_fast(const uint4 ch, uint32_t c2, uint32_t s2, uint32_t* out) {
  const uint32_t words[4] = {ch.x, ch.y, ch.z, ch.w};
  constexpr uint32_t kMagic = BF16 ? 0x43004300u : 0x64006400u;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t t = ((words[w] >> (4 * j)) & 0x000F000Fu) | kMagic;
      uint32_t v = add2<BF16>(t, c2);
      if constexpr (MUL) v = mul2<BF16>(v, s2);
      out[4 * w + j] = v;
    }
  }
}

// General path: w = round((q + off) * s) through fp32.
template <bool BF16>
__device__ __forceinline__ void dq4_general(const uint4 ch, float off, float s, uint32_t* out) {
  const uint32_t words[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t u = (words[w] >> (4 * j)) & 0x000F000Fu;  // two biased nibbles (q + 8)
      const float lo = static_cast<float>(static_cast<int>(u & 0xFu) - 8);
      const float hi = static_cast<float>(static_cast<int>(u >> 16) - 8);
      out[4 * w + j] = pack2<BF16>((lo + off) * s, (hi + off) * s);
    }
  }
}

// ---------------------------------------------------------------- int8
// 16-byte chunk = 16 k values (biased bytes q + 128) -> 8 operand registers.
template <bool BF16, bool MUL>
__device__ __forceinline__ void dq8_fast(const uint4 ch, float off, float s, uint32_t c2, uint32_t s2,
                                         uint32_t* out) {
  const uint32_t words[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v;
      if constexpr (!BF16) {
        // f16: 0x6400 | byte = 1024 + q + 128 exactly; add (off - 1152) exactly.
        const uint32_t t = __byte_perm(words[w], 0x64646464u, h ? 0x7372 : 0x7170);
        v = add2<false>(t, c2);
        if constexpr (MUL) v = mul2<false>(v, s2);
      } else {
        // fp32: 0x4B000000 | byte = 2^23 + q + 128; subtracting (2^23 + 128 - off) is exact.
        const float base = 8388736.f - off;
        const float lo = __uint_as_float(__byte_perm(words[w], 0x4B000000u, h ? 0x7442 : 0x7440)) - base;
        const float hi = __uint_as_float(__byte_perm(words[w], 0x4B000000u, h ? 0x7443 : 0x7441)) - base;
        v = MUL ? pack2<true>(lo * s, hi * s) : pack2<true>(lo, hi);
      }
      out[2 * w + h] = v;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void dq8_general(const uint4 ch, float off, float s, uint32_t* out) {
  const uint32_t words[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float lo = static_cast<float>(static_cast<int>((words[w] >> (16 * h)) & 0xFFu) - 128);
      const float hi = static_cast<float>(static_cast<int>((words[w] >> (16 * h + 8)) & 0xFFu) - 128);
      out[2 * w + h] = pack2<BF16>((lo + off) * s, (hi + off) * s);
    }
  }
}

// ---------------------------------------------------------------- fp8-e4m3
template <bool BF16>
__device__ __forceinline__ void dq_fp8(const uint4 ch, uint32_t* out) {
  const uint32_t words[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((words[w] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      if constexpr (BF16) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        out[2 * w + h] = pack2<true>(f.x, f.y);
      } else {
        out[2 * w + h] = static_cast<uint32_t>(hr.x) | (static_cast<uint32_t>(hr.y) << 16);
      }
    }
  }
}

// ---------------------------------------------------------------- per-group halves
// Half H (32 k values) of a k step in per-group mode, given the raw scale and
// offset bits of this column's group row for that half (0 for a half past k
// or a column past n: those weights become 0).
template <bool BF16, int H>
__device__ __forceinline__ void dq4_group_half(const uint4 ch, uint16_t sb, uint16_t ob, uint32_t* a) {
  const float off = act_f32(ob, BF16);
  if (__all_sync(kFull, small_int(off))) {
    const float c = off - (BF16 ? 136.f : 1032.f);
    dq4_fast<BF16, true>(ch, pack2<BF16>(c, c), splat_bits(sb), a + 16 * H);
  } else {
    dq4_general<BF16>(ch, off, act_f32(sb, BF16), a + 16 * H);
  }
}

template <bool BF16, int H>
__device__ __forceinline__ void dq8_group_half(const uint4 chA, const uint4 chB, uint16_t sb, uint16_t ob,
                                               uint32_t* a) {
  const float s = act_f32(sb, BF16);
  const float off = act_f32(ob, BF16);
  if (__all_sync(kFull, small_int(off))) {
    const float c = off - 1152.f;
    const uint32_t c2 = pack2<BF16>(c, c);
    dq8_fast<BF16, true>(chA, off, s, c2, splat_bits(sb), a + 16 * H);
    dq8_fast<BF16, true>(chB, off, s, c2, splat_bits(sb), a + 16 * H + 8);
  } else {
    dq8_general<BF16>(chA, off, s, a + 16 * H);
    dq8_general<BF16>(chB, off, s, a + 16 * H + 8);
  }
}

// Group row of half index hidx = 2*kt (+1 for the second half): row = hidx / gq,
// gq = G / 32 halves per group.  Advanced without division along a group's
// k steps.
struct GroupRow {
  int row, rem;
  __device__ __forceinline__ void init(int hidx, int gq) {
    row = hidx / gq;
    rem = hidx - row * gq;
  }
  // advance by q * gq + rq halves (q, rq precomputed once: rq < gq)
  __device__ __forceinline__ void advance(int q, int rq, int gq) {
    row += q;
    rem += rq;
    if (rem >= gq) {
      rem -= gq;
      ++row;
    }
  }
};

// Position in a ring of N slots (and its phase parity) of the k steps one
// dequantisation group handles: they are D apart, so the position advances by
// a compile-time stride instead of being recomputed by division.
template <uint32_t N, uint32_t D>
struct Cursor {
  uint32_t i, ph;
  __device__ __forceinline__ void init(uint32_t v) {
    i = v % N;
    ph = (v / N) & 1u;
  }
  __device__ __forceinline__ void adv() {
    uint32_t j = i + D % N;
    ph ^= (D / N) & 1u;
    if (j >= N) {
      j -= N;
      ph ^= 1u;
    }
    i = j;
  }
};

// Scale/offset bits of one column for the NH 32-wide halves of one turn of a
// dequantisation group (NH = 2 SPG), per-group mode.
template <int NH>
struct GroupSOn {
  uint16_t s[NH], o[NH];
  bool one_row;  // warp-uniform: all halves use the same group row and lie inside k
};

template <int NH>
__device__ __forceinline__ GroupSOn<NH> load_group_son(const WqParams& p, int kt, const GroupRow& gr, int gq, int nn,
                                                       bool col_ok) {
  GroupSOn<NH> r;
  int rows[NH];
  int row = gr.row, rem = gr.rem;
  rows[0] = row;
#pragma unroll
  for (int h = 1; h < NH; ++h) {
    if (++rem >= gq) {
      rem -= gq;
      ++row;
    }
    rows[h] = row;
  }
  r.one_row = rows[NH - 1] == rows[0] && kt * kWqKTile + 32 * (NH - 1) < p.k;
  // every half loads (predicated, no branch): loads behind a branch issue late
  // and their latency shows
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const bool use = col_ok && (kt * kWqKTile + 32 * h < p.k);
    const int64_t idx = static_cast<int64_t>(rows[h]) * p.n + nn;
    r.s[h] = use ? __ldg(p.scale + idx) : uint16_t(0);
    r.o[h] = (use && p.offset) ? __ldg(p.offset + idx) : uint16_t(0);
  }
  return r;
}

// ---------------------------------------------------------------- schedule
struct Item {
  int tile, kt0, kt1, slot;  // slot < 0: whole tile, write the output
  int nadd;                  // > 0: this CTA finishes a split tile: add the partials of
                             // slots 1 .. nadd (the other owners), write the output
};

// Identical walk of this CTA's work in every role.
// The CTA's work items in order.  Whole tiles: tile = blockIdx.x, + grid, ...
// (all tiles without stream-K; the first dp_tiles with it).  Stream-K: then
// the CTA's even share of the k steps of the remaining tiles, cut at tile
// boundaries; an item that is a part of a tile shared with other CTAs gets its
// slot among the tile's owners (its fp32 partial goes to the fix-up kernel, or,
// in inline mode, to the first owner, which adds them all and writes the
// output); a tile the CTA owns alone is an ordinary whole tile (slot -1).
struct Walker {
  int64_t dcur, dend, step;  // whole tiles
  int64_t cur, end, T;       // stream-K range, in k steps from the first split tile; T in units
  // pair: both CTAs of a pair walk the same pair tiles (no stream-K then)
  __device__ __forceinline__ void init(const WqParams& p, bool pair) {
    dcur = pair ? (blockIdx.x >> 1) : blockIdx.x;
    step = pair ? (gridDim.x >> 1) : gridDim.x;
    if (p.stream_k) {
      dend = p.dp_tiles;
      T = static_cast<int64_t>(p.num_tiles - p.dp_tiles) * p.kt_total / p.sk_unit;
      const bool in_sk = static_cast<int>(blockIdx.x) < p.sk_grid;
      cur = in_sk ? sk_start(blockIdx.x, T, p.sk_grid) * p.sk_unit : 0;
      end = in_sk ? sk_start(blockIdx.x + 1, T, p.sk_grid) * p.sk_unit : 0;
    } else {
      dend = p.num_tiles;
      T = cur = end = 0;
    }
  }
  __device__ __forceinline__ bool next(const WqParams& p, Item& it) {
    if (dcur < dend) {
      it.tile = static_cast<int>(dcur);
      it.kt0 = 0;
      it.kt1 = p.kt_total;
      it.slot = -1;
      it.nadd = 0;
      dcur += step;
      return true;
    }
    if (cur >= end) return false;
    const int64_t r = cur / p.kt_total;  // split tile index
    const int64_t tile_end = (r + 1) * p.kt_total;
    const int64_t e = end < tile_end ? end : tile_end;
    it.tile = static_cast<int>(p.dp_tiles + r);
    it.kt0 = static_cast<int>(cur - r * p.kt_total);
    it.kt1 = it.kt0 + static_cast<int>(e - cur);
    const SkOwners o = sk_tile_owners(r, p.kt_total, p.sk_unit, T, p.sk_grid);
    it.slot = (o.first == o.last) ? -1 : static_cast<int>(blockIdx.x - o.first);
    // The first owner reaches its part (the tile's first k steps) last of all
    // its items, after the others have written theirs at the start of theirs.
    it.nadd = (p.sk_inline && it.slot == 0) ? static_cast<int>(o.last - o.first) : 0;
    cur = e;
    return true;
  }
};

// Per-column constants of per-tensor / per-channel modes for one tile.
struct ColConst {
  float s, off;
  uint32_t c2;
  bool fast;  // warp-uniform: every column of this warp has a small-integer offset
};

template <bool BF16, int WK>
__device__ __forceinline__ ColConst col_const(const WqParams& p, int nn, bool col_ok) {
  ColConst c;
  if constexpr (WK == kWH) {  // non-quantised: no scale, no offset
    c.s = 1.f;
    c.off = 0.f;
    c.c2 = 0u;
    c.fast = true;
    return c;
  }
  const int idx = (p.mode == kPerTensor) ? 0 : (col_ok ? nn : 0);
  c.s = act_f32(p.scale[idx], BF16);
  c.off = p.offset ? act_f32(p.offset[idx], BF16) : 0.f;
  c.fast = __all_sync(kFull, small_int(c.off));
  const float magic = (WK == kW4) ? (BF16 ? 136.f : 1032.f) : (BF16 ? 0.f : 1152.f);
  c.c2 = pack2<BF16>(c.off - magic, c.off - magic);
  return c;
}

}  // namespace
}  // namespace wqmm
