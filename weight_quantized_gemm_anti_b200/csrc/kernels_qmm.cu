// kernels_qmm.cu -- int8 x int8 GEMM on the sm_100a tensor cores, after
// aclnnQuantMatmulAllReduceV2 ("Function", cases 1 and 2):
//     out = dequantScale * pertokenScale * (x1_int8 @ x2_int8 + bias_int32) + x3
//
// A persistent, warp-specialised kernel, one CTA per SM, output tiles of
// 128 (m) x 256 (n) dealt round-robin to the CTAs:
//   warp 0      x1 producer: per 128-byte k step, the x1 tile (2-D tensor copy,
//               128-byte swizzle) into the operand ring;
//   warp 6      weight producer: the packed weight tile -- already stored in
//               that swizzled order by the packing kernel -- as one bulk copy
//               into the same ring (a copy holds its issuing thread for
//               hundreds of cycles, so the two streams have their own warps);
//   warp 1      MMA issuer: four tcgen05.mma kind::i8 (M=128, N=256, K=32) per
//               k step, both operands from shared memory, int32 accumulators in
//               TMEM, two buffers of 256 columns so that the epilogue of one
//               tile overlaps the main loop of the next; the whole warp walks
//               the loop and one elected lane issues;
//   warps 2..5  epilogue, each on its own 32 accumulator lanes (= output rows)
//               and independent of the others.  Per 32-column chunk the warp
//               brings that 32 x 32 block of x3 into a 4-deep per-warp ring
//               with 16-byte cp.async copies (three chunks ahead; the tile's
//               x3 is prefetched into L2 while the main loop runs), the thread
//               of each row reads its accumulator row with tcgen05.ld and
//               computes (acc + bias) * dq[n] * pt[m] + x3 in fp32 with one
//               rounding over the x3 block, and the warp writes the block out
//               row-major, 8 whole 64-byte rows per store instruction.  Small
//               tensor copies are not used here: the SM's copy engine takes a
//               few hundred cycles for each 2 KB block, which made a
//               copy-engine epilogue several times slower than the tile's
//               MMAs.  Optionally the raw int32 accumulator (+ bias) is also
//               stored, for bit-exact testing.
// Pair mode (PAIR): clusters of two CTAs share each MMA (cta_group::2, M = 256
// rows of x1, 128 per CTA; each CTA stages only its half of the 256-column
// weight tile, so the ring is six stages deep in the same shared memory).  The
// even CTA issues the MMAs.  Both CTAs' tensor copies complete on the even
// CTA's full barriers (the odd CTA's through the pair form of the copy), so the
// MMA issuer waits on its own barriers only; commits reach both CTAs' empty
// barriers.
// The int32 sum of x1*x2 products is exact (|sum| < 2^31 for k <= 65535 with
// the bias added in two's complement, as a 32-bit accumulator does).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace wqmm {

namespace {

constexpr int kThreads = 224;
constexpr int kBM = 128;
constexpr int kBN = kQNBlock;       // 256
constexpr int kABytes = kBM * 128;  // 16 KB of x1 per k step
constexpr int kBBytes = kQTileBytes;
constexpr int kNAcc = 2;
constexpr int kTmemCols = 512;
constexpr int kMaxStages = 6;
constexpr int kEC = 32;                     // epilogue chunk: columns
constexpr int kChunks = kBN / kEC;          // chunks per tile
constexpr int kEBufs = 4;                   // per-warp ring of 32 x 32 blocks
constexpr int kEBufBytes = 32 * kEC * 2;    // 2 KB, 64-byte rows, 64-byte swizzle
constexpr int kEpiBytes = 4 * kEBufs * kEBufBytes;
constexpr unsigned kFullMask = 0xFFFFFFFFu;

template <bool PAIR>
struct QCfg {
  static constexpr int kStages = PAIR ? 6 : 4;
  static constexpr int kBStage = PAIR ? kBBytes / 2 : kBBytes;  // weight bytes this CTA stages per step
  static constexpr int kSmemBytes = kStages * (kABytes + kBStage) + kEpiBytes + 1024;
  static_assert(kStages <= kMaxStages, "barrier arrays");
  static_assert(kSmemBytes + 512 <= 232448, "shared memory per CTA");
};

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

// Byte offset of the 16-byte unit q (0..3) of row r in a block of 64-byte rows,
// units permuted by row pair (bits 4..5 XOR bits 7..8) so that both the
// thread-per-row and the row-major access of 8 lanes hit distinct banks.
__device__ __forceinline__ uint32_t sw64_offset(uint32_t r, uint32_t q) { return r * 64u + ((q ^ ((r >> 1) & 3u)) << 4); }

// Per-column constants of the 32 output columns from nc: dequant scale and
// int32 bias (warp-wide broadcast vector loads); dq0 / 0 when absent or !ok.
__device__ __forceinline__ void load_chunk_consts(const QParams& p, int nc, bool ok, float dq0, float (&dq)[kEC],
                                                  int32_t (&bs)[kEC]) {
#pragma unroll
  for (int i = 0; i < kEC; ++i) {
    dq[i] = dq0;
    bs[i] = 0;
  }
  if (!ok) return;
  if (!p.dq_per_tensor) {
    if (p.dq_bf16) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dq) + nc);
#pragma unroll
      for (int q = 0; q < kEC / 8; ++q) {
        const uint4 u = __ldg(src + q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          dq[8 * q + 2 * h] = __uint_as_float(w[h] << 16);
          dq[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
        }
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.dq) + nc);
#pragma unroll
      for (int q = 0; q < kEC / 4; ++q) {
        const float4 f = __ldg(src + q);
        dq[4 * q] = f.x;
        dq[4 * q + 1] = f.y;
        dq[4 * q + 2] = f.z;
        dq[4 * q + 3] = f.w;
      }
    }
  }
  if (p.bias) {
    const int4* src = reinterpret_cast<const int4*>(p.bias + nc);
#pragma unroll
    for (int q = 0; q < kEC / 4; ++q) {
      const int4 b = __ldg(src + q);
      bs[4 * q] = b.x;
      bs[4 * q + 1] = b.y;
      bs[4 * q + 2] = b.z;
      bs[4 * q + 3] = b.w;
    }
  }
}

template <bool BF16, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    qmm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x1, const __grid_constant__ CUtensorMap tmap_w,
                  const QParams p) {
  using C = QCfg<PAIR>;
  constexpr int kSt = C::kStages;
  constexpr uint32_t kIdesc = idesc_make(2u, 1u, PAIR ? 2 * kBM : kBM, kBN);
  constexpr int kBLoad = C::kBStage;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;
  uint8_t* s_b = s_a + kSt * kABytes;
  uint8_t* s_e = s_b + kSt * C::kBStage;

  // pair: the even CTA's full barriers count the bytes of both CTAs
  __shared__ __align__(8) uint64_t bar_afull[kMaxStages];  // x1 tile landed
  __shared__ __align__(8) uint64_t bar_bfull[kMaxStages];  // weight tile landed
  __shared__ __align__(8) uint64_t bar_empty[kMaxStages];  // both read by the MMA
  __shared__ __align__(8) uint64_t bar_accfull[kNAcc];
  __shared__ __align__(8) uint64_t bar_accempty[kNAcc];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_iter = p.kt_total;
  // pair: tiles of 256 rows x 256 columns walked by both CTAs of a pair
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool mma_cta = rank == 0;
  const int num_mt = PAIR ? (p.num_mb + 1) / 2 : p.num_mb;
  const int num_tiles = num_mt * p.num_nb;
  const int t_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int t_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  auto row0_of = [&](int t) {  // first x1 row of this CTA's 128 rows of tile t
    return static_cast<int64_t>(t / p.num_nb) * (PAIR ? 2 * kBM : kBM) + static_cast<int64_t>(rank) * kBM;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSt; ++i) {
      mbar_init(&bar_afull[i], 1);
      mbar_init(&bar_bfull[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < kNAcc; ++i) {
      mbar_init(&bar_accfull[i], 1);
      mbar_init(&bar_accempty[i], PAIR ? 8 : 4);
    }
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc2(&tmem_base_sh, kTmemCols);
      tmem_relinquish2();
    } else {
      tmem_alloc(&tmem_base_sh, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the other CTA's barriers are initialised
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0 || warp == 6) {
    // ---------------------------------------------------------------- producers
    const bool is_a = (warp == 0);
    if (elect_one()) prefetch_tensormap(is_a ? &tmap_x1 : &tmap_w);
    __syncwarp();
    // pair: the even CTA's full barriers, which the odd CTA's copies complete
    const uint32_t lead_full = mapa_shared(smem_u32(is_a ? &bar_afull[0] : &bar_bfull[0]), 0u);
    uint32_t g = 0;  // k step counter over this CTA's tiles
    bool live = true;
    for (int t = t_first; t < num_tiles && live; t += t_step) {
      const int nb = t % p.num_nb;
      const int32_t m0 = static_cast<int32_t>(row0_of(t));
      for (int i = 0; i < n_iter; ++i, ++g) {
        const int st = g % kSt;
        const bool ok = mbar_wait(&bar_empty[st], ((g / kSt) & 1) ^ 1, abort_flag, p.err, kDevTimeoutProducer);
        if (!__all_sync(kFullMask, ok)) {
          live = false;
          break;
        }
        if (elect_one()) {
          if constexpr (!PAIR) {
            if (is_a) {
              mbar_arrive_expect_tx(&bar_afull[st], kABytes);
              tma_load_2d(s_a + st * kABytes, &tmap_x1, &bar_afull[st], i * kQKTile, m0);
            } else {
              mbar_arrive_expect_tx(&bar_bfull[st], kBLoad);
              bulk_g2s(s_b + st * kBLoad, p.wpack + (static_cast<int64_t>(nb) * p.kt_total + i) * kBBytes, kBLoad,
                       &bar_bfull[st]);
            }
          } else {
            // x1: this CTA's 128 rows; weight: this CTA's 128 of the tile's 256
            // packed rows (a 2-D view of the packed weight, 128 bytes per row)
            const CUtensorMap* map = is_a ? &tmap_x1 : &tmap_w;
            uint8_t* dst = is_a ? s_a + st * kABytes : s_b + st * kBLoad;
            const int32_t c0 = is_a ? i * kQKTile : 0;
            const int32_t c1 = is_a ? m0 : static_cast<int32_t>((nb * p.kt_total + i) * kBN + rank * (kBN / 2));
            if (mma_cta) {
              uint64_t* bar = is_a ? &bar_afull[st] : &bar_bfull[st];
              mbar_arrive_expect_tx(bar, 2 * (is_a ? kABytes : kBLoad));
              tma_load_2d(dst, map, bar, c0, c1);
            } else {
              tma_load_2d_pair(dst, map, lead_full + st * 8, c0, c1);
            }
          }
        }
        __syncwarp();
      }
    }
    // every copy issued has landed before the CTA may exit (pair: the even
    // CTA's barriers count both CTAs' copies, and the odd CTA stays until the
    // even one has drained them)
    if (lane == 0 && mma_cta) {
      uint64_t* full = is_a ? bar_afull : bar_bfull;
      for (uint32_t i = (g > kSt ? g - kSt : 0); i < g; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&full[i % kSt], (i / kSt) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1 && mma_cta) {
    // ---------------------------------------------------------------- MMA issuer
    const uint64_t adesc0 = sdesc_kmajor_sw128(smem_u32(s_a));
    const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(s_b));
    auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
      if constexpr (PAIR)
        mma_i8_ss2(d, a, b, kIdesc, acc);
      else
        mma_i8_ss(d, a, b, kIdesc, acc);
    };
    auto commit = [&](uint64_t* bar, uint16_t mask) {
      if constexpr (PAIR)
        mma_commit2_mc(bar, mask);
      else
        mma_commit(bar);
    };
    uint32_t g = 0, j = 0;
    bool live = true;
    for (int t = t_first; t < num_tiles && live; t += t_step, ++j) {
      const int ab = j % kNAcc;
      if (!__all_sync(kFullMask, mbar_wait(&bar_accempty[ab], ((j / kNAcc) & 1) ^ 1, abort_flag, p.err,
                                           kDevTimeoutMma)))
        break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + ab * kBN;
      for (int i = 0; i < n_iter; ++i, ++g) {
        const int st = g % kSt;
        const uint32_t ph = (g / kSt) & 1;
        const bool ok = mbar_wait(&bar_afull[st], ph, abort_flag, p.err, kDevTimeoutMma) &&
                        mbar_wait(&bar_bfull[st], ph, abort_flag, p.err, kDevTimeoutMma);
        if (!__all_sync(kFullMask, ok)) {
          live = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = adesc0 + static_cast<uint64_t>(st) * (kABytes >> 4);
        const uint64_t bd = bdesc0 + static_cast<uint64_t>(st) * (kBLoad >> 4);
        const uint32_t acc0 = i > 0 ? 1u : 0u;
        if (elect_one()) {
          mma(d_tmem, ad, bd, acc0);
          mma(d_tmem, ad + 2, bd + 2, 1u);
          mma(d_tmem, ad + 4, bd + 4, 1u);
          mma(d_tmem, ad + 6, bd + 6, 1u);
          commit(&bar_empty[st], 0x3);
        }
        __syncwarp();
      }
      if (!live) break;
      if (elect_one()) commit(&bar_accfull[ab], 0x3);
      __syncwarp();
    }
    if (elect_one()) {
      commit(&bar_drain, 0x1);
      volatile int no_abort = 0;
      mbar_wait(&bar_drain, 0, &no_abort, p.err, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* ebuf = s_e + quad * (kEBufs * kEBufBytes);
    const bool has_x3 = p.x3 != nullptr;
    const int my_tiles = t_first < num_tiles ? (num_tiles - 1 - t_first) / t_step + 1 : 0;
    const int n_chunks = my_tiles * kChunks;
    // Row-major moves of a 32 x 32 block: lane l takes 16-byte unit (l & 3) of
    // rows (l >> 2) + 8 i, so one warp instruction covers 8 whole 64-byte rows.
    const int ur = lane >> 2, uu = lane & 3;
    // chunk c: columns [col, col + 32) of this warp's rows [row, row + 32) of
    // the CTA's tile c / kChunks; it is live when both start inside the output
    // (n is a multiple of 32, so a live chunk's columns are all inside)
    auto chunk_col = [&](int c) { return ((t_first + (c / kChunks) * t_step) % p.num_nb) * kBN + (c % kChunks) * kEC; };
    auto chunk_row = [&](int c) { return row0_of(t_first + (c / kChunks) * t_step) + quad * 32; };
    // Every lane: its units of chunk c's x3 block into ring slot c % kEBufs (rows
    // past m read as zero), then one cp.async group per chunk index, empty when
    // there is nothing to load.
    auto load_x3 = [&](int c) {
      if (has_x3 && c < n_chunks) {
        const int col = chunk_col(c);
        const int64_t row = chunk_row(c);
        if (col < p.n && row < p.m) {
          uint8_t* slot = ebuf + (c % kEBufs) * kEBufBytes;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = ur + 8 * i;
            const bool ok = row + r < p.m;
            const uint16_t* src = p.x3 + (ok ? row + r : row) * p.n + col + 8 * uu;
            cp_async_16(slot + sw64_offset(static_cast<uint32_t>(r), static_cast<uint32_t>(uu)), src, ok ? 16u : 0u);
          }
        }
      }
      cp_async_commit();
    };
    for (int c = 0; c < kEBufs - 1; ++c) load_x3(c);
    const float dq0 = p.dq_bf16 ? act_f32(static_cast<const uint16_t*>(p.dq)[0], true) : static_cast<const float*>(p.dq)[0];
    uint32_t j = 0;
    int c = 0;  // chunk counter over this CTA's tiles
    for (int t = t_first; t < num_tiles; t += t_step, ++j) {
      const int ab = j % kNAcc;
      const int64_t r0 = row0_of(t) + quad * 32;
      const int n0 = (t % p.num_nb) * kBN;
      const int64_t mm = r0 + lane;  // output row of this thread
      const bool row_ok = mm < p.m;
      const bool rows_live = r0 < p.m;
      const float pt = (p.pertoken && row_ok) ? p.pertoken[mm] : 1.f;
      // The first chunk's per-column constants (later ones are loaded a chunk
      // ahead), and this thread's row of the tile's x3 brought into L2: issued
      // before the wait for the accumulator, which they outlast.
      float dq[kEC];
      int32_t bs[kEC];
      load_chunk_consts(p, n0, rows_live && n0 < p.n, dq0, dq, bs);
      if (has_x3 && row_ok) {
        const char* xrow = reinterpret_cast<const char*>(p.x3 + mm * p.n + n0);
        const int bytes = 2 * ((p.n - n0) < kBN ? (p.n - n0) : kBN);
        for (int off = 0; off < bytes; off += 128) prefetch_l2(xrow + off);
      }
      bool ready = mbar_wait_sleep(&bar_accfull[ab], (j / kNAcc) & 1, abort_flag, p.err, kDevTimeoutEpilogue, 64, 512);
      if (!__all_sync(kFullMask, ready && !*abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < kChunks; ++cc, ++c) {
        const int nc = n0 + cc * kEC;
        const bool ok_chunk = rows_live && nc < p.n;  // warp-uniform
        float dq_next[kEC];
        int32_t bs_next[kEC];
        load_chunk_consts(p, nc + kEC, cc + 1 < kChunks && rows_live && nc + kEC < p.n, dq0, dq_next, bs_next);
        uint32_t v[kEC];
        tmem_ld_x32(tmem + lane_addr + ab * kBN + cc * kEC, v);
        tmem_wait_ld();
        if (cc == kChunks - 1) {
          // the whole accumulator has been read: hand it back to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR)
              mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bar_accempty[ab]), 0u));
            else
              mbar_arrive_relaxed(&bar_accempty[ab]);
          }
        }
        uint8_t* slot = ebuf + (c % kEBufs) * kEBufBytes;
        cp_async_wait_group<kEBufs - 2>();  // this chunk's x3 units (the later two may be in flight)
        __syncwarp();                       // ... and the other lanes' units
        if (ok_chunk) {
          int32_t acc[kEC];
#pragma unroll
          for (int i = 0; i < kEC; ++i) acc[i] = static_cast<int32_t>(v[i] + static_cast<uint32_t>(bs[i]));
          if (p.raw_acc && row_ok) {
            int4* dst = reinterpret_cast<int4*>(p.raw_acc + mm * p.n + nc);
#pragma unroll
            for (int q = 0; q < kEC / 4; ++q) dst[q] = make_int4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
          }
          // thread = row: x3 in, result out, in place
#pragma unroll
          for (int q = 0; q < kEC / 8; ++q) {
            uint4* loc = reinterpret_cast<uint4*>(slot + sw64_offset(static_cast<uint32_t>(lane), q));
            const uint4 xv = has_x3 ? *loc : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            uint32_t ow[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              float y[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int i = 8 * q + 2 * h + e;
                float u = static_cast<float>(acc[i]) * dq[i] * pt;
                if (has_x3) u += act_f32(static_cast<uint16_t>(xw[h] >> (16 * e)), BF16);
                y[e] = u;
              }
              ow[h] = pack2<BF16>(y[0], y[1]);
            }
            *loc = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
          __syncwarp();
          // row-major: whole 64-byte row segments to the output
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = ur + 8 * i;
            const uint4 val =
                *reinterpret_cast<const uint4*>(slot + sw64_offset(static_cast<uint32_t>(r), static_cast<uint32_t>(uu)));
            if (r0 + r < p.m) *reinterpret_cast<uint4*>(p.out + (r0 + r) * p.n + nc + 8 * uu) = val;
          }
        }
        __syncwarp();  // the slot is read: it takes the x3 block three chunks ahead
        load_x3(c + kEBufs - 1);
#pragma unroll
        for (int i = 0; i < kEC; ++i) {
          dq[i] = dq_next[i];
          bs[i] = bs_next[i];
        }
      }
    }
    cp_async_wait_group<0>();  // no copy may land after the CTA has exited
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // no arrival or commit may target an exited CTA
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc2(tmem, kTmemCols);
    else
      tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

namespace {

template <bool BF16, bool PAIR>
cudaError_t launch_q(const CUtensorMap& tmap_x1, const CUtensorMap& tmap_w, const QParams& p, unsigned grid,
                     cudaStream_t s) {
  auto kern = qmm_tc_kernel<BF16, PAIR>;
  constexpr int kSmem = QCfg<PAIR>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  if constexpr (!PAIR) {
    kern<<<grid, kThreads, kSmem, s>>>(tmap_x1, tmap_w, p);
    return cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap_x1, tmap_w, p);
  }
}

template <bool BF16>
int q_pair_slots() {
  auto kern = qmm_tc_kernel<BF16, true>;
  constexpr int kSmem = QCfg<true>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

int qmm_pair_slots(bool out_bf16) { return out_bf16 ? q_pair_slots<true>() : q_pair_slots<false>(); }

// p.pair_grid > 0: pair mode with that many CTAs (an even number).
cudaError_t launch_qmm_gemm(const CUtensorMap& tmap_x1, const CUtensorMap& tmap_w, const QParams& p,
                            cudaStream_t s) {
  const int64_t tiles = static_cast<int64_t>(p.num_mb) * p.num_nb;
  if (tiles <= 0 || tiles > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  if (p.pair_grid > 0) {
    if (p.pair_grid % 2 != 0) return cudaErrorInvalidConfiguration;
    return p.out_bf16 ? launch_q<true, true>(tmap_x1, tmap_w, p, p.pair_grid, s)
                      : launch_q<false, true>(tmap_x1, tmap_w, p, p.pair_grid, s);
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);  // persistent: one CTA per SM
  return p.out_bf16 ? launch_q<true, false>(tmap_x1, tmap_w, p, grid, s)
                    : launch_q<false, false>(tmap_x1, tmap_w, p, grid, s);
}

}  // namespace wqmm
