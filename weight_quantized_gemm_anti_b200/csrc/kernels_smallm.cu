// kernels_smallm.cu -- the anti-quant weight GEMM for small m (m <= 32), the
// decode shape of aclnnWeightQuantMatmulAllReduce ("计算公式":
//     out = x1 @ ((x2 + antiquantOffset) * antiquantScale) + bias + x3).
//
// For a few rows of x1 the product is bound by streaming the weight from HBM,
// and the per-k-step work of a tensor-core pipeline -- dequantise 128 x 64
// weights, hand them to the MMA, issue four small MMAs -- has to keep pace
// with it on instruction issue.  The general kernel funnels every k step
// through one MMA-issuing thread and two x1 copy warps; at m <= 32 those
// serial hand-offs, not HBM, set its speed.  This kernel is built around the
// issue budget instead:
//
//   * DG dequantisation groups of four warps (one per TMEM lane quadrant,
//     thread = weight column) take turns of SPG consecutive k steps,
//     round-robin.  A group dequantises its turn into its own TMEM A stages
//     and its warps arrive (without waiting) at the turn's named barrier; the
//     group's own MMA-issuer warp waits there and one of its lanes issues the
//     turn's 4 * SPG tcgen05.mma (M = 128 weight columns, N = BN rows of x1,
//     K = 16) into the group's OWN accumulator and commits once: DG issuers in
//     parallel, one hand-off per turn, and no dequantiser ever waits for an
//     issuer;
//   * each group fetches its turn's x1 slabs itself with 16-byte cp.async (one
//     per thread per step for BN = 16) into shared-memory buffers tied to its
//     A stages, in the 128-byte-swizzled K-major layout the MMA reads;
//   * warp 0 streams the packed weight in 32 KB bulk copies (8 int4 k steps)
//     with an evict-first L2 policy, and in per-group mode copies each step's
//     scale and offset rows (128 columns) beside it with cp.async tied to the
//     same stage barrier, so a dequantiser reads everything from shared memory;
//   * warps 1..4 (epilogue) add the DG accumulators of an item in group order,
//     apply the per-channel scale, + bias + x3, round once and store -- or
//     write / gather the fp32 partials of a split tile.
//
// Dequantisation is the exact construction of wqmm_common.cuh.  Work: the
// persistent walk of wqmm_common.cuh, planned as stream-K over all tiles in
// units of SPG k steps: the CTAs share the k steps of all output tiles
// evenly, so a tile is split among a few CTAs; the owner of its first k steps
// adds the other owners' partials in slot order (bounded flag waits, a
// per-launch token), or, with more than four owners, every owner writes a
// partial and wqmm_fixup_kernel sums them.  Accumulation orders are fixed, so
// repeated runs agree bit for bit.  The inline wait assumes the CTAs of a
// launch are resident together (one per SM, grid <= SM count).
//
// No cluster multicast; every mbarrier wait is bounded (ptx.cuh); a group's
// four warps take every exit decision together (named barrier with AND).
#include "internal.h"
#include "ptx.cuh"
#include "wqmm_common.cuh"

namespace wqmm {

namespace {

constexpr int smin(int a, int b) { return a < b ? a : b; }

template <int BN, int WK, bool GRP, int SPG>
struct SmCfg {
  static constexpr int kTile = wq_tile_bytes(WK);      // one packed k step of a 128-column block
  static constexpr int kWStageBytes = 32768;
  static constexpr int kQ = kWStageBytes / kTile;      // k steps per weight stage
  // dequantisation groups of four warps (one per TMEM lane quadrant): four
  // single-step groups, or fewer two-step groups (a weight stage must hold a
  // turn of every group, see the producer)
  static constexpr int kDG = SPG == 1 ? 4 : (WK == kW4 && BN == 16 ? 3 : 2);
  static constexpr int kGW = 4;                        // warps per group
  static constexpr int kAccTotal = kDG * 2 * BN;       // TMEM columns: two accumulators per group
  // turn stages per group (each SPG A stages of 32 TMEM columns + SPG x1 slabs)
  static constexpr int kTS = smin(3, (512 - kAccTotal) / (32 * kDG * SPG));
  static constexpr int kX1Bytes = BN * 128;            // x1 slab of one k step (BN rows x 64 k)
  static constexpr int kXBufBytes = kDG * kTS * SPG * kX1Bytes;
  // per-group scale/offset rows of a stage: [step][half][scale, offset][128 columns]
  static constexpr int kSoBytes = GRP ? kQ * 2 * 2 * 128 * 2 : 0;
  static constexpr int kStageBytes = kWStageBytes + kSoBytes;
  static constexpr int kSmemBudget = 225 * 1024;
  static constexpr int kWStages = (kSmemBudget - kXBufBytes) / kStageBytes;
  static constexpr int kWarp0Mma = 5;                  // first MMA-issuer warp (one per group)
  static constexpr int kWarp0Dq = kWarp0Mma + kDG;     // first dequantisation warp
  static constexpr int kThreads = 32 * (kWarp0Dq + kGW * kDG);
  static constexpr int kBarCount = 32 * (kGW + 1);     // a group's warps and its issuer
  static constexpr int kSmemBytes = kXBufBytes + kWStages * kStageBytes + 1024;
  static_assert(kTS >= 2, "each group needs two turn stages");
  static_assert(kDG * SPG <= kQ, "every weight stage holds a turn of every group");
  static_assert(kQ % SPG == 0, "turns do not straddle weight stages");
  static_assert(kWStages >= 3, "weight ring depth");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kAccTotal + kDG * kTS * SPG * 32 <= 512, "TMEM budget");
  static_assert(2 + kDG * kTS <= 16, "named barriers: 0, 1 (epilogue), one per group turn stage");
};

template <int BN, int WK, bool BF16, bool GRP, int SPG>
__global__ void __launch_bounds__(SmCfg<BN, WK, GRP, SPG>::kThreads, 1) wqmm_smallm_kernel(const WqParams p) {
  using C = SmCfg<BN, WK, GRP, SPG>;
  constexpr int DG = C::kDG;
  constexpr int TS = C::kTS;
  constexpr int SW = C::kWStages;
  constexpr int Q = C::kQ;
  constexpr int kTile = C::kTile;
  constexpr uint32_t kIdesc = idesc_make(1u, BF16 ? 1u : 0u, 128u, static_cast<uint32_t>(BN));

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_x1 = smem;                      // [DG][TS][SPG] x1 slabs, 1024-aligned
  uint8_t* s_w = smem + C::kXBufBytes;       // SW stages: packed weights, then (per-group) scale/offset rows

  __shared__ __align__(8) uint64_t bar_wfull[SW];
  __shared__ __align__(8) uint64_t bar_wempty[SW];
  __shared__ __align__(8) uint64_t bar_done[DG][TS];   // a group's turn stage (A stages, x1 slabs) free again
  __shared__ __align__(8) uint64_t bar_accfull[2];     // every group's part of an item accumulated
  __shared__ __align__(8) uint64_t bar_accempty[2];    // the epilogue has read an accumulator set
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SW; ++i) {
      mbar_init(&bar_wfull[i], 1);
      mbar_init(&bar_wempty[i], 4 * (Q / SPG));  // the four warps of each turn of the stage
    }
    for (int g = 0; g < DG; ++g)
      for (int i = 0; i < TS; ++i) mbar_init(&bar_done[g][i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_accfull[i], DG);
      mbar_init(&bar_accempty[i], 4);
    }
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  Walker walk;
  walk.init(p, false);
  Item it;
  auto tile_mb = [&](int t) { return t / p.num_nb; };
  auto tile_nb = [&](int t) { return t % p.num_nb; };
  // Does group gg own a turn of the item whose turns are [tbase, tbase + nturn)?
  // (CTA turn T belongs to group T % DG.)
  auto group_has = [](int gg, uint32_t tbase, int nturn) {
    return static_cast<int>((static_cast<uint32_t>(gg) + DG - tbase % DG) % DG) < nturn;
  };

  if (warp == 0) {
    // ============================================================ producer
    // Stage s holds this CTA's k steps s*Q .. s*Q + Q - 1: one bulk copy per run
    // of consecutive k steps of one tile (a column block's packed tiles are
    // contiguous along k), so usually one 32 KB copy per stage.  In per-group
    // mode the warp's lanes also copy, with 16-byte cp.async, the scale and
    // offset rows of each step's two 32-wide k halves (128 columns each) into
    // the stage, and tie those copies to the stage's barrier before the bulk
    // copy's arrival, so that the barrier completes only once all have landed.
    const uint64_t policy = policy_evict_first();
    constexpr int kPiece = 8192 / kTile;  // k steps per bulk copy
    // per-group mode: this lane's tensor (scale / offset) and 8-column chunk
    const int so_t = lane >> 4, so_c = lane & 15;
    const uint16_t* so_base = so_t ? p.offset : p.scale;
    const int so_gq = GRP ? p.group_size / 32 : 1;  // 32-wide k halves per group row
    uint32_t s = 0;
    bool have = walk.next(p, it);
    int kt = have ? it.kt0 : 0;
    while (have) {
      const int st = s % SW;
      // the ring is several stages ahead: a slow poll costs nothing, and a
      // busy one would take issue slots from the dequantisers
      const bool ok = mbar_wait_sleep(&bar_wempty[st], ((s / SW) & 1) ^ 1, abort_flag, p.err, kDevTimeoutProducer,
                                      128, 1024);
      if (!__all_sync(kFull, ok)) break;
      uint8_t* stage = s_w + st * C::kStageBytes;
      int n_in = 0;
      while (n_in < Q && have) {
        const int nb = tile_nb(it.tile);
        const int run = min(Q - n_in, it.kt1 - kt);
        // the run's weight bytes: announced on the stage barrier, then fetched
        // in pieces of kPiece k steps (8 KB), one piece per lane, all by one
        // instruction of the warp (a bulk copy holds its issuing thread while
        // it fetches, so the pieces go out in parallel)
        if (lane == 0) mbar_expect_tx(&bar_wfull[st], static_cast<uint32_t>(run * kTile));
        __syncwarp();
        if (lane * kPiece < run) {
          const int s0 = lane * kPiece;
          bulk_g2s_hint(stage + (n_in + s0) * kTile,
                        p.wpack + (static_cast<int64_t>(nb) * p.kt_total + kt + s0) * kTile,
                        static_cast<uint32_t>(min(kPiece, run - s0) * kTile), &bar_wfull[st], policy);
        }
        if constexpr (GRP) {
          // The run's scale/offset rows, per 32-wide k half (half index
          // hidx = 2 kt + h uses group row hidx / gq): lane L copies 8
          // columns (chunk L & 15) of the scale (L < 16) or the offset, for
          // every half of the run, the row advanced without division.
          const int col = nb * kWqNBlock + so_c * 8;
          const bool col_in = so_base != nullptr && col < p.n;
          int hidx = 2 * kt;
          int row = hidx / so_gq;
          int rem = hidx - row * so_gq;
          const uint16_t* gsrc = so_base + static_cast<int64_t>(row) * p.n + col;
          uint32_t dst = smem_u32(stage + C::kWStageBytes) + static_cast<uint32_t>(n_in * 1024 + so_t * 256 + so_c * 16);
          for (int hh = 0; hh < 2 * run; ++hh) {
            const bool in = col_in && hidx * 32 < p.k;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(in ? gsrc : p.scale),
                         "r"(in ? 16u : 0u)
                         : "memory");
            dst += 512;
            ++hidx;
            if (++rem == so_gq) {
              rem = 0;
              gsrc += p.n;
            }
          }
        }
        n_in += run;
        kt += run;
        if (kt >= it.kt1) {
          have = walk.next(p, it);
          if (have) kt = it.kt0;
        }
      }
      // the stage completes once every announced byte and every lane's
      // cp.async has landed, and the single arrival below has been made
      if constexpr (GRP) cp_async_mbar_arrive(&bar_wfull[st]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_wfull[st]);
      __syncwarp();
      ++s;
    }
    // every copy this warp issued has landed before the CTA may exit
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      const uint32_t first = s > static_cast<uint32_t>(SW) ? s - SW : 0;
      for (uint32_t i = first; i < s; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&bar_wfull[i % SW], (i / SW) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp < C::kWarp0Mma) {
    // ============================================================ epilogue
    // Thread = weight column (its TMEM lane); holds the BN accumulator values
    // of its column (one per row of x1) in registers.
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 32;  // 0..127 over warps 1..4
    const int nl = quad * 32 + lane;  // weight column within the 128-column block
    uint32_t j = 0, tbase = 0;
    while (walk.next(p, it)) {
      const int nturn = (it.kt1 - it.kt0) / SPG;
      const int ab = j & 1;
      // An item's accumulators take tens of microseconds: poll slowly, so that
      // four idle warps do not take issue slots from the dequantisers -- but
      // quickly for the CTA's last item, whose epilogue ends the kernel.
      Walker peek = walk;
      Item nx;
      const bool last_item = !peek.next(p, nx);
      const bool ready = mbar_wait_sleep(&bar_accfull[ab], (j >> 1) & 1, abort_flag, p.err, kDevTimeoutEpilogue,
                                         last_item ? 64u : 512u, last_item ? 256u : 2048u);
      if (!named_bar_and(1, 128, ready && !*abort_flag)) break;
      tc_fence_after();
      float acc[BN];
#pragma unroll
      for (int q = 0; q < BN; ++q) acc[q] = 0.f;
#pragma unroll
      for (int gg = 0; gg < DG; ++gg) {
        if (!group_has(gg, tbase, nturn)) continue;  // uniform over the CTA
        uint32_t v[BN];
        if constexpr (BN == 32)
          tmem_ld_x32(tmem + lane_addr + (gg * 2 + ab) * BN, *reinterpret_cast<uint32_t(*)[32]>(v));
        else
          tmem_ld_x16(tmem + lane_addr + (gg * 2 + ab) * BN, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < BN; ++q) acc[q] += __uint_as_float(v[q]);
      }
      // the accumulators are in registers: hand them back to the groups
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&bar_accempty[ab]);

      const int nb = tile_nb(it.tile);
      const int64_t m0 = static_cast<int64_t>(tile_mb(it.tile)) * BN;
      const int nn = nb * kWqNBlock + nl;
      const bool col_ok = nn < p.n;
      const bool finisher = it.nadd > 0;
      const bool writes_out = it.slot < 0 || finisher;
      const int64_t sk_r = static_cast<int64_t>(it.tile - p.dp_tiles);
      if (!writes_out) {
        // a part of a split tile: its fp32 partial, then (inline) its flag
        float* part = p.partial + (sk_r * p.max_slots + it.slot) * (BN * kWqNBlock);
#pragma unroll
        for (int q = 0; q < BN; ++q) part[q * kWqNBlock + nl] = acc[q];
        if (p.sk_inline) {
          __threadfence();
          named_bar_sync(1, 128);
          if (et == 0) st_release_gpu_u64(p.sk_flags + sk_r * p.max_slots + it.slot, p.sk_token);
        }
      } else {
        if (finisher) {
          // wait (bounded) until every other owner has written its partial
          bool ok = true;
          if (et == 0) {
            const uint64_t t0 = globaltimer();
            for (int sl = 1; sl <= it.nadd && ok; ++sl) {
              const uint64_t* flag = p.sk_flags + sk_r * p.max_slots + sl;
              while (ld_acquire_gpu_u64(flag) != p.sk_expect) {
                if (*abort_flag || globaltimer() - t0 > p.sk_wait_ns) {
                  ok = false;
                  *abort_flag = 1;
                  atomicCAS(p.err, 0u, static_cast<uint32_t>(kDevTimeoutEpilogue));
                  break;
                }
              }
            }
            // this CTA is the flags' only reader: clear them, so that a replay
            // of this launch (a CUDA graph reuses the token) waits for its own
            if (ok)
              for (int sl = 1; sl <= it.nadd; ++sl) p.sk_flags[sk_r * p.max_slots + sl] = 0;
          }
          if (!named_bar_and(1, 128, ok)) break;
          __threadfence();
          const float* others = p.partial + sk_r * p.max_slots * (BN * kWqNBlock);
          for (int sl = 1; sl <= it.nadd; ++sl) {
            const float* src = others + static_cast<int64_t>(sl) * (BN * kWqNBlock) + nl;
#pragma unroll
            for (int q = 0; q < BN; ++q) acc[q] += src[q * kWqNBlock];
          }
        }
        float escale = 1.f;
        if constexpr (!GRP) {
          const ColConst cc = col_const<BF16, WK>(p, nn, col_ok);
          escale = (WK == kWFp8 || cc.fast) ? cc.s : 1.f;
        }
        if (col_ok) {
          const float b = p.bias ? act_f32(p.bias[nn], BF16) : 0.f;
#pragma unroll
          for (int q = 0; q < BN; ++q) {
            const int64_t mm = m0 + q;
            if (mm < p.m) {
              float y = acc[q] * escale + b;
              if (p.x3) y += act_f32(p.x3[mm * p.n + nn], BF16);
              p.out[mm * p.n + nn] = f32_act(y, BF16);
            }
          }
        }
      }
      tbase += static_cast<uint32_t>(nturn);
      ++j;
    }
  } else if (warp < C::kWarp0Dq) {
    // ============================================================ MMA issuers
    // One warp per group walks the group's turns: it waits (bar.sync) until
    // the group's four dequantisation warps have arrived for the turn -- its
    // A stages written and its x1 slabs landed -- and then one elected lane
    // issues the turn's 4 * SPG MMAs into the group's accumulator and commits
    // once.  A single issuing thread per group keeps the group's MMAs in order
    // and lets one commit track all of them.
    const int dg = warp - C::kWarp0Mma;
    uint32_t T = static_cast<uint32_t>(dg), tbase = 0, tg = 0, tg_done = 0, j = 0;
    bool dead = false;
    while (!dead && walk.next(p, it)) {
      const int nturn = (it.kt1 - it.kt0) / SPG;
      const int ab = j & 1;
      bool first = true;
      if (!group_has(dg, tbase, nturn)) {
        // no turn in this item: still count this group's arrival, once the
        // accumulator set's previous item has been read out
        bool ok = j < 2 || mbar_wait_hint(&bar_accempty[ab], ((j >> 1) & 1) ^ 1, abort_flag, p.err, kDevTimeoutMma);
        ok = __all_sync(kFull, ok);
        if (!ok) break;
        if (lane == 0) mbar_arrive(&bar_accfull[ab]);
      }
      for (; T - tbase < static_cast<uint32_t>(nturn); T += DG, ++tg) {
        const bool last = T + DG - tbase >= static_cast<uint32_t>(nturn);
        const int ts = tg % TS;
        if (__any_sync(kFull, *abort_flag != 0)) {  // one decision for the whole warp
          dead = true;
          break;
        }
        named_bar_sync(2 + dg * TS + ts, C::kBarCount);
        bool ok = !*abort_flag;  // a dequantisation warp that failed arrived after raising it
        ok = ok && (!first || j < 2 ||
                    mbar_wait_hint(&bar_accempty[ab], ((j >> 1) & 1) ^ 1, abort_flag, p.err, kDevTimeoutMma));
        if (!__all_sync(kFull, ok)) {
          dead = true;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t d = tmem + (dg * 2 + ab) * BN;
#pragma unroll
          for (int i = 0; i < SPG; ++i) {
            const uint32_t sl = static_cast<uint32_t>((dg * TS + ts) * SPG + i);
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(s_x1) + sl * static_cast<uint32_t>(C::kX1Bytes));
            const uint32_t a_t = tmem + C::kAccTotal + sl * 32;
            mma_f16_ts(d, a_t, bd, kIdesc, (first && i == 0) ? 0u : 1u);
            mma_f16_ts(d, a_t + 8, bd + 2, kIdesc, 1u);
            mma_f16_ts(d, a_t + 16, bd + 4, kIdesc, 1u);
            mma_f16_ts(d, a_t + 24, bd + 6, kIdesc, 1u);
          }
          mma_commit(&bar_done[dg][ts]);
          if (last) mma_commit(&bar_accfull[ab]);
        }
        __syncwarp();
        tg_done = tg + 1;
        first = false;
      }
      tbase += static_cast<uint32_t>(nturn);
      ++j;
    }
    // every MMA this warp issued has completed before the CTA may exit
    if (tg_done > 0 && lane == 0) {
      volatile int no_abort = 0;
      mbar_wait(&bar_done[dg][(tg_done - 1) % TS], ((tg_done - 1) / TS) & 1, &no_abort, p.err, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ============================================================ dequantisation groups
    const int dg = (warp - C::kWarp0Dq) / C::kGW;  // group: takes the CTA's turns T with T % DG == dg
    const int quad = warp & 3;                    // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;               // weight column within the 128-column block
    const int gt = ((warp - C::kWarp0Dq) % C::kGW) * 32 + lane;  // thread within the group, 0..127
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    // this thread's x1 chunks: row xr (+16 for BN = 32), 16-byte chunk xc of the 128-byte k row
    const int xr = gt >> 3, xc = gt & 7;
    const uint32_t x1_dst0 = smem_u32(s_x1) + static_cast<uint32_t>(dg * TS * SPG * C::kX1Bytes + xr * 128 +
                                                                   ((xc ^ (xr & 7)) << 4));
    const uint32_t a_base = tmem + C::kAccTotal + dg * TS * SPG * 32 + lane_addr;

    uint32_t T = static_cast<uint32_t>(dg);  // CTA turn index of this group's next turn (steps T*SPG ..)
    uint32_t tbase = 0;                      // CTA turn index of the current item's first turn
    uint32_t tg = 0;                         // this group's turns so far: turn stage tg % TS
    bool dead = false;

    while (!dead && walk.next(p, it)) {
      const int nturn = (it.kt1 - it.kt0) / SPG;
      const int nb = tile_nb(it.tile);
      const int64_t m0 = static_cast<int64_t>(tile_mb(it.tile)) * BN;
      const int nn = nb * kWqNBlock + r;
      const bool col_ok = nn < p.n;
      ColConst cc{};
      if constexpr (!GRP) {
        if (group_has(dg, tbase, nturn)) cc = col_const<BF16, WK>(p, nn, col_ok);
      }
      // x1 source of this thread's chunk(s) at the item's k step 0; rows past m
      // and columns past k are zero-filled
      const uint16_t* x1_src[BN / 16];
      bool x1_row_ok[BN / 16];
#pragma unroll
      for (int i = 0; i < BN / 16; ++i) {
        const int64_t mm = m0 + xr + 16 * i;
        x1_row_ok[i] = mm < p.m;
        x1_src[i] = p.x1 + (x1_row_ok[i] ? mm : 0) * p.k + xc * 8;
      }
      for (; T - tbase < static_cast<uint32_t>(nturn); T += DG, ++tg) {
        const int kt = it.kt0 + static_cast<int>(T - tbase) * SPG;  // the turn's first k step
        const int ts = tg % TS;
        // 1) the turn stage is free once the MMAs of this group's turn tg - TS are done
        // (a warp that runs ahead of its group waits here or for the weights
        // below; it sleeps, so as not to take issue slots from the others)
        bool ok = !*abort_flag &&
                  (tg < static_cast<uint32_t>(TS) ||
                   mbar_wait_sleep(&bar_done[dg][ts], ((tg / TS) & 1) ^ 1, abort_flag, p.err, kDevTimeoutDequant, 64,
                                   512));
        ok = __all_sync(kFull, ok);
        // 2) the turn's x1 slabs
        if (ok) {
#pragma unroll
          for (int i = 0; i < SPG; ++i) {
            const int kk = (kt + i) * kWqKTile + xc * 8;
#pragma unroll
            for (int h = 0; h < BN / 16; ++h) {
              const bool in = x1_row_ok[h] && kk < p.k;
              const uint32_t dst = x1_dst0 + static_cast<uint32_t>((ts * SPG + i) * C::kX1Bytes + h * 2048);
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                           "l"(in ? x1_src[h] + (kt + i) * kWqKTile : p.x1), "r"(in ? 16u : 0u)
                           : "memory");
            }
          }
        }
        cp_async_commit();
        // 3) the turn's weights (and scale/offset rows) have landed
        const uint32_t step0 = T * SPG;
        const uint32_t ws = (step0 / Q) % SW;
        const uint32_t wph = (step0 / (Q * SW)) & 1u;
        const uint32_t slot0 = step0 % Q;
        ok = ok && mbar_wait_sleep(&bar_wfull[ws], wph, abort_flag, p.err, kDevTimeoutDequant, 64, 512);
        ok = __all_sync(kFull, ok);
        if (ok) {
          const uint32_t stage = smem_u32(s_w) + ws * static_cast<uint32_t>(C::kStageBytes);
          // every shared-memory load of the turn first, so that their latency overlaps
          constexpr int kChunks = (WK == kW4) ? 2 : 4;
          uint4 chs[SPG][kChunks];
          uint16_t sos[SPG][4];
#pragma unroll
          for (int i = 0; i < SPG; ++i) {
            const uint32_t wt = stage + (slot0 + i) * kTile + r * 16;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) chs[i][c] = lds_v4(wt + c * kWqNBlock * 16);
            if constexpr (GRP) {
              const uint32_t so = stage + C::kWStageBytes + (slot0 + i) * 1024 + r * 2;
#pragma unroll
              for (int q = 0; q < 4; ++q) sos[i][q] = lds_u16(so + 256 * q);
            }
          }
#pragma unroll
          for (int i = 0; i < SPG; ++i) {
            const uint4* ch = chs[i];
            // 4) dequantise in registers
            uint32_t a[32];
            if constexpr (GRP) {
              const uint16_t s0 = sos[i][0], o0 = sos[i][1], s1 = sos[i][2], o1 = sos[i][3];
              if constexpr (WK == kW4) {
                const float off = act_f32(o0, BF16);
                if (__all_sync(kFull, s0 == s1 && o0 == o1 && small_int(off))) {
                  const float cst = off - (BF16 ? 136.f : 1032.f);
                  const uint32_t c2 = pack2<BF16>(cst, cst), s2 = splat_bits(s0);
                  dq4_fast<BF16, true>(ch[0], c2, s2, a);
                  dq4_fast<BF16, true>(ch[1], c2, s2, a + 16);
                } else {
                  dq4_group_half<BF16, 0>(ch[0], s0, o0, a);
                  dq4_group_half<BF16, 1>(ch[1], s1, o1, a);
                }
              } else {
                dq8_group_half<BF16, 0>(ch[0], ch[1], s0, o0, a);
                dq8_group_half<BF16, 1>(ch[2], ch[3], s1, o1, a);
              }
            } else if constexpr (WK == kW4) {
              if (cc.fast) {
                dq4_fast<BF16, false>(ch[0], cc.c2, 0u, a);
                dq4_fast<BF16, false>(ch[1], cc.c2, 0u, a + 16);
              } else {
                dq4_general<BF16>(ch[0], cc.off, cc.s, a);
                dq4_general<BF16>(ch[1], cc.off, cc.s, a + 16);
              }
            } else if constexpr (WK == kW8) {
              if (cc.fast) {
#pragma unroll
                for (int c = 0; c < 4; ++c) dq8_fast<BF16, false>(ch[c], cc.off, cc.s, cc.c2, 0u, a + 8 * c);
              } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) dq8_general<BF16>(ch[c], cc.off, cc.s, a + 8 * c);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c) dq_fp8<BF16>(ch[c], a + 8 * c);
            }
            // 5) into the turn stage's A stage i
            tmem_st_x32(a_base + (ts * SPG + i) * 32, a);
          }
          // The stage's weights and scales are consumed (the stores above cannot
          // issue before every register they store is computed from them):
          // release it.  Relaxed: nothing else of this warp's has to land first.
          __syncwarp();
          if (lane == 0) mbar_arrive_relaxed(&bar_wempty[ws]);
        }
        // 6) this turn's x1 has landed and is visible to the tensor core, the A
        // stages are written: arrive for the group's issuer, and go on.  A warp
        // whose wait failed (the abort flag is raised) arrives too, so that the
        // issuer's wait ends, and then leaves.
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        named_bar_arrive(2 + dg * TS + ts, C::kBarCount);
        if (!ok) {
          dead = true;
          break;
        }
      }
      tbase += static_cast<uint32_t>(nturn);
    }
    // nothing of this thread's may still be in flight when the CTA exits
    cp_async_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BN, int WK, bool BF16, bool GRP, int SPG>
cudaError_t launch_sm_one(const WqParams& p, int grid, cudaStream_t s) {
  using C = SmCfg<BN, WK, GRP, SPG>;
  auto kern = wqmm_smallm_kernel<BN, WK, BF16, GRP, SPG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

template <int BN, int WK, bool BF16, int SPG>
cudaError_t launch_sm_mode(const WqParams& p, int grid, cudaStream_t s) {
  if constexpr (WK == kWFp8) {  // fp8 weights have per-channel scales only
    return launch_sm_one<BN, WK, BF16, false, SPG>(p, grid, s);
  } else {
    return p.mode == kPerGroup ? launch_sm_one<BN, WK, BF16, true, SPG>(p, grid, s)
                               : launch_sm_one<BN, WK, BF16, false, SPG>(p, grid, s);
  }
}

// Two-step turns when every work item starts on an even k step and has an
// even length (the planner's stream-K unit is then two steps); one otherwise.
template <int BN, int WK, bool BF16>
cudaError_t launch_sm_spg(const WqParams& p, int grid, cudaStream_t s) {
  if (p.sk_unit == 2 && p.kt_total % 2 == 0) return launch_sm_mode<BN, WK, BF16, 2>(p, grid, s);
  return launch_sm_mode<BN, WK, BF16, 1>(p, grid, s);
}

template <int BN>
cudaError_t launch_sm_bn(const WqParams& p, int wk, bool bf16, int grid, cudaStream_t s) {
  if (wk == kWH) return cudaErrorInvalidValue;  // 16-bit weights run on the general kernel
  if (wk == kW4) return bf16 ? launch_sm_spg<BN, kW4, true>(p, grid, s) : launch_sm_spg<BN, kW4, false>(p, grid, s);
  if (wk == kW8) return bf16 ? launch_sm_spg<BN, kW8, true>(p, grid, s) : launch_sm_spg<BN, kW8, false>(p, grid, s);
  return bf16 ? launch_sm_spg<BN, kWFp8, true>(p, grid, s) : launch_sm_spg<BN, kWFp8, false>(p, grid, s);
}

}  // namespace

cudaError_t launch_wqmm_smallm(const WqParams& p, int bn, int wk, bool act_bf16, int grid, cudaStream_t s) {
  if (bn == 16) return launch_sm_bn<16>(p, wk, act_bf16, grid, s);
  if (bn == 32) return launch_sm_bn<32>(p, wk, act_bf16, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace wqmm
