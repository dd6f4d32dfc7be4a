// kernels_wqmm.cu -- anti-quant weight GEMM on the sm_100a tensor cores.
//
// Computes, per aclnnWeightQuantMatmulAllReduce "计算公式",
//     out = x1 @ ((x2 + antiquantOffset) * antiquantScale) + bias + x3
// as the transposed product  out^T = W^T x1^T,  so the dequantised weight is
// the tcgen05 A operand held in tensor memory and x1 is the B operand in
// shared memory.  A persistent, warp-specialised kernel, one CTA per SM:
//
//   warps 0 and 7 + 4 DG
//               x1 producers, alternate k steps: per 64-wide k step, the x1
//               tile (one 2-D tensor copy, 128-byte swizzle) into the x1 ring,
//               which the MMA reads;
//   warp 6      weight producer: the packed 128-column weight tile (one 1-D
//               bulk copy) into the weight ring, which the dequantisers read
//               and release as soon as the tile is in registers -- so weights
//               stream far ahead of the MMA while x1 tiles wait for it;
//   warp 1      MMA issuer: four tcgen05.mma kind::f16 (M=128, N=BN, K=16) per
//               k step, A from TMEM, B from shared memory, fp32 accumulators in
//               TMEM (two buffers when they fit, so the epilogue of one tile
//               overlaps the main loop of the next); stages are released with
//               tcgen05.commit;
//   warps 2..5  epilogue (one per TMEM lane quadrant, each on its own):
//               tcgen05.ld of the accumulator 16 columns at a time, fp32 scale,
//               staging of the warp's 32 columns, + bias / + x3, one rounding,
//               16-byte stores -- or an fp32 partial tile in stream-K mode;
//   warps 7..   DG dequantisation groups of four warps (one per lane
//               quadrant; thread = weight column).  Group g takes turns of SPG
//               consecutive k steps (steps g*SPG .. g*SPG+SPG-1 mod DG*SPG):
//               loads its column's per-group scale/offset from L2 one turn
//               ahead, unpacks its column's weights, dequantises them in
//               registers and tcgen05.st's them into its own TMEM A stages, so
//               DG turns are dequantised concurrently (DG = 2, SPG = 2 for
//               wide tiles with an even k-step count, single CTAs and CTA
//               pairs alike; DG = 4, SPG = 1 otherwise).  16-bit weights (the
//               non-quantised scenario) are stored to the A stages as they are.
//
// CTA pairs (256-row m tiles, int4 by default): clusters of two CTAs share
// each MMA (cta_group::2, M = 256 weight columns); each CTA holds half of the
// x1 slab and its own 128 weight columns, and only the even CTA issues.
//
// Work is whole output tiles dealt round-robin to the CTAs, optionally
// followed by "stream-K" tiles whose k steps are split evenly over the CTAs
// (few tiles, or the partly filled last wave of narrow tiles).  A split tile's
// owners each produce an fp32 partial.  With at most four owners, the owner of
// the tile's first k steps -- which reaches that part last of all its items --
// waits (bounded, on per-launch-token flags) for the others' partials and adds
// them in slot order in its own epilogue; with more owners, every owner writes
// a partial and wqmm_fixup_kernel sums them.  Both orders are fixed, so
// repeated runs agree bit for bit.  The inline wait assumes the persistent
// CTAs of a launch are resident together (one per SM, grid <= SM count).
//
// Dequantisation: the exact constructions of wqmm_common.cuh.
// No cluster multicast anywhere; every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"
#include "wqmm_common.cuh"

namespace wqmm {

namespace {

constexpr int pow2ceil(int v) { return v <= 32 ? 32 : v <= 64 ? 64 : v <= 128 ? 128 : v <= 256 ? 256 : 512; }
constexpr int cmin(int a, int b) { return a < b ? a : b; }

constexpr int cmax(int a, int b) { return a > b ? a : b; }

// SPG: k steps a dequantisation group takes per turn (1 or 2); a group's
// per-turn costs (barrier waits, loop and ring bookkeeping, scale/offset
// loads) are shared by its SPG steps.
template <int BN, int DG, int WK, bool PAIR = false, int SPG = 1>
struct Cfg {
  static constexpr int kTile = wq_tile_bytes(WK);
  // x1 slab of one k step held by this CTA: BN rows, or BN / 2 when a CTA pair
  // shares the MMA (each CTA holds half of the B operand)
  static constexpr int kX1Bytes = (PAIR ? BN / 2 : BN) * 128;
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr int kNAcc = (2 * kAccCols + 4 * 32 <= 512) ? 2 : 1;
  static constexpr int kACol0 = kNAcc * kAccCols;
  // TMEM A stages: as many as fit (up to 12), a multiple of DG * SPG so that
  // every dequantisation group owns its own stages
  static constexpr int kAStages = cmin(12, (512 - kACol0) / 32 / (DG * SPG) * (DG * SPG));
  static constexpr int kTmemCols = pow2ceil(kACol0 + kAStages * 32);
  // shared memory: a weight ring (read by the dequantisers, released as soon
  // as a tile is in registers) and an x1 ring (read by the MMA).  An x1 slab is
  // refilled only after the MMA of the step SX earlier has finished, so SX - 1
  // steps of MMA work have to cover the latency of its tensor copy: for wide m
  // tiles the x1 ring gets the depth and 40-48 KB of weights cover theirs.
  // Narrow m tiles stream weights from HBM: the weight ring then takes most of
  // the space, to keep enough bytes in flight.
  // epilogue staging: per epilogue warp, kEpiRows output rows x its 32
  // columns, fp32, rows kEpiPitch floats apart (the padding keeps the
  // row-wise 16-byte reads free of bank conflicts)
  static constexpr int kEpiRows = 16;
  static constexpr int kEpiPitch = 36;
  static constexpr int kStageBytes = 4 * kEpiRows * kEpiPitch * 4;
  static constexpr int kSmemBudget = 224 * 1024 - kStageBytes;
  // A weight stage holds kWQ consecutive k steps (16 KB) and is filled by one
  // or two bulk copies: a copy instruction holds its issuing thread for hundreds
  // of cycles whatever its size, so fewer, larger copies stream faster.
  static constexpr int kWQ = 16384 / kTile;
  static constexpr int kWStageBytes = kWQ * kTile;
  // A parity wait on an mbarrier can only look one phase ahead: the
  // dequantisation groups' turns of one cycle (DG * SPG steps, DG * SPG / kWQ
  // stages) must all lie in distinct stages of the weight ring, or a group
  // would wait for a stage's next fill while the current one is still pending
  // and see it as complete.
  static constexpr int kWCycle = DG * SPG / kWQ;
  static constexpr int kWStages =
      BN <= 64 ? cmin(12, (kSmemBudget - 8 * kX1Bytes) / kWStageBytes) : cmax(3, kWCycle);
  static constexpr int kXStages = cmin(16, (kSmemBudget - kWStages * kWStageBytes) / kX1Bytes);
  // The MMA issuer waits once per batch of k steps (half the A stages) and then
  // issues the whole batch: every barrier wait in the issuing thread costs the
  // tensor pipe its queued overlap, so a wait has to be followed by roughly
  // 800+ cycles of MMA work to keep the pipe busy.
  static constexpr int kBatch = cmax(1, cmin(kAStages / 2, kXStages / 2));
  // warps: 0 and kXWarp2 x1 producers, 1 MMA, 2..5 epilogue, 6 weight producer,
  // 7 .. 7 + 4 DG - 1 dequantisation
  static constexpr int kXWarp2 = 7 + 4 * DG;
  static constexpr int kThreads = 32 * (8 + 4 * DG);
  static constexpr int kSmemBytes = kXStages * kX1Bytes + kWStages * kWStageBytes + kStageBytes + 1024;
  static_assert(kAStages >= DG * SPG && kAStages % (DG * SPG) == 0, "A stages");
  static_assert(kWStages >= kWCycle, "one cycle of dequantisation turns fits in the weight ring");
  static_assert(kXStages >= DG * SPG, "one cycle of dequantisation turns fits in the x1 ring");
  static_assert(kWQ % SPG == 0 && (DG * SPG) % kWQ == 0, "a group's turn lies in one weight stage; turns cover whole stages");
  static_assert(kACol0 + kAStages * 32 <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kXStages >= 2 * kBatch && kAStages >= 2 * kBatch, "a batch must fit twice in each ring");
};

// GRP: per-group scale/offset (compile-time, so each kernel carries the code of
// its own mode only)
template <int BN, int DG, int WK, bool BF16, bool PAIR, bool GRP, int SPG>
__global__ void __launch_bounds__(Cfg<BN, DG, WK, PAIR, SPG>::kThreads, 1)
    wqmm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x1, const WqParams p) {
  using C = Cfg<BN, DG, WK, PAIR, SPG>;
  constexpr int SX = C::kXStages;
  constexpr int SW = C::kWStages;
  constexpr int AS = C::kAStages;
  // Completion of k step g is one commit on bar_done[g % RD] (phase g / RD).  A
  // waiter for step g - SX (x1 producer) or g - AS (dequantiser) can never see
  // that barrier lapped, since step g - X + RD needs data it has not yet made.
  constexpr int RD = SX + AS;
  constexpr int kTile = C::kTile;
  constexpr uint32_t kIdesc = idesc_make(1u, BF16 ? 1u : 0u, PAIR ? 256u : 128u, static_cast<uint32_t>(BN));

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_x1 = smem;                  // SX x (BN x 128 B), 1024-aligned slabs
  uint8_t* s_w = s_x1 + SX * C::kX1Bytes;  // SW x packed weight tile
  uint8_t* s_stage = s_w + SW * C::kWStageBytes;  // epilogue staging tile (fp32)

  __shared__ __align__(8) uint64_t bar_xfull[SX];
  __shared__ __align__(8) uint64_t bar_done[RD];  // one commit per k step: x1 slab and A stage free
  __shared__ __align__(8) uint64_t bar_wfull[SW];
  __shared__ __align__(8) uint64_t bar_wempty[SW];
  __shared__ __align__(8) uint64_t bar_afull[AS];
  __shared__ __align__(8) uint64_t bar_accfull[2];
  __shared__ __align__(8) uint64_t bar_accempty[2];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pairs: rank 0 issues the pair's MMAs; the A-stage and accumulator-free
  // barriers of rank 0 count the arrivals of both CTAs
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool mma_cta = (rank == 0);
  constexpr uint32_t kArrivers = PAIR ? 8u : 4u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SX; ++i) {
      mbar_init(&bar_xfull[i], 1);
    }
    for (int i = 0; i < SW; ++i) {
      mbar_init(&bar_wfull[i], 1);
      mbar_init(&bar_wempty[i], 4 * C::kWQ / SPG);
    }
    for (int i = 0; i < AS; ++i) {
      mbar_init(&bar_afull[i], kArrivers);
    }
    for (int i = 0; i < RD; ++i) mbar_init(&bar_done[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_accfull[i], 1);
      mbar_init(&bar_accempty[i], kArrivers);
    }
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc2(&tmem_base_sh, C::kTmemCols);
      tmem_relinquish2();
    } else {
      tmem_alloc(&tmem_base_sh, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the other CTA's barriers are initialised
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  Walker walk;
  walk.init(p, PAIR);
  Item it;
  // tile -> (m block, 128-column weight block of this CTA)
  auto tile_mb = [&](int t) { return PAIR ? t / p.num_pnb : t / p.num_nb; };
  auto tile_nb = [&](int t) { return PAIR ? 2 * (t % p.num_pnb) + static_cast<int>(rank) : t % p.num_nb; };
  // arrival on a barrier that counts the arrivals of both CTAs of a pair, for
  // tensor-memory hand-offs (A stage written, accumulator read): the data is
  // ordered by tcgen05.wait::st/ld and tcgen05.fence::before_thread_sync, so
  // the arrival is relaxed -- a release would first wait for the arriving
  // warp's outstanding prefetch loads (hundreds of cycles from L2)
  auto arrive_mma_cta = [&](uint64_t* bar) {
    if constexpr (PAIR)
      mbar_arrive_remote_relaxed(mapa_shared(smem_u32(bar), 0u));
    else
      mbar_arrive_relaxed(bar);
  };

  if (warp == 0 || warp == C::kXWarp2) {
    // ============================================================ x1 producers
    // Two warps take alternate k steps: one 2-D tensor copy (BN rows x 64 k,
    // 128-byte swizzle) per step into the x1 ring.  The whole warp walks the
    // ring and waits; one elected lane issues, so its operands are warp-uniform.
    const uint32_t xp = (warp == 0) ? 0u : 1u;
    if (xp == 0 && elect_one()) prefetch_tensormap(&tmap_x1);
    __syncwarp();
    uint32_t g = 0;
    bool live = true;
    while (live && walk.next(p, it)) {
      const int32_t m0 = static_cast<int32_t>(static_cast<int64_t>(tile_mb(it.tile)) * BN +
                                              (PAIR ? static_cast<int64_t>(rank) * (BN / 2) : 0));
      for (int kt = it.kt0; kt < it.kt1; ++kt, ++g) {
        if ((g & 1u) != xp) continue;
        const int st = g % SX;
        // the slab is free once the MMA of step g - SX is done
        const bool ok = g < static_cast<uint32_t>(SX) ||
                        mbar_wait(&bar_done[(g - SX) % RD], ((g - SX) / RD) & 1, abort_flag, p.err,
                                  kDevTimeoutProducer);
        if (!__all_sync(kFull, ok)) {
          live = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&bar_xfull[st], static_cast<uint32_t>(C::kX1Bytes));
          tma_load_2d(s_x1 + st * C::kX1Bytes, &tmap_x1, &bar_xfull[st], kt * kWqKTile, m0);
        }
        __syncwarp();
      }
    }
    // every copy this warp issued has landed before the CTA may exit
    if (lane == 0) {
      const uint32_t first = g > static_cast<uint32_t>(SX) ? g - SX : 0;
      for (uint32_t i = first; i < g; ++i) {
        if ((i & 1u) != xp) continue;
        volatile int no_abort = 0;
        mbar_wait(&bar_xfull[i % SX], (i / SX) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ============================================================ weight producer
    // Stage s holds this CTA's k steps s*kWQ .. s*kWQ + kWQ - 1: one bulk copy per
    // run of consecutive k steps of one tile (packed tiles of one column block
    // are contiguous along k), so usually one copy per stage.
    constexpr int Q = C::kWQ;
    uint32_t s = 0;
    bool have = walk.next(p, it);
    int kt = have ? it.kt0 : 0;
    while (have) {
      const int st = s % SW;
      const bool ok = mbar_wait_sleep(&bar_wempty[st], ((s / SW) & 1) ^ 1, abort_flag, p.err, kDevTimeoutProducer,
                                      32, 256);
      if (!__all_sync(kFull, ok)) break;
      const uint8_t* src[Q];
      int cnt[Q];
      int np = 0, n_in = 0;
      while (n_in < Q && have) {
        const int nb = tile_nb(it.tile);
        const int run = min(Q - n_in, it.kt1 - kt);
        // a column block past n (pairs over an odd block count) loads nothing:
        // its stage keeps stale bytes and its outputs are never written
        src[np] = nb < p.num_nb ? p.wpack + (static_cast<int64_t>(nb) * p.kt_total + kt) * kTile : nullptr;
        cnt[np] = run;
        ++np;
        n_in += run;
        kt += run;
        if (kt >= it.kt1) {
          have = walk.next(p, it);
          if (have) kt = it.kt0;
        }
      }
      if (elect_one()) {
        int bytes = 0;
        for (int i = 0; i < np; ++i) bytes += src[i] ? cnt[i] * kTile : 0;
        mbar_arrive_expect_tx(&bar_wfull[st], static_cast<uint32_t>(bytes));
        int off = 0;
        for (int i = 0; i < np; ++i) {
          if (src[i])
            bulk_g2s(s_w + st * C::kWStageBytes + off * kTile, src[i], static_cast<uint32_t>(cnt[i] * kTile),
                     &bar_wfull[st]);
          off += cnt[i];
        }
      }
      __syncwarp();
      ++s;
    }
    if (lane == 0) {
      const uint32_t first = s > static_cast<uint32_t>(SW) ? s - SW : 0;
      for (uint32_t i = first; i < s; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&bar_wfull[i % SW], (i / SW) & 1, &no_abort, p.err, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // The whole warp walks the schedule and waits; the elected lane issues the
    // MMAs and their commits (a commit tracks the MMAs of its own thread, and
    // elect.sync of a converged warp always picks the same lane).  With CTA
    // pairs only rank 0 issues: one MMA covers both CTAs, and each commit
    // arrives on the barrier of both.
    if (mma_cta) {
      // barrier waits for arrivals that may come from the other CTA of the pair
      auto wait_pair = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait(bar, parity, abort_flag, p.err, kDevTimeoutMma);
      };
      auto mma = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t acc) {
        if constexpr (PAIR)
          mma_f16_ts2(d, a, b, kIdesc, acc);
        else
          mma_f16_ts(d, a, b, kIdesc, acc);
      };
      auto commit = [&](uint64_t* bar) {
        if constexpr (PAIR)
          mma_commit2_mc(bar, static_cast<uint16_t>(0x3));
        else
          mma_commit(bar);
      };
      // The issuing warp shares its sub-partition with busy dequantisation
      // warps, so its loop is kept short: ring positions advance by one
      // instead of by modulo, and each MMA's operands are one add away from
      // precomputed bases (a descriptor's start address counts 16-byte units).
      const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(s_x1));
      constexpr uint64_t kSlabDesc = C::kX1Bytes >> 4;
      const uint32_t a_base = tmem + C::kACol0;
      uint32_t xs = 0, as_ = 0, rd = 0, a_par = 0;  // ring positions of the next step
      uint32_t j = 0;
      bool live = true;
      while (live && walk.next(p, it)) {
        const int ab = j % C::kNAcc;
        if (!__all_sync(kFull, wait_pair(&bar_accempty[ab], ((j / C::kNAcc) & 1) ^ 1))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + ab * C::kAccCols;
        for (int kt = it.kt0; kt < it.kt1;) {
          const int nbs = min(C::kBatch, it.kt1 - kt);
          // wait for every A stage of the batch, then issue it whole; afull of a
          // step implies its x1 slab has landed (the dequantisers check)
          bool ok = true;
          {
            uint32_t s = as_, par = a_par;
            for (int jj = 0; jj < nbs && ok; ++jj) {
              ok = wait_pair(&bar_afull[s], par);
              if (++s == AS) {
                s = 0;
                par ^= 1u;
              }
            }
          }
          if (!__all_sync(kFull, ok)) {
            live = false;
            break;
          }
          tc_fence_after();
          // operands are computed by the whole warp (warp-uniform); only the
          // tcgen05 instructions sit in the elected lane's branch
          for (int jj = 0; jj < nbs; ++jj) {
            const uint64_t bd = bdesc0 + xs * kSlabDesc;
            const uint32_t a = a_base + as_ * 32;
            const uint32_t acc0 = (kt + jj > it.kt0) ? 1u : 0u;
            uint64_t* done_bar = &bar_done[rd];
            if (elect_one()) {
              mma(d_tmem, a, bd, acc0);
              mma(d_tmem, a + 8, bd + 2, 1u);
              mma(d_tmem, a + 16, bd + 4, 1u);
              mma(d_tmem, a + 24, bd + 6, 1u);
              commit(done_bar);
            }
            __syncwarp();
            if (++xs == SX) xs = 0;
            if (++rd == RD) rd = 0;
            if (++as_ == AS) {
              as_ = 0;
              a_par ^= 1u;
            }
          }
          kt += nbs;
        }
        if (!live) break;
        if (elect_one()) commit(&bar_accfull[ab]);
        __syncwarp();
        ++j;
      }
      if (elect_one()) {
        if constexpr (PAIR)
          mma_commit2_mc(&bar_drain, static_cast<uint16_t>(0x1));
        else
          mma_commit(&bar_drain);
        volatile int no_abort = 0;
        mbar_wait(&bar_drain, 0, &no_abort, p.err, kDevTimeoutDrain);
      }
      __syncwarp();
    }
  } else if (warp < 6) {
    // ============================================================ epilogue
    // Each warp drains its own TMEM lane quadrant (32 weight columns) in
    // chunks of kEpiRows accumulator columns (output rows): (1) each thread
    // reads its weight column's values from TMEM, applies the per-column scale
    // and writes them, fp32, into the warp's staging tile [row][column]; (2)
    // after a __syncwarp, each thread takes 8 consecutive columns of one row:
    // + bias, + x3 (16-byte loads), one rounding, one 16-byte store (64
    // contiguous bytes per row and warp).  The next chunk's TMEM load is in
    // flight during (2), and no barrier couples the four warps, so the
    // accumulator is handed back to the MMA after BN / kEpiRows short rounds.
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 64;        // 0..127 over warps 2..5
    const int col8 = quad * 32 + (lane & 3) * 8;  // phase 2: 8 columns ...
    const int prow = lane >> 2;                   // ... of rows prow, prow + 8, ...
    constexpr int kER = C::kEpiRows;
    constexpr int kEP = C::kEpiPitch;
    constexpr int kPasses = kER / 8;
    static_assert(kER == 16, "the drain loads 16 accumulator columns at a time");
    // the next chunk's load is issued before phase 2 where registers allow
    // (512 threads: 128 per thread); the 768-thread kernels load each chunk
    // in turn
    constexpr bool kPrefetch = C::kThreads <= 512;
    float* wst = reinterpret_cast<float*>(s_stage) + quad * (kER * kEP);
    const bool addends = p.bias != nullptr || p.x3 != nullptr;  // uniform: bias or x3 to add
    uint32_t j = 0;
    while (walk.next(p, it)) {
      const int ab = j % C::kNAcc;
      const bool ready =
          // short sleeps: the drain of a finished tile should start promptly
          mbar_wait_sleep(&bar_accfull[ab], (j / C::kNAcc) & 1, abort_flag, p.err, kDevTimeoutEpilogue, 32, 128);
      // one decision for all four warps: they meet at named barriers below
      if (!named_bar_and(1, 128, ready && !*abort_flag)) break;
      tc_fence_after();
      const int nb = tile_nb(it.tile);
      const int64_t m0 = static_cast<int64_t>(tile_mb(it.tile)) * BN;
      const int nl = quad * 32 + lane;  // phase 1: weight column within the tile
      const int nn = nb * kWqNBlock + nl;
      const bool col_ok = nn < p.n;
      const int nn8 = nb * kWqNBlock + col8;
      const bool col8_ok = nn8 < p.n;  // n is a multiple of 32: all 8 columns or none
      float escale = 1.f;
      float bias8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) bias8[i] = 0.f;
      const bool finisher = it.nadd > 0;
      const bool writes_out = it.slot < 0 || finisher;
      if (writes_out) {
        if constexpr (!GRP) {
          const ColConst cc = col_const<BF16, WK>(p, nn, col_ok);
          escale = (WK == kWFp8 || cc.fast) ? cc.s : 1.f;
        }
        if (p.bias && col8_ok) {
          const uint4 b = *reinterpret_cast<const uint4*>(p.bias + nn8);
          const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            bias8[2 * i] = act_f32(static_cast<uint16_t>(bw[i] & 0xFFFFu), BF16);
            bias8[2 * i + 1] = act_f32(static_cast<uint16_t>(bw[i] >> 16), BF16);
          }
        }
      }
      const int64_t sk_r = static_cast<int64_t>(it.tile - p.dp_tiles);  // split tile index (stream-K items)
      float* part = writes_out ? nullptr
                               : p.partial + (sk_r * p.max_slots + it.slot) * (BN * kWqNBlock);
      // Finisher: wait (bounded) until every other owner has written its partial
      // of this tile; one thread polls, the barrier hands the result to all.
      const float* others = nullptr;
      if (finisher) {
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
          // This CTA is the flags' only reader: clear them, so that a replay of
          // this launch (a CUDA graph reuses the token) waits for its own writes.
          if (ok)
            for (int sl = 1; sl <= it.nadd; ++sl) p.sk_flags[sk_r * p.max_slots + sl] = 0;
        }
        if (!named_bar_and(1, 128, ok)) break;
        __threadfence();
        others = p.partial + sk_r * p.max_slots * (BN * kWqNBlock);  // slot s at others + s * BN * 128
      }
      const uint32_t acc_addr = tmem + lane_addr + ab * C::kAccCols;
      uint32_t v[kER];
      if constexpr (kPrefetch) tmem_ld_x16(acc_addr, v);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += kER) {
        const bool last = (c0 + kER >= BN);
        // x3 of this thread's phase-2 rows, loaded first so its latency
        // overlaps the TMEM read and the staging
        uint4 xv[kPasses];
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps) {
          const int64_t mm = m0 + c0 + ps * 8 + prow;
          xv[ps] = (part == nullptr && p.x3 && col8_ok && mm < p.m)
                       ? *reinterpret_cast<const uint4*>(p.x3 + mm * p.n + nn8)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (!kPrefetch) tmem_ld_x16(acc_addr + c0, v);
        tmem_wait_ld_r16(v);
        if (last) {
          // the whole accumulator has been read: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_mma_cta(&bar_accempty[ab]);
        }
        if (part) {
#pragma unroll
          for (int q = 0; q < kER; ++q) part[(c0 + q) * kWqNBlock + nl] = __uint_as_float(v[q]);
          if (kPrefetch && !last) tmem_ld_x16(acc_addr + c0 + kER, v);
          continue;
        }
        if (others) {
          // the owners' partials in slot order after this CTA's own (slot 0)
          float acc[kER];
#pragma unroll
          for (int q = 0; q < kER; ++q) acc[q] = __uint_as_float(v[q]);
          for (int sl = 1; sl <= it.nadd; ++sl) {
            const float* src = others + static_cast<int64_t>(sl) * (BN * kWqNBlock) + c0 * kWqNBlock + nl;
#pragma unroll
            for (int q = 0; q < kER; ++q) acc[q] += src[q * kWqNBlock];
          }
#pragma unroll
          for (int q = 0; q < kER; ++q) wst[q * kEP + lane] = acc[q] * escale;
        } else {
#pragma unroll
          for (int q = 0; q < kER; ++q) wst[q * kEP + lane] = __uint_as_float(v[q]) * escale;
        }
        __syncwarp();
        if (kPrefetch && !last) tmem_ld_x16(acc_addr + c0 + kER, v);  // in flight during phase 2
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps) {
          const int row = ps * 8 + prow;
          const int64_t mm = m0 + c0 + row;
          if (col8_ok && mm < p.m) {
            const float* src = wst + row * kEP + (lane & 3) * 8;
            const float4 lo = *reinterpret_cast<const float4*>(src);
            const float4 hi = *reinterpret_cast<const float4*>(src + 4);
            const float y[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            const uint32_t xw[4] = {xv[ps].x, xv[ps].y, xv[ps].z, xv[ps].w};
            uint32_t o[4];
            if (addends) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float a = y[2 * i] + bias8[2 * i] + act_f32(static_cast<uint16_t>(xw[i] & 0xFFFFu), BF16);
                const float b = y[2 * i + 1] + bias8[2 * i + 1] + act_f32(static_cast<uint16_t>(xw[i] >> 16), BF16);
                o[i] = pack2<BF16>(a, b);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) o[i] = pack2<BF16>(y[2 * i], y[2 * i + 1]);
            }
            *reinterpret_cast<uint4*>(p.out + mm * p.n + nn8) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        __syncwarp();  // the staging tile is rewritten by the next chunk
      }
      if (part && p.sk_inline) {
        // this owner's partial is complete: publish it to the tile's first owner
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) st_release_gpu_u64(p.sk_flags + sk_r * p.max_slots + it.slot, p.sk_token);
      }
      ++j;
    }
  } else {
    // ============================================================ dequantisation
    const int dg = (warp - 7) >> 2;               // group: takes k steps g with g % DG == dg
    const int quad = warp & 3;                    // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;               // weight column within the 128-column block
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    constexpr bool grp = GRP;
    const int gq = grp ? p.group_size / 32 : 1;   // 32-wide halves per group
    // Group dg takes turns of SPG consecutive k steps: its turns start at
    // g = SPG * dg, SPG * (dg + DG), ... of the CTA's walk, so every ring
    // position advances by CYC = DG * SPG steps per turn.  (With SPG = 2 the
    // launcher guarantees that a turn never spans two tiles.)
    constexpr int Q = C::kWQ;
    constexpr uint32_t CYC = DG * SPG;
    constexpr int NH = 2 * SPG;  // 32-wide halves of a turn
    Cursor<SW, CYC / Q> wcur;    // weight stage of the turn
    Cursor<AS, CYC> acur;        // A stage of the turn's first step
    Cursor<SX, CYC> xcur;        // x1 slab of the turn's first step
    Cursor<RD, CYC> dcur;        // done barrier of the turn's last step - AS (valid once that is >= 0)
    wcur.init(static_cast<uint32_t>(SPG * dg) / Q);
    acur.init(static_cast<uint32_t>(SPG * dg));
    xcur.init(static_cast<uint32_t>(SPG * dg));
    dcur.init(static_cast<uint32_t>(SPG * dg + SPG - 1) + RD - AS);  // phase flipped
    const uint32_t wslot = static_cast<uint32_t>(SPG * dg) % Q;      // first slot of the turn in its stage
    const int gadv_q = grp ? static_cast<int>(2 * CYC) / gq : 0;     // group rows per turn
    const int gadv_r = grp ? static_cast<int>(2 * CYC) - gadv_q * gq : 0;
    uint32_t g = static_cast<uint32_t>(SPG * dg);  // first k step of this group's next turn
    uint32_t gbase = 0;                             // step index of the current item's first k step
    bool live = true;
    while (live && walk.next(p, it)) {
      const int len = it.kt1 - it.kt0;
      const int nb = tile_nb(it.tile);
      const int nn = nb * kWqNBlock + r;
      const bool col_ok = nn < p.n;
      ColConst cc{};
      if (!grp) cc = col_const<BF16, WK>(p, nn, col_ok);
      // per-group scale/offset come straight from global memory (L2), one turn
      // ahead of their use
      GroupRow grow{};
      GroupSOn<NH> so_next{};
      if (grp && g - gbase < static_cast<uint32_t>(len)) {
        const int kt_first = it.kt0 + static_cast<int>(g - gbase);
        grow.init(2 * kt_first, gq);
        so_next = load_group_son<NH>(p, kt_first, grow, gq, nn, col_ok);
      }
      for (; g - gbase < static_cast<uint32_t>(len); g += CYC) {
        const int kt = it.kt0 + static_cast<int>(g - gbase);
        const GroupSOn<NH> so = so_next;
        if (grp && kt + static_cast<int>(CYC) < it.kt1) {
          grow.advance(gadv_q, gadv_r, gq);
          so_next = load_group_son<NH>(p, kt + CYC, grow, gq, nn, col_ok);
        }
        const int sw = static_cast<int>(wcur.i);
        // 1) the turn's weight tiles -> registers, then hand the stage back
        bool got = mbar_wait_sleep(&bar_wfull[sw], wcur.ph, abort_flag, p.err, kDevTimeoutDequant, 32, 256);
        if (!__all_sync(kFull, got)) {
          live = false;
          break;
        }
        constexpr int kChunks = wq_chunks_per_col(WK);
        uint4 ch[SPG][kChunks];
#pragma unroll
        for (int j = 0; j < SPG; ++j) {
          const uint8_t* wt = s_w + sw * C::kWStageBytes + (wslot + j) * kTile;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) ch[j][c] = *reinterpret_cast<const uint4*>(wt + (c * kWqNBlock + r) * 16);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_wempty[sw]);
        // per-group int4 with one group row for the whole turn: constants once
        bool row_fast = false;
        uint32_t rc2 = 0, rs2 = 0;
        if constexpr (GRP && WK == kW4) {
          const float off = act_f32(so.o[0], BF16);
          row_fast = so.one_row && __all_sync(kFull, small_int(off));
          const float c = off - (BF16 ? 136.f : 1032.f);
          rc2 = pack2<BF16>(c, c);
          rs2 = splat_bits(so.s[0]);
        }
#pragma unroll
        for (int j = 0; j < SPG; ++j) {
          // 2) dequantise step j in registers: needs nothing but the weights
          uint32_t a[32];
          if constexpr (WK == kW4) {
            if constexpr (GRP) {
              if (row_fast) {
                dq4_fast<BF16, true>(ch[j][0], rc2, rs2, a);
                dq4_fast<BF16, true>(ch[j][1], rc2, rs2, a + 16);
              } else {
                dq4_group_half<BF16, 0>(ch[j][0], so.s[2 * j], so.o[2 * j], a);
                dq4_group_half<BF16, 1>(ch[j][1], so.s[2 * j + 1], so.o[2 * j + 1], a);
              }
            } else if (cc.fast) {
              dq4_fast<BF16, false>(ch[j][0], cc.c2, 0u, a);
              dq4_fast<BF16, false>(ch[j][1], cc.c2, 0u, a + 16);
            } else {
              dq4_general<BF16>(ch[j][0], cc.off, cc.s, a);
              dq4_general<BF16>(ch[j][1], cc.off, cc.s, a + 16);
            }
          } else if constexpr (WK == kWH) {
            // non-quantised: the weight is already in the MMA's operand type
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
              a[4 * c] = ch[j][c].x;
              a[4 * c + 1] = ch[j][c].y;
              a[4 * c + 2] = ch[j][c].z;
              a[4 * c + 3] = ch[j][c].w;
            }
          } else if constexpr (WK == kW8) {
            if constexpr (GRP) {
              dq8_group_half<BF16, 0>(ch[j][0], ch[j][1], so.s[2 * j], so.o[2 * j], a);
              dq8_group_half<BF16, 1>(ch[j][2], ch[j][3], so.s[2 * j + 1], so.o[2 * j + 1], a);
            } else if (cc.fast) {
#pragma unroll
              for (int c = 0; c < 4; ++c) dq8_fast<BF16, false>(ch[j][c], cc.off, cc.s, cc.c2, 0u, a + 8 * c);
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c) dq8_general<BF16>(ch[j][c], cc.off, cc.s, a + 8 * c);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) dq_fp8<BF16>(ch[j][c], a + 8 * c);
          }
          if (j == 0) {
            // 3) the turn's A stages are free once the MMA of its last step -
            // AS is done (MMAs complete in order, so that covers every step)
            got = g + SPG - 1 < static_cast<uint32_t>(AS) ||
                  mbar_wait(&bar_done[dcur.i], dcur.ph ^ 1u, abort_flag, p.err, kDevTimeoutDequant);
            got = __all_sync(kFull, got);  // tcgen05.st below is warp-collective
            if (!got) break;
          }
          tmem_st_x32(tmem + lane_addr + C::kACol0 + (acur.i + j) * 32, a);
        }
        if (!got) {
          live = false;
          break;
        }
        tmem_wait_st();
        tc_fence_before();
        // 4) each step may be issued once its x1 slab has landed too
#pragma unroll
        for (int j = 0; j < SPG; ++j) {
          uint32_t xi = xcur.i + j, xph = xcur.ph;
          if (xi >= static_cast<uint32_t>(SX)) {
            xi -= SX;
            xph ^= 1u;
          }
          got = got && mbar_wait(&bar_xfull[xi], xph, abort_flag, p.err, kDevTimeoutDequant);
        }
        if (!__all_sync(kFull, got)) {
          live = false;
          break;
        }
        if (lane == 0) {
#pragma unroll
          for (int j = 0; j < SPG; ++j) arrive_mma_cta(&bar_afull[acur.i + j]);
        }
        wcur.adv();
        acur.adv();
        xcur.adv();
        dcur.adv();
      }
      gbase += static_cast<uint32_t>(len);
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair tears down together: no arrival or commit may target an exited CTA
  if constexpr (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc2(tmem, C::kTmemCols);
    else
      tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int DG, int WK, bool BF16, bool PAIR, bool GRP, int SPG>
cudaError_t launch_one(const CUtensorMap& tmap, const WqParams& p, int grid, cudaStream_t s) {
  using C = Cfg<BN, DG, WK, PAIR, SPG>;
  auto kern = wqmm_tc_kernel<BN, DG, WK, BF16, PAIR, GRP, SPG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaErrorInvalidConfiguration;
  if constexpr (!PAIR) {
    kern<<<static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, s>>>(tmap, p);
    return cudaGetLastError();
  } else {
    if (grid % 2 != 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, p);
  }
}

// Pairs of CTAs (clusters of two) that can be resident at once for this
// configuration, or 0 if none.
template <int BN, int DG, int WK, bool BF16>
int pair_slots_one() {
  using C = Cfg<BN, DG, WK, true>;
  auto kern = wqmm_tc_kernel<BN, DG, WK, BF16, true, (WK != kWFp8), 1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
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

// dequantisation groups: small tiles have little MMA work per k step, so more
// k steps must be dequantised at once to keep the weight stream flowing
template <int BN>
constexpr int dgroups() {
  return 4;
}

// Turns of two k steps per dequantisation group (two groups) for wide m
// tiles with an even number of k steps, whose work items then all start on an
// even step and have an even length (stream-K splits fall on pairs of steps);
// one step per turn (four groups) otherwise.
template <int BN, bool PAIR, int WK, bool BF16, int SPG>
cudaError_t launch_spg(const CUtensorMap& tmap, const WqParams& p, int grid, cudaStream_t s) {
  constexpr int DG = SPG == 2 ? 2 : dgroups<BN>();
  if constexpr (WK == kWFp8 || WK == kWH) {  // fp8: per-channel scales only; 16-bit: none
    return launch_one<BN, DG, WK, BF16, PAIR, false, SPG>(tmap, p, grid, s);
  } else {
    return p.mode == kPerGroup ? launch_one<BN, DG, WK, BF16, PAIR, true, SPG>(tmap, p, grid, s)
                               : launch_one<BN, DG, WK, BF16, PAIR, false, SPG>(tmap, p, grid, s);
  }
}

template <int BN, bool PAIR, int WK, bool BF16>
cudaError_t launch_mode(const CUtensorMap& tmap, const WqParams& p, int grid, cudaStream_t s) {
  if constexpr (BN >= 128 && WK != kWH) {  // a 16-bit step fills a whole weight stage
    if (p.kt_total % 2 == 0 && (!p.stream_k || p.sk_unit == 2))
      return launch_spg<BN, PAIR, WK, BF16, 2>(tmap, p, grid, s);
  }
  return launch_spg<BN, PAIR, WK, BF16, 1>(tmap, p, grid, s);
}

template <int BN, bool PAIR>
cudaError_t launch_bn(const CUtensorMap& tmap, const WqParams& p, int wk, bool bf16, int grid, cudaStream_t s) {
  if (wk == kW4)
    return bf16 ? launch_mode<BN, PAIR, kW4, true>(tmap, p, grid, s) : launch_mode<BN, PAIR, kW4, false>(tmap, p, grid, s);
  if (wk == kW8)
    return bf16 ? launch_mode<BN, PAIR, kW8, true>(tmap, p, grid, s) : launch_mode<BN, PAIR, kW8, false>(tmap, p, grid, s);
  if (wk == kWH) {
    if constexpr (PAIR) {
      return cudaErrorInvalidValue;  // no pair mode for 16-bit weights
    } else {
      return bf16 ? launch_mode<BN, false, kWH, true>(tmap, p, grid, s)
                  : launch_mode<BN, false, kWH, false>(tmap, p, grid, s);
    }
  }
  return bf16 ? launch_mode<BN, PAIR, kWFp8, true>(tmap, p, grid, s)
              : launch_mode<BN, PAIR, kWFp8, false>(tmap, p, grid, s);
}

// ---------------------------------------------------------------- stream-K fix-up
// For every split tile with more than one owner:
// out = (sum of the tile's partials, in slot order) * epilogue scale + bias + x3.
// A block takes 16 rows x 128 columns of one tile: thread = 8 consecutive
// columns of one row, 16-byte loads of each partial, of bias and x3, one
// 16-byte store.  The per-channel choice of applying the scale here is made per
// 32 aligned columns (four threads), the grouping of the GEMM's dequantisation
// warps.
constexpr int kFixRows = 16;
__global__ void __launch_bounds__(256) wqmm_fixup_kernel(const FixupParams p) {
  const int64_t split = p.num_tiles - p.dp_tiles;  // tiles after the whole-tile waves
  const int64_t T = split * p.kt_total / p.sk_unit;
  const int rb_per_tile = p.bn / kFixRows;
  const int64_t row_blocks = split * rb_per_tile;
  const int c8 = (threadIdx.x & 15) * 8;  // this thread's first column within the 128-column block
  const int rsub = threadIdx.x >> 4;      // its row within the block's 16
  const bool bf16 = p.act_bf16 != 0;
  for (int64_t rb = blockIdx.x; rb < row_blocks; rb += gridDim.x) {
    const int64_t r = rb / rb_per_tile;  // split tile index (the same for the whole block)
    const SkOwners o = sk_tile_owners(r, p.kt_total, p.sk_unit, T, p.sk_grid);
    if (o.first == o.last) continue;     // one owner: the GEMM wrote this tile whole
    const int tile = static_cast<int>(p.dp_tiles + r);
    const int ml = static_cast<int>(rb % rb_per_tile) * kFixRows + rsub;
    const int nb = tile % p.num_nb;
    const int64_t mm = static_cast<int64_t>(tile / p.num_nb) * p.bn + ml;
    const int nn = nb * kWqNBlock + c8;
    const bool col_ok = nn < p.n;  // n is a multiple of 32: 8 columns are all in or all out
    const int slots = static_cast<int>(o.last - o.first) + 1;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int sl = 0; sl < slots; ++sl) {
      const float4* src =
          reinterpret_cast<const float4*>(p.partial + ((r * p.max_slots + sl) * p.bn + ml) * kWqNBlock + c8);
      const float4 a = src[0], b = src[1];
      acc[0] += a.x, acc[1] += a.y, acc[2] += a.z, acc[3] += a.w;
      acc[4] += b.x, acc[5] += b.y, acc[6] += b.z, acc[7] += b.w;
    }
    float escale[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) escale[e] = 1.f;
    if (p.mode == kPerTensor || p.mode == kPerChannel) {
      bool small = true;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int idx = (p.mode == kPerTensor) ? 0 : (col_ok ? nn + e : 0);
        small = small && small_int(p.offset ? act_f32(p.offset[idx], bf16) : 0.f);
      }
      // the four threads of each 32-column group (lanes differing in bits 0-1) agree
      small = small && __shfl_xor_sync(kFull, static_cast<int>(small), 1);
      small = small && __shfl_xor_sync(kFull, static_cast<int>(small), 2);
      if (small) {
#pragma unroll
        for (int e = 0; e < 8; ++e) escale[e] = act_f32(p.scale[(p.mode == kPerTensor) ? 0 : (col_ok ? nn + e : 0)], bf16);
      }
    }
    if (col_ok && mm < p.m) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = acc[e] * escale[e];
      if (p.bias) {
        const uint4 bv = *reinterpret_cast<const uint4*>(p.bias + nn);
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          y[2 * h] += act_f32(static_cast<uint16_t>(bw[h] & 0xFFFFu), bf16);
          y[2 * h + 1] += act_f32(static_cast<uint16_t>(bw[h] >> 16), bf16);
        }
      }
      if (p.x3) {
        const uint4 xv = *reinterpret_cast<const uint4*>(p.x3 + mm * p.n + nn);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          y[2 * h] += act_f32(static_cast<uint16_t>(xw[h] & 0xFFFFu), bf16);
          y[2 * h + 1] += act_f32(static_cast<uint16_t>(xw[h] >> 16), bf16);
        }
      }
      uint32_t ow[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        ow[h] = static_cast<uint32_t>(f32_act(y[2 * h], bf16)) | (static_cast<uint32_t>(f32_act(y[2 * h + 1], bf16)) << 16);
      *reinterpret_cast<uint4*>(p.out + mm * p.n + nn) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
  }
}

}  // namespace

int wqmm_ctas_per_sm(int bn, int wk) {
  (void)bn;
  (void)wk;
  return 1;  // every configuration uses most of the SM's shared memory for its ring
}

template <int BN>
int pair_slots_bn(int wk, bool act_bf16) {
  constexpr int DG = dgroups<BN>();
  if (wk == kW4) return act_bf16 ? pair_slots_one<BN, DG, kW4, true>() : pair_slots_one<BN, DG, kW4, false>();
  if (wk == kW8) return act_bf16 ? pair_slots_one<BN, DG, kW8, true>() : pair_slots_one<BN, DG, kW8, false>();
  if (wk == kWH) return 0;
  return act_bf16 ? pair_slots_one<BN, DG, kWFp8, true>() : pair_slots_one<BN, DG, kWFp8, false>();
}

int wqmm_pair_slots(int bn, int wk, bool act_bf16) {
  // CTA pairs are built for the 192- and 256-row m tiles
  if (bn == 192) return pair_slots_bn<192>(wk, act_bf16);
  if (bn == 256) return pair_slots_bn<256>(wk, act_bf16);
  return 0;
}

cudaError_t launch_wqmm_gemm(const CUtensorMap& tmap_x1, const WqParams& p, int bn, int wk, bool act_bf16,
                             int grid, cudaStream_t s) {
  if (p.pair) {
    if (bn == 192) return launch_bn<192, true>(tmap_x1, p, wk, act_bf16, grid, s);
    if (bn == 256) return launch_bn<256, true>(tmap_x1, p, wk, act_bf16, grid, s);
    return cudaErrorInvalidValue;
  }
  switch (bn) {
    case 16: return launch_bn<16, false>(tmap_x1, p, wk, act_bf16, grid, s);
    case 32: return launch_bn<32, false>(tmap_x1, p, wk, act_bf16, grid, s);
    case 64: return launch_bn<64, false>(tmap_x1, p, wk, act_bf16, grid, s);
    case 128: return launch_bn<128, false>(tmap_x1, p, wk, act_bf16, grid, s);
    case 192: return launch_bn<192, false>(tmap_x1, p, wk, act_bf16, grid, s);
    case 256: return launch_bn<256, false>(tmap_x1, p, wk, act_bf16, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_wqmm_fixup(const FixupParams& p, cudaStream_t s) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = static_cast<int64_t>(p.num_tiles - p.dp_tiles) * (p.bn / kFixRows);
  if (blocks <= 0) return cudaSuccess;
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 256-thread blocks: 8 per SM fill it
  wqmm_fixup_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wqmm
