// internal.h -- kernel parameter blocks and launchers shared by the host API
// (api.cu) and the kernel translation units.  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace wqmm {

// Weight kinds of the anti-quant GEMM; kWH: a float16/bfloat16 weight of the
// activations' own type (the non-quantised scenario: no scale, no offset).
enum WeightKind : int { kW4 = 0, kW8 = 1, kWFp8 = 2, kWH = 3 };
// Scale / offset modes ("计算公式" symbol table: per-tensor, per-channel,
// per-group); kNoQuant: no antiquantScale / antiquantOffset at all.
enum QuantMode : int { kPerTensor = 0, kPerChannel = 1, kPerGroup = 2, kNoQuant = 3 };

// Packed weight geometry for the anti-quant GEMM: tiles of 128 n-rows x 64 k,
// tile (nb, kt) at byte ((nb * KT + kt) * tile_bytes); inside a tile, 16-byte
// chunk c of row r sits at ((c * 128 + r) * 16).
constexpr int kWqNBlock = 128;
constexpr int kWqKTile = 64;
__host__ __device__ constexpr int wq_tile_bytes(int wk) { return wk == kW4 ? 4096 : (wk == kWH ? 16384 : 8192); }
// 16-byte chunks per weight column of one packed tile (64 k values)
__host__ __device__ constexpr int wq_chunks_per_col(int wk) { return wq_tile_bytes(wk) / (kWqNBlock * 16); }
// Packed weight geometry for the int8 GEMM: tiles of 256 n-rows x 128 k bytes,
// 32 KB each, stored in the 128-byte-swizzled K-major order (16-byte chunk c of
// row r at r * 128 + ((c ^ (r & 7)) * 16)).
constexpr int kQNBlock = 256;
constexpr int kQKTile = 128;
constexpr int kQTileBytes = kQNBlock * kQKTile;

struct WqParams {
  const uint16_t* x1;     // (m, k) row-major activations (read directly by the small-m kernel)
  const uint8_t* wpack;   // packed weight (see above)
  const uint16_t* scale;  // raw f16/bf16 bits, (rows, n) row-major after any transpose
  const uint16_t* offset; // may be null
  const uint16_t* bias;   // may be null
  const uint16_t* x3;     // may be null, (m, n)
  uint16_t* out;          // (m, n)
  float* partial;         // stream-K partial tiles [num_tiles - dp_tiles][max_slots][BN][128] fp32, or null
  uint32_t* err;          // device error word
  int64_t m;
  int n, k;
  int kt_total;           // ceil(k / 64)
  int num_nb;             // ceil(n / 128)
  int num_mb;             // ceil(m / BN)
  int num_tiles;          // num_mb * num_nb; tile t = (mb = t / num_nb, nb = t % num_nb)
                          // pair: num_mb * num_pnb pair tiles (mb = t / num_pnb,
                          // column blocks 2 * (t % num_pnb) + cluster rank)
  int pair;               // 1: clusters of two CTAs share each MMA (cta_group::2)
  int num_pnb;            // pair: ceil(num_nb / 2)
  int stream_k;           // 0: whole tiles round-robin over the grid; 1: stream-K (below)
  int dp_tiles;           // stream-K: tiles [0, dp_tiles) run whole, round-robin (a multiple of the grid);
                          // the k steps of the tiles after them are split evenly over the grid
  int sk_unit;            // stream-K: split points fall on multiples of this many k steps (1 or 2)
  int sk_grid;            // stream-K: CTAs 0 .. sk_grid - 1 share the split tiles (each gets >= 1 unit)
  int max_slots;          // stream-K: partial slots per split tile
  int sk_inline;          // stream-K: 1 -- the owner of a split tile's first k steps (which it reaches
                          // last) adds the other owners' partials and writes the output (no fix-up
                          // kernel); 0 -- every owner writes a partial, the fix-up kernel reduces
  uint64_t* sk_flags;     // stream-K inline: [num_tiles - dp_tiles][max_slots] "partial written" flags
  uint64_t sk_token;      // stream-K inline: the value a flag holds once written in this launch
  uint64_t sk_expect;     // stream-K inline: the value a tile's first owner waits for (sk_token;
                          // another value only in the test hook that makes the wait run out)
  uint64_t sk_wait_ns;    // stream-K inline: bound of that wait, in ns of %globaltimer
  int mode;               // QuantMode
  int group_size;         // per-group only
  int num_groups;         // rows of scale/offset in per-group mode
};

// Stream-K ownership: the k steps of the split tiles (tiles dp_tiles ..) are
// counted in units of U steps from the first split tile; with T units split over
// G CTAs, CTA c owns units [floor(c*T/G), floor((c+1)*T/G)); the owner of unit u
// is floor(((u+1)*G - 1) / T).  Shared by the GEMM, the fix-up kernel and the
// planner.
__host__ __device__ inline int64_t sk_start(int64_t c, int64_t T, int64_t G) { return c * T / G; }
__host__ __device__ inline int64_t sk_owner(int64_t s, int64_t T, int64_t G) { return ((s + 1) * G - 1) / T; }

// CTAs holding a part of split tile r (0-based among the split tiles): first
// and last owner.  A tile with a single owner is written whole by that CTA.
struct SkOwners {
  int64_t first, last;
};
__host__ __device__ inline SkOwners sk_tile_owners(int64_t r, int kt_total, int unit, int64_t T, int64_t G) {
  const int64_t s0 = r * kt_total;
  return {sk_owner(s0 / unit, T, G), sk_owner((s0 + kt_total - 1) / unit, T, G)};
}

struct FixupParams {      // stream-K reduction + epilogue
  const float* partial;
  const uint16_t* scale;
  const uint16_t* offset;
  const uint16_t* bias;
  const uint16_t* x3;
  uint16_t* out;
  int64_t m;
  int n;
  int bn;
  int num_nb;
  int num_tiles;
  int dp_tiles;
  int kt_total;
  int sk_unit;
  int sk_grid;
  int max_slots;
  int mode;
  int act_bf16;
};

struct QParams {
  const uint8_t* wpack;        // packed int8 weight (int8 tiling)
  const int32_t* bias;         // may be null
  const void* dq;              // dequant scale: bf16 bits or f32
  const float* pertoken;       // may be null
  const uint16_t* x3;          // may be null
  uint16_t* out;
  int32_t* raw_acc;            // test-only raw accumulator output, may be null
  uint32_t* err;
  int64_t m;
  int n, k;
  int kt_total;                // ceil(k / 128)
  int num_nb;                  // ceil(n / 256)
  int num_mb;                  // ceil(m / 128)
  int dq_bf16;                 // 1: bf16 dequant scale, 0: f32
  int dq_per_tensor;           // 1: dq has one element
  int out_bf16;                // 1: bf16 output, 0: f16
  int pair_grid;               // > 0: clusters of two CTAs share each MMA (tiles of 256 rows); grid size
};

struct PackParams {
  const uint8_t* src;     // x2 storage
  uint8_t* dst;           // packed output
  int64_t s0, s1;         // logical element strides of x2 viewed as (k, n)
  int k, n;
  int wk;                 // WeightKind (the int8 GEMM tiling uses kW8)
  int for_qmm;            // 1: int8-GEMM tiling
};

struct EpiParams {        // split-K reduction + epilogue, and the k == 0 case
  const float* partial;   // [splits][m][n] (ignored when splits == 0)
  const uint16_t* scale;
  const uint16_t* offset;
  const uint16_t* bias;
  const uint16_t* x3;
  uint16_t* out;
  int64_t m;
  int n;
  int splits;
  int mode;
  int wk;
  int act_bf16;
};

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_pack(const PackParams& p, cudaStream_t s);
cudaError_t launch_transpose_u16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t s);
// Launch configuration of the anti-quant GEMM for a BN-row m tile: CTAs per SM
// the kernel's shared/tensor memory allows (the grid is a multiple of it).
int wqmm_ctas_per_sm(int bn, int wk);
// Clusters of two CTAs of the pair-mode anti-quant GEMM that fit at once (0 if
// the m tile has no pair mode or clusters cannot be scheduled).
int wqmm_pair_slots(int bn, int wk, bool act_bf16);
cudaError_t launch_wqmm_gemm(const CUtensorMap& tmap_x1, const WqParams& p, int bn, int wk, bool act_bf16,
                             int grid, cudaStream_t s);
// The small-m kernel (m tile of 16 or 32 rows, stream-K over all tiles); reads
// x1 directly (p.x1), no tensor map.
cudaError_t launch_wqmm_smallm(const WqParams& p, int bn, int wk, bool act_bf16, int grid, cudaStream_t s);
cudaError_t launch_wqmm_fixup(const FixupParams& p, cudaStream_t s);
cudaError_t launch_wqmm_epilogue(const EpiParams& p, cudaStream_t s);
// tmap_w: the packed int8 weight viewed as rows of 128 bytes (box 128 x 128,
// no swizzle), used by the pair mode only.
cudaError_t launch_qmm_gemm(const CUtensorMap& tmap_x1, const CUtensorMap& tmap_w, const QParams& p,
                            cudaStream_t s);
// Clusters of two CTAs of the pair-mode int8 GEMM that fit at once (0 if none).
int qmm_pair_slots(bool out_bf16);

// Device error word of the library (first kernel error code, 0 if none).
uint32_t* device_error_word();

// Set the calling thread's wqmm_last_error() message and return `code`.
int32_t report_error(int32_t code, const char* msg);

// Workspace ceiling for the planner on this thread (0: none): a stream-K split
// of the last wave, which only saves time, is not planned when its partial
// tiles would not fit.  Set around planning by callers with a fixed workspace.
extern thread_local uint64_t g_plan_ws_cap;

}  // namespace wqmm
