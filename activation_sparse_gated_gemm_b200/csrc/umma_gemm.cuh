// Persistent tcgen05 GEMM for sm_100a: C[M,N] = A[M,K] . B[N,K]^T with bf16
// operands and an fp32 accumulator in tensor memory, and three epilogues:
//
//   kModeTwell  -- the gate GEMM z = x . Wg. The epilogue applies ReLU and packs
//                  each 128-column tile of every row into Tile-wise ELLPACK
//                  (count, first W (column, bf16 value) pairs in ascending
//                  column order) straight from the accumulator, so the format
//                  is assembled at the end of the GEMM's own pass with no
//                  separate launch and no extra trip through memory
//                  (intellectnews.ru "Sakana AI и NVIDIA ... TwELL", section
//                  "Формат TwELL вместо классической sparse-упаковки";
//                  gate.com post 20977915, paragraph on TwELL).
//   kModeGateUp -- z and u = x . Wu in one MMA (B = 128 rows of Wg stacked on
//                  the same 128 rows of Wu); the epilogue stores
//                  h = ReLU(z) * u as bf16, and optionally the bf16 remainder
//                  h - bf16(h) beside it. The dense layer's first half.
//   kModeTwellHidden -- z and u as in kModeGateUp; the epilogue packs the
//                  positions where z > 0 into TwELL exactly as kModeTwell does,
//                  but stores h = z * u there instead of z (the up projection
//                  then runs on the tensor cores, densely).
//   kModeRelu   -- h = ReLU(x . W1) stored as bf16 (and optionally the bf16
//                  remainder, as in kModeGateUp): the first half of the dense
//                  non-gated layer.
//   kModeActivity -- the gate GEMM z = x . Wg with an epilogue that only marks
//                  the columns where some row has z > 0 (a bitmap, one bit per
//                  hidden unit, OR-ed in with one atomic per warp and 32
//                  columns): the profile that finds dead hidden units.
//   kModeF32    -- plain C = A . B^T (B K-major, like the gate GEMM) stored as
//                  fp32, with K split over the grid when the output tiles
//                  cannot fill it (partial sums added into zeroed rows): the
//                  gate (or up) pre-activations of a small batch, packed or
//                  combined by a separate kernel.
//   kModeZU     -- z and u as in kModeGateUp, both stored as fp32 ([z | u]
//                  rows): the dense backward's recomputed forward.
//   kModeBwdDh  -- dh = dy . Wd^T (B = Wd, K-major) with the backward's
//                  elementwise step in the epilogue: from the stored z and u,
//                  dz = dh u [z > 0], du = dh ReLU(z), h = ReLU(z) u, each kept
//                  as bf16 plus bf16 remainder, written token-major as
//                  [dz | du | dz_lo | du_lo | h | h_lo] (the A operand of dx
//                  over its first 4N columns, and read MN-major with the
//                  tokens as K, of the weight gradients).
//   kModeSlots  -- C = A . B^T as in kModeF32, but only the entries at the
//                  stored slots of a TwELL pack leave the accumulator: with
//                  slots_pass 0 (A = dy, B = Wd) each slot's dh_j goes to its
//                  record; with slots_pass 1 (A = x, B = Wu) the record becomes
//                  {h = g u_j, du = dh_j g, dz = dh_j u_j, token} from u_j, the
//                  stored g and the dh_j left there (the backward's records
//                  without writing dh and u in full).
//   kModeDown   -- y = h . Wd with Wd read N-major ([K][N] in memory); the
//                  epilogue stores fp32 rows, optionally scattered through a
//                  row map (the dense branch of the hybrid route). With the
//                  remainder stored, K runs over [h | h - bf16(h)] against
//                  [Wd ; Wd], which removes the bf16 rounding of h to ~2^-16.
//   kModeUnion  -- the down projection of the rows that fit over the hidden
//                  units their 128-row tile activates: per M tile, K runs over
//                  that tile's union of stored units only (its own length,
//                  read on the device), A is the tile's hidden values at those
//                  units (a block written by union_prep_kernel) and B is the
//                  union's rows of Wd, gathered four rows per TMA instruction
//                  (tile::gather4) into the layout kModeDown's boxes give.
//
// Structure: one CTA per SM walks output tiles of 128 x 256 (x 128 h-columns
// for kModeGateUp). Warp 0 issues TMA loads into a 4-stage shared-memory ring,
// warp 1 issues tcgen05.mma (M=128, N=256, K=16) into two 256-column TMEM
// accumulators in turn, and each accumulator has its own group of four
// epilogue warps (2-5 and 6-9) that drains it with tcgen05.ld, so the
// epilogues of tiles i and i+1 overlap each other and the MMAs of tile i+2.
// No cluster, no multicast: every CTA loads its own operand tiles.
#pragma once

#include "ptx.cuh"

namespace twell {

enum GemmMode : int {
  kModeTwell = 0,
  kModeGateUp = 1,
  kModeDown = 2,
  kModeTwellHidden = 3,
  kModeRelu = 4,
  kModeActivity = 5,
  kModeF32 = 6,
  kModeZU = 7,
  kModeBwdDh = 8,
  kModeUnion = 9,
  kModeSlots = 10
};

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;  // 64 bf16 = 128 bytes = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kAStageBytes = kBM * kBK * 2;  // 16 KB
constexpr int kBStageBytes = kBN * kBK * 2;  // 32 KB
constexpr int kEpiWarps = 8;                 // two groups of four, one per TMEM accumulator
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiPitch = 17;                // 32-bit words per row of the bf16 value buffer (16 pairs + pad)
constexpr int kEpiBytes = kEpiWarps * 32 * kEpiPitch * 4;
constexpr int kGemmThreads = 64 + kEpiThreads;
constexpr int kTmemCols = 512;  // two 256-column fp32 accumulators

constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStages * kAStageBytes;
constexpr int kOffEpi = kOffB + kStages * kBStageBytes;
constexpr int kOffBar = kOffEpi + kEpiBytes;
constexpr int kNumBars = 2 * kStages + 4 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kGemmSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base to 1024 (misc: TMEM base, abort flag, K splits)
static_assert(kGemmSmemBytes <= 232448, "GEMM shared memory exceeds the 227 KB per-CTA limit");

struct GemmParams {
  int M;             // rows of A (an upper bound when M_dev is set)
  const int* M_dev;  // optional device-side row count, clamped to [0, M]
  int N;             // output columns: f (TwELL), f (gate-up, h columns), d (down)
  int K;             // reduction length, a multiple of 64
  // kModeTwell outputs
  int16_t* counts;
  int16_t* idx;
  uint16_t* vals;
  uint8_t* row_ovf;
  int nT;
  int W;
  // kModeGateUp / kModeRelu output (bf16) / kModeDown output (fp32), leading dimension ldo
  uint16_t* out;
  float* out_f32;
  int ldo;
  uint32_t* active;    // kModeActivity: column bitmap, OR-ed into
  // kModeBwdDh: zu = [z | u] rows ([M][2N] fp32); a2 = [t_pad][6N] bf16 rows
  // [dz | du | dz_lo | du_lo | h | h_lo] (bf16 value and remainder), rows in
  // [M, t_pad) of the tile written as zeros. With h_split == 0 only the bf16
  // values are kept: a2 = [t_pad][3N] rows [dz | du | h]. dx reads the first
  // 2N (4N) columns along K; the weight gradients read the block as an
  // MN-major A operand with the tokens along K.
  const float* zu;
  uint16_t* a2;
  int t_pad;
  // kModeDown: B rows at or past k_split_b (after k_wrap) come from tmB1, at
  // row - k_split_b (two matrices stacked along K without copying them).
  int k_split_b;
  // kModeDown: with k_dev set, K holds two halves of k_half rows each and only
  // the first *k_dev rows (rounded up to 64) of each half are summed.
  const int* k_dev;
  int k_half;
  // kModeDown / kModeF32: add into out_f32 even when K is not split.
  int accumulate;
  // Rows of A per TMA box (0: all 128). A small batch loads only its rows (a
  // multiple of 8); the A rows past them in shared memory hold stale data that
  // only reaches accumulator rows the epilogue never stores.
  int a_box_rows;
  // kModeDown: A stored MN-major, i.e. as [K][...] rows with the M index
  // contiguous (tmA covers that array; boxes of 64 M columns by 64 K rows).
  // K block k reads rows k mod k_wrap at columns a_col_hi + m (k < k_wrap, or
  // k_wrap == 0) or a_col_lo + m (k >= k_wrap): the value and remainder halves
  // of one token-major block.
  int a_mn_major;
  int a_col_hi, a_col_lo;
  const int* row_map;  // kModeDown: output row of each A row, or null
  int out_rows;        // valid range of output rows
  // kModeGateUp / kModeRelu: also store h_lo = bf16(h - bf16(h)) at column N + c (ldo = 2N).
  int h_split;
  // kModeDown: B rows are read at k mod k_wrap (k_wrap > 0), so K = 2 * k_wrap
  // runs [h_hi | h_lo] against [Wd ; Wd].
  int k_wrap;
  // kModeDown / kModeF32: when the output tiles do not fill the grid, K is cut into up to
  // this many splits whose partial sums are added into out_f32 (which must
  // hold zeros in the rows written); 0 or 1 disables splitting.
  int k_splits_max;
  // With split_waves set (the caller zeroes the rows written in every case),
  // K is also split when the tiles fill the grid but leave its last wave
  // short.
  int split_waves;
  // kModeUnion: K blocks of each M tile (>= 1) and the B rows of each M tile
  // ([num_m][union_stride] row indices into tmB0's rows, ascending, padded to
  // a multiple of 64 with a valid row; 16-byte aligned).
  const int* kb_tile;
  const int* union_rows;
  int union_stride;
  // kModeTwellHidden and kModeTwell, optional (ovf_h set): the dense branch's
  // hidden activations of the overflowing rows, written here for their
  // overflowing tiles (h = ReLU(z) u, or ReLU(z) for the non-gated layer). A row's first overflowing tile claims a compact slot s (slot_of_row
  // holds s + 1, 0 while unclaimed, -1 while being claimed; slot_row[s] = the
  // row; *ovf_n counts the slots) and the tile's exact h goes to row s of
  // ovf_h ([slots][2 N] bf16: h at column j, h - bf16(h) at N + j).
  int* slot_of_row;
  int* slot_row;
  int* ovf_n;
  uint16_t* ovf_h;
  // kModeSlots: the records ([M][nT][W] float4, beside the TwELL slots of
  // counts / idx / vals / row_ovf above) and the pass (see the mode's note).
  float4* s_rec;
  int slots_pass;
  int* dev_status;
};


// The last eight (column, bf16 value) slots of one row's list, held in
// registers: a push shifts both 128-bit queues down by one 16-bit entry and
// enters the new one at the top, so after eight pushes entry k sits at bits
// 16k..16k+15 and the group leaves as one 16-byte store per array.
struct SlotQueue {
  uint32_t i0 = 0, i1 = 0, i2 = 0, i3 = 0, v0 = 0, v1 = 0, v2 = 0, v3 = 0;
};

__device__ __forceinline__ void q_push(SlotQueue& q, uint32_t idx16, uint32_t val16) {
  q.i0 = __funnelshift_r(q.i0, q.i1, 16);
  q.i1 = __funnelshift_r(q.i1, q.i2, 16);
  q.i2 = __funnelshift_r(q.i2, q.i3, 16);
  q.i3 = __funnelshift_r(q.i3, idx16, 16);
  q.v0 = __funnelshift_r(q.v0, q.v1, 16);
  q.v1 = __funnelshift_r(q.v1, q.v2, 16);
  q.v2 = __funnelshift_r(q.v2, q.v3, 16);
  q.v3 = __funnelshift_r(q.v3, val16, 16);
}

__device__ __forceinline__ void q_store(const SlotQueue& q, int16_t* gidx, uint16_t* gval) {
  *reinterpret_cast<uint4*>(gidx) = make_uint4(q.i0, q.i1, q.i2, q.i3);
  *reinterpret_cast<uint4*>(gval) = make_uint4(q.v0, q.v1, q.v2, q.v3);
}

// Appends the set bits of `mask` (column col0 + i, bf16 value vrow[i]) to one
// row's slot list of a TwELL tile in ascending column order, storing each full
// group of 8 with 16-byte stores.
__device__ __forceinline__ void twell_append(uint32_t mask, const uint16_t* vrow, int col0, int& cnt, int W,
                                             SlotQueue& q, int16_t* gidx, uint16_t* gval) {
  while (mask != 0) {
    const int i = __ffs(mask) - 1;
    mask &= mask - 1u;
    if (cnt < W) {
      q_push(q, static_cast<uint32_t>(col0 + i), vrow[i]);
      if ((cnt & 7) == 7) q_store(q, gidx + (cnt - 7), gval + (cnt - 7));
    }
    ++cnt;
  }
}

// Stores the last partial group of a row's slot list, padded with (-1, 0).
__device__ __forceinline__ void twell_close(int cnt, int W, SlotQueue& q, int16_t* gidx, uint16_t* gval) {
  const int n = min(cnt, W);
  if (n & 7) {
    for (int k = n & 7; k < 8; ++k) q_push(q, 0xFFFFu, 0u);
    q_store(q, gidx + (n & ~7), gval + (n & ~7));
  }
}

// Stores 32 hidden values of one row as bf16 at row_out[col ..], and with
// `split` the remainder h - bf16(h), itself rounded to bf16, at row_out[N + col ..].
__device__ __forceinline__ void store_h32(const float (&h)[32], uint16_t* row_out, int col, int N, bool split) {
  uint32_t hv[16], lv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    hv[i] = pack_bf16x2(h[2 * i], h[2 * i + 1]);
    lv[i] = pack_bf16x2(h[2 * i] - __uint_as_float(hv[i] << 16), h[2 * i + 1] - __uint_as_float(hv[i] & 0xffff0000u));
  }
  uint4* dst = reinterpret_cast<uint4*>(row_out + col);
#pragma unroll
  for (int v = 0; v < 4; ++v) dst[v] = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2], hv[4 * v + 3]);
  if (split) {
    uint4* dlo = reinterpret_cast<uint4*>(row_out + N + col);
#pragma unroll
    for (int v = 0; v < 4; ++v) dlo[v] = make_uint4(lv[4 * v], lv[4 * v + 1], lv[4 * v + 2], lv[4 * v + 3]);
  }
}

// The compact dense-branch slot of `row`, claimed by the first of its
// overflowing tiles to get here: returns s + 1 (see GemmParams::slot_of_row),
// or 0 after raising a timeout status if another tile's claim never lands.
__device__ __forceinline__ int claim_ovf_slot(const GemmParams& p, int row) {
  volatile int* so = p.slot_of_row + row;
  int sl = *so;
  if (sl == 0) {
    const int old = atomicCAS(p.slot_of_row + row, 0, -1);
    if (old == 0) {
      const int sn = atomicAdd(p.ovf_n, 1);
      p.slot_row[sn] = row;
      __threadfence();
      atomicExch(p.slot_of_row + row, sn + 1);
      return sn + 1;
    }
    sl = old;
  }
  // another tile of this row is claiming: a few instructions away
  for (int it = 0; sl < 0 && it < (1 << 22); ++it) sl = *so;
  if (sl <= 0) {
    raise_status(p.dev_status, kDevTimeout);
    return 0;
  }
  return sl;
}

// Output tiles are visited in groups of group_n consecutive N blocks: inside
// a group, every M block in turn with its group_n tiles side by side. The CTAs
// running at once then share the few B tiles of one group, which stay in L2
// while A streams past (B comes from HBM about once, A once per group); in
// plain row order every wave would touch all of B, which at the 2B layer's
// 85 MB of [Wg; Wu] does not stay in L2 (11x the algorithmic DRAM reads).
constexpr size_t kGroupBBytes = 32u << 20;

__device__ __forceinline__ void tile_mn(int mn, int num_m, int num_n, int group_n, int& m_blk, int& n_blk) {
  const int per_group = group_n * num_m;
  const int g = mn / per_group;
  const int n0 = g * group_n;
  const int gs = min(group_n, num_n - n0);
  const int r = mn - g * per_group;
  m_blk = r / gs;
  n_blk = n0 + (r - m_blk * gs);
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                     // [kStages] TMA -> MMA
  uint64_t* empty = bars + kStages;          // [kStages] MMA -> TMA
  uint64_t* tfull = bars + 2 * kStages;      // [2] MMA -> epilogue
  uint64_t* tempty = bars + 2 * kStages + 2; // [2] epilogue -> MMA
  uint64_t* drain = bars + 2 * kStages + 4;  // abort path: MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool kStacked = (MODE == kModeGateUp || MODE == kModeTwellHidden || MODE == kModeZU);  // B = [Wg; Wu]
  constexpr int kTileN = kStacked ? 128 : kBN;  // output columns per tile

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (kStacked) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Everything above is private to this CTA; what follows reads the previous
  // kernels' outputs (device-side row counts included).
  griddep_wait();
  int M = p.M;
  if (p.M_dev != nullptr) M = min(max(*p.M_dev, 0), p.M);
  const int num_m = (M + kBM - 1) / kBM;
  const int num_n = (p.N + kTileN - 1) / kTileN;
  int num_kb = p.K / kBK;
  // compact K (kModeDown with k_dev): blocks [0, nkb_half) of each half
  int nkb_half = 0;
  if (MODE == kModeDown && p.k_dev != nullptr) {
    nkb_half = (min(max(*p.k_dev, 0), p.k_half) + kBK - 1) / kBK;
    num_kb = 2 * nkb_half;
  }
  // K splits (kModeDown / kModeF32, output zeroed beforehand; when the tiles
  // fill the grid only with split_waves): the count whose work units
  // (tiles x splits) finish soonest on the grid, counting the waves of the
  // slowest CTA in units of a whole-K tile, with 2% per extra split for the
  // partial sums it adds (e.g. 189 tiles on 148 CTAs: 3 splits, 1.33 waves
  // instead of 2).
  // Warp 0 scores the candidate counts, two per lane, and the choice reaches
  // the other warps through shared memory (the divisions are too slow to run
  // in every thread of every CTA).
  int kb_per = num_kb, k_splits = 1;
  if ((MODE == kModeDown || MODE == kModeF32) && p.k_splits_max > 1 && num_m * num_n > 0 && num_kb > 0 &&
      (p.split_waves || num_m * num_n < static_cast<int>(gridDim.x))) {
    int* split_slot = reinterpret_cast<int*>(smem + kOffMisc + 8);
    if (warp == 0) {
      const long long tiles = static_cast<long long>(num_m) * num_n, grid = gridDim.x;
      const int most = min(min(p.k_splits_max, num_kb), 64);
      float best = 3.0e38f;
      int want = 1;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int ks = lane + 1 + 32 * h;
        if (ks <= most) {
          const int per = (num_kb + ks - 1) / ks;
          const int splits = (num_kb + per - 1) / per;
          const float waves = static_cast<float>((tiles * splits + grid - 1) / grid) * per / num_kb;
          const float cost = waves * (1.0f + 0.02f * (splits - 1));
          if (cost < best - 1e-6f) {
            best = cost;
            want = ks;
          }
        }
      }
      // the lowest cost, ties to the fewest splits
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int ow = __shfl_xor_sync(0xffffffffu, want, o);
        if (ob < best - 1e-6f || (fabsf(ob - best) <= 1e-6f && ow < want)) {
          best = ob;
          want = ow;
        }
      }
      if (lane == 0) *split_slot = want;
    }
    __syncthreads();
    const int want = *split_slot;
    kb_per = (num_kb + want - 1) / want;
    k_splits = (num_kb + kb_per - 1) / kb_per;
  }
  // no K block at all (an empty compact K): nothing to compute or store
  const int num_tiles = num_kb > 0 ? num_m * num_n * k_splits : 0;
  // N blocks per group: as many as keep the group's B tiles within kGroupBBytes
  const size_t b_bytes_n = static_cast<size_t>(kTileN) * (kStacked ? 2 : 1) * static_cast<size_t>(max(num_kb, 1)) * kBK * 2;
  const size_t fit_n = kGroupBBytes / b_bytes_n;
  const int group_n = fit_n < 1 ? 1 : (fit_n >= static_cast<size_t>(max(num_n, 1)) ? max(num_n, 1) : static_cast<int>(fit_n));

  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_par = 0;  // per stage: a load is outstanding / its phase parity
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mn = tile / k_splits;
        const int ks = tile - mn * k_splits;
        int m_blk, n_blk;
        tile_mn(mn, num_m, num_n, group_n, m_blk, n_blk);
        int kb_begin = ks * kb_per, kb_end = min(num_kb, (ks + 1) * kb_per);
        const int* urows = nullptr;
        int slabs = 4;
        if (MODE == kModeUnion) {
          // this M tile's union length, and the 64-column slabs of B inside d
          kb_begin = 0;
          kb_end = min(max(p.kb_tile[m_blk], 0), num_kb);
          urows = p.union_rows + static_cast<size_t>(m_blk) * p.union_stride;
          slabs = min(4, (p.N - n_blk * kBN) / 64);
        }
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          int4 rq[16];
          if (MODE == kModeUnion) {
            // the K block's 64 rows of B, fetched before the wait
#pragma unroll
            for (int q = 0; q < 16; ++q) rq[q] = __ldg(reinterpret_cast<const int4*>(urows + kb * kBK) + q);
          }
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + kOffA + s * kAStageBytes;
          uint8_t* b_dst = smem + kOffB + s * kBStageBytes;
          if (MODE == kModeUnion) {
            // A: the tile's hidden values over the union (one TMA box). B: each
            // 64-column slab gets the K block's 64 rows of Wd four at a time
            // (tile::gather4 with a one-row box), landing in the same
            // 128-byte-swizzled N-major layout a 64 x 64 box gives.
            mbar_arrive_expect_tx(&full[s], kAStageBytes + slabs * (kBStageBytes / 4));
            tma_load_2d(a_dst, &tmA, &full[s], kb * kBK, m_blk * kBM);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int lim = p.K - 1;  // a row outside Wd would be a fault in the list: clamped
              const int r0 = min(max(rq[q].x, 0), lim), r1 = min(max(rq[q].y, 0), lim);
              const int r2 = min(max(rq[q].z, 0), lim), r3 = min(max(rq[q].w, 0), lim);
              for (int i = 0; i < slabs; ++i)
                tma_gather4(b_dst + i * (kBStageBytes / 4) + q * 4 * 128, &tmB0, &full[s], n_blk * kBN + i * 64,
                            r0, r1, r2, r3);
            }
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
            continue;
          }
          // the K block's position in A (and B): compact K skips the empty
          // tail of each half
          const int kc = (nkb_half > 0 && kb >= nkb_half) ? p.k_half / kBK + (kb - nkb_half) : kb;
          mbar_arrive_expect_tx(&full[s], (p.a_box_rows > 0 ? p.a_box_rows * kBK * 2 : kAStageBytes) + kBStageBytes);
          if (MODE == kModeDown && p.a_mn_major) {
            // two 64-column slabs of M, each the K block's 64 rows
            const int kr = kc * kBK;
            const bool lo = p.k_wrap > 0 && kr >= p.k_wrap;
            const int col = (lo ? p.a_col_lo : p.a_col_hi) + m_blk * kBM;
            const int row = p.k_wrap > 0 ? kr % p.k_wrap : kr;
            tma_load_2d(a_dst, &tmA, &full[s], col, row);
            tma_load_2d(a_dst + kAStageBytes / 2, &tmA, &full[s], col + 64, row);
          } else {
            tma_load_2d(a_dst, &tmA, &full[s], kc * kBK, m_blk * kBM);
          }
          if (MODE == kModeTwell || MODE == kModeRelu || MODE == kModeActivity || MODE == kModeF32 ||
              MODE == kModeBwdDh || MODE == kModeSlots) {
            tma_load_2d(b_dst, &tmB0, &full[s], kc * kBK, n_blk * kBN);
          } else if (kStacked) {
            tma_load_2d(b_dst, &tmB0, &full[s], kc * kBK, n_blk * 128);
            tma_load_2d(b_dst + kBStageBytes / 2, &tmB1, &full[s], kc * kBK, n_blk * 128);
          } else {
            int kb_row = p.k_wrap > 0 ? (kc * kBK) % p.k_wrap : kc * kBK;
            const CUtensorMap* bm = &tmB0;
            if (p.k_split_b > 0 && kb_row >= p.k_split_b) {
              bm = &tmB1;
              kb_row -= p.k_split_b;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
              tma_load_2d(b_dst + i * (kBStageBytes / 4), bm, &full[s], n_blk * kBN + i * 64, kb_row);
          }
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(p.dev_status, kDevTimeout);
      }
      if (*abort_flag) {
        // Let every load still in flight land before the CTA's shared memory goes away.
        for (int t = 0; t < kStages; ++t)
          if (issued & (1u << t)) mbar_wait(&full[t], (issued_par >> t) & 1u, nullptr, kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const bool a_mn = MODE == kModeDown && p.a_mn_major != 0;
      const uint32_t idesc = umma_idesc_bf16(kBM, kBN, (MODE == kModeDown || MODE == kModeUnion) ? 1 : 0) |
                             (a_mn ? (1u << 15) : 0u);  // bit 15: A MN-major
      int s = 0;
      uint32_t ph = 0;
      int buf = 0;
      uint32_t tph = 0;
      bool ok = true, any_mma = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
        const int ks = tile % k_splits;
        int kb_begin = ks * kb_per, kb_end = min(num_kb, (ks + 1) * kb_per);
        if (MODE == kModeUnion) {
          kb_begin = 0;
          int m_u, n_u;
          tile_mn(tile / k_splits, num_m, num_n, group_n, m_u, n_u);
          kb_end = min(max(p.kb_tile[m_u], 0), num_kb);
        }
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + kOffA + s * kAStageBytes);
          const uint32_t b_addr = smem_u32(smem + kOffB + s * kBStageBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; a K step of
            // 16 bf16 is 32 bytes inside the swizzle row.
            // (MN-major A: two 64-wide slabs of M 8 KB apart, laid out like B below)
            const uint64_t adesc = a_mn ? umma_smem_desc(a_addr + k * 2048, kAStageBytes / 2, 1024)
                                        : umma_smem_desc(a_addr + k * 32, 16, 1024);
            uint64_t bdesc;
            if (MODE == kModeDown || MODE == kModeUnion) {
              // N-major, 128-byte swizzle: 64-column slabs 8 KB apart (LBO), 8-row
              // K groups 1 KB apart (SBO); a K step of 16 rows is 2 KB.
              bdesc = umma_smem_desc(b_addr + k * 2048, kBStageBytes / 4, 1024);
            } else {
              bdesc = umma_smem_desc(b_addr + k * 32, 16, 1024);
            }
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb != kb_begin || k != 0) ? 1u : 0u);
            any_mma = true;
          }
          umma_commit(&empty[s]);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
        if (++buf == 2) {
          buf = 0;
          tph ^= 1u;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(p.dev_status, kDevTimeout);
      }
      if (*abort_flag && any_mma) {
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, kDrainTimeoutNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    // Two groups of four warps: group g drains accumulator g, i.e. every other
    // tile of this CTA, so two tiles' epilogues run side by side while the
    // MMAs of the next tile proceed.
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 are reachable from this warp
    const int buf = (warp - 2) >> 2;
    uint32_t* ebuf = reinterpret_cast<uint32_t*>(smem + kOffEpi) + (warp - 2) * 32 * kEpiPitch;
    uint32_t tph = 0;
    for (int tile = blockIdx.x + buf * gridDim.x; tile < num_tiles; tile += 2 * gridDim.x) {
      // kModeSlots: the row's slot data for the block's two TwELL tiles (count,
      // first eight indices, and for the second pass their g and dh), loaded
      // while the accumulator is still being formed
      bool pre_skip = true;
      int pre_n[2] = {0, 0};
      uint4 pre_iq[2], pre_g8[2];
      float pre_dh[2][8];
      if (MODE == kModeSlots) {
        int mb0, nb0;
        tile_mn(tile / k_splits, num_m, num_n, group_n, mb0, nb0);
        const int r0 = mb0 * kBM + q * 32 + lane;
        pre_skip = r0 >= M || p.row_ovf[r0] != 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = nb0 * 2 + h;
          pre_iq[h] = pre_g8[h] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int e = 0; e < 8; ++e) pre_dh[h][e] = 0.0f;
          if (!pre_skip && c < p.nT) {
            const size_t b = (static_cast<size_t>(r0) * p.nT + c) * p.W;  // W is a multiple of 8
            pre_n[h] = p.counts[static_cast<size_t>(r0) * p.nT + c];
            pre_iq[h] = *reinterpret_cast<const uint4*>(p.idx + b);
            if (p.slots_pass == 1) {
              pre_g8[h] = *reinterpret_cast<const uint4*>(p.vals + b);
#pragma unroll
              for (int e = 0; e < 8; ++e) pre_dh[h][e] = reinterpret_cast<const float*>(p.s_rec + b + e)[0];
            }
          }
        }
      }
      const bool got = mbar_wait(&tfull[buf], tph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        if (lane == 0) raise_status(p.dev_status, kDevTimeout);
        break;
      }
      tc_fence_after();
      const int mn = tile / k_splits;
      int m_blk, n_blk;
      tile_mn(mn, num_m, num_n, group_n, m_blk, n_blk);
      const uint32_t t_row = tmem_base + static_cast<uint32_t>(buf * kBN) + (static_cast<uint32_t>(q * 32) << 16);
      const int row_base = m_blk * kBM + q * 32;
      const int my_row = row_base + lane;

      if (MODE == kModeTwell) {
        // Each thread owns one row (its TMEM lane). Per 32-column chunk it
        // builds the mask of strictly positive values, then walks only the set
        // bits in ascending column order, appending (column, bf16 value) to its
        // row's slot list. Slots go through an 8-entry staging buffer in shared
        // memory and leave as 16-byte stores.
        uint32_t* vrow = ebuf + lane * kEpiPitch;
        const bool row_ok = my_row < M;
        // The 8 chunks of 32 columns (TwELL tiles 2 n_blk and 2 n_blk + 1,
        // four chunks each) come out of TMEM one ahead of the walk: chunk k + 1
        // is in flight while chunk k is walked.
        int cnt = 0;  // nonzeros of my_row in the current tile so far (not capped)
        int over2 = 0;  // bit i: TwELL tile 2 n_blk + i of my_row overflowed
        SlotQueue q;
        auto walk = [&](const uint32_t (&r)[32], int k) {
          const int c = n_blk * 2 + (k >> 2);  // TwELL column tile
          const bool tile_ok = row_ok && c < p.nT;
          const size_t slot0 = (static_cast<size_t>(my_row) * p.nT + c) * p.W;
          if ((k & 3) == 0) cnt = 0;
          if (tile_ok) {
            uint32_t mask = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) mask |= (static_cast<int32_t>(r[i]) > 0 ? 1u : 0u) << i;
            if (mask != 0) {
#pragma unroll
              for (int i = 0; i < 16; ++i) vrow[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
              twell_append(mask, reinterpret_cast<const uint16_t*>(vrow), c * 128 + (k & 3) * 32, cnt, p.W, q,
                           p.idx + slot0, p.vals + slot0);
            }
            if ((k & 3) == 3) {
              twell_close(cnt, p.W, q, p.idx + slot0, p.vals + slot0);
              p.counts[static_cast<size_t>(my_row) * p.nT + c] = static_cast<int16_t>(cnt);
              if (cnt > p.W) {
                p.row_ovf[my_row] = 1;
                over2 |= 1 << (k >> 2);
              }
            }
          }
        };
        uint32_t ra[32], rb[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row, ra);
#pragma unroll 1
        for (int k = 0; k < 8; k += 2) {
          tmem_wait_ld(ra);  // chunk k is in ra
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((k + 1) * 32), rb);
          walk(ra, k);
          tmem_wait_ld(rb);  // chunk k + 1 is in rb
          if (k < 6) {
            __syncwarp();
            tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((k + 2) * 32), ra);
          } else if (p.ovf_h == nullptr) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);  // all 256 columns are out of TMEM
          }
          walk(rb, k + 1);
        }
        if (p.ovf_h != nullptr) {
          // The overflowing tiles' exact h = ReLU(z) for the dense branch, read
          // again from TMEM (the accumulator is released only after this).
          if (__any_sync(0xffffffffu, over2 != 0)) {
            const int sl = over2 != 0 ? claim_ovf_slot(p, my_row) : 0;
            uint16_t* hrow = sl > 0 ? p.ovf_h + static_cast<size_t>(sl - 1) * 2 * p.N : nullptr;
#pragma unroll 1
            for (int k = 0; k < 8; ++k) {
              const bool mine = ((over2 >> (k >> 2)) & 1) != 0;
              if (!__any_sync(0xffffffffu, mine)) continue;
              __syncwarp();
              tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(k * 32), ra);
              tmem_wait_ld(ra);
              if (hrow != nullptr && mine) {
                float h[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) h[i] = fmaxf(__uint_as_float(ra[i]), 0.0f);
                store_h32(h, hrow, (n_blk * 2 + (k >> 2)) * 128 + (k & 3) * 32, p.N, true);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&tempty[buf]);  // all 256 columns are out of TMEM
        }
      } else if (MODE == kModeTwellHidden) {
        // Same pattern as above from z (columns 0..127 of the accumulator),
        // value h = z * u with u in columns 128..255.
        uint32_t* vrow = ebuf + lane * kEpiPitch;
        const int c = n_blk;  // the 128 hidden units of this tile are TwELL tile c
        const bool tile_ok = my_row < M && c < p.nT;
        const size_t slot0 = (static_cast<size_t>(my_row) * p.nT + c) * p.W;
        int cnt = 0;
        SlotQueue q;
        // Chunk k's mask and bf16 values go to registers and shared memory
        // first; then chunk k + 1's loads are issued into the same registers and
        // the walk of chunk k runs while they are in flight.
        uint32_t zr[32], ur[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row, zr);
        tmem_ld_32x32b_x32(t_row + 128u, ur);
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          tmem_wait_ld(zr);
          tmem_wait_ld(ur);
          uint32_t mask = 0;
#pragma unroll
          for (int i = 0; i < 32; ++i) mask |= (static_cast<int32_t>(zr[i]) > 0 ? 1u : 0u) << i;
          if (!tile_ok) mask = 0;
          if (mask != 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              vrow[i] = pack_bf16x2(__uint_as_float(zr[2 * i]) * __uint_as_float(ur[2 * i]),
                                    __uint_as_float(zr[2 * i + 1]) * __uint_as_float(ur[2 * i + 1]));
          }
          if (ch < 3) {
            __syncwarp();
            tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((ch + 1) * 32), zr);
            tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(128 + (ch + 1) * 32), ur);
          } else if (p.ovf_h == nullptr) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);  // all 256 columns are out of TMEM
          }
          if (mask != 0)
            twell_append(mask, reinterpret_cast<const uint16_t*>(vrow), c * 128 + ch * 32, cnt, p.W, q,
                         p.idx + slot0, p.vals + slot0);
        }
        if (tile_ok) {
          twell_close(cnt, p.W, q, p.idx + slot0, p.vals + slot0);
          p.counts[static_cast<size_t>(my_row) * p.nT + c] = static_cast<int16_t>(cnt);
          if (cnt > p.W) p.row_ovf[my_row] = 1;
        }
        if (p.ovf_h != nullptr) {
          // An overflowing tile's exact h for the dense branch, read again from
          // TMEM (the accumulator is released only after this).
          const bool over = tile_ok && cnt > p.W;
          if (__any_sync(0xffffffffu, over)) {
            const int sl = over ? claim_ovf_slot(p, my_row) : 0;
            uint16_t* hrow = sl > 0 ? p.ovf_h + static_cast<size_t>(sl - 1) * 2 * p.N : nullptr;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              __syncwarp();
              tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), zr);
              tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(128 + ch * 32), ur);
              tmem_wait_ld(zr);
              tmem_wait_ld(ur);
              if (hrow != nullptr) {
                float h[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) h[i] = fmaxf(__uint_as_float(zr[i]), 0.0f) * __uint_as_float(ur[i]);
                store_h32(h, hrow, c * 128 + ch * 32, p.N, true);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&tempty[buf]);  // all 256 columns are out of TMEM
        }
      } else if (MODE == kModeGateUp) {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t zr[32], ur[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), zr);
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(128 + ch * 32), ur);
          tmem_wait_ld();
          if (ch == 3) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * 128 + ch * 32;
          if (my_row < M && col < p.N) {
            float h[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) h[i] = fmaxf(__uint_as_float(zr[i]), 0.0f) * __uint_as_float(ur[i]);
            store_h32(h, p.out + static_cast<size_t>(my_row) * p.ldo, col, p.N, p.h_split != 0);
          }
        }
      } else if (MODE == kModeZU) {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t zr[32], ur[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), zr);
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(128 + ch * 32), ur);
          tmem_wait_ld();
          if (ch == 3) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * 128 + ch * 32;
          if (my_row < M && col < p.N) {
            uint4* dz4 = reinterpret_cast<uint4*>(p.out_f32 + static_cast<size_t>(my_row) * p.ldo + col);
            uint4* du4 = reinterpret_cast<uint4*>(p.out_f32 + static_cast<size_t>(my_row) * p.ldo + p.N + col);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              dz4[v] = make_uint4(zr[4 * v], zr[4 * v + 1], zr[4 * v + 2], zr[4 * v + 3]);
              du4[v] = make_uint4(ur[4 * v], ur[4 * v + 1], ur[4 * v + 2], ur[4 * v + 3]);
            }
          }
        }
      } else if (MODE == kModeBwdDh) {
        const bool pair = p.h_split != 0;
        const size_t pitch = (pair ? 6 : 3) * static_cast<size_t>(p.N);
        // column of each value's bf16 part and (pair) of its remainder
        const size_t c_hi[3] = {0, static_cast<size_t>(p.N), (pair ? 4 : 2) * static_cast<size_t>(p.N)};
        const size_t c_lo[3] = {2 * static_cast<size_t>(p.N), 3 * static_cast<size_t>(p.N),
                                5 * static_cast<size_t>(p.N)};
#pragma unroll 1
        for (int ch = 0; ch < kBN / 32; ++ch) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), r);
          tmem_wait_ld();
          if (ch == kBN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * kBN + ch * 32;
          if (col >= p.N || my_row >= p.t_pad) continue;
          uint16_t* arow = p.a2 + static_cast<size_t>(my_row) * pitch + col;
          if (my_row < M) {
            const float4* z4 = reinterpret_cast<const float4*>(p.zu + static_cast<size_t>(my_row) * 2 * p.N + col);
            const float4* u4 = reinterpret_cast<const float4*>(p.zu + static_cast<size_t>(my_row) * 2 * p.N + p.N + col);
            uint32_t hi[3][16], lo[3][16];  // dz, du, h of the chunk's 32 units, as bf16 pairs
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 zq = z4[q], uq = u4[q];
              const float zz[4] = {zq.x, zq.y, zq.z, zq.w};
              const float uu[4] = {uq.x, uq.y, uq.z, uq.w};
              float v[3][4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float dh = __uint_as_float(r[4 * q + e]);
                const float g = fmaxf(zz[e], 0.0f);
                v[0][e] = zz[e] > 0.0f ? dh * uu[e] : 0.0f;  // dz
                v[1][e] = dh * g;                           // du
                v[2][e] = g * uu[e];                        // h
              }
#pragma unroll
              for (int b = 0; b < 3; ++b)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                  const int k = 2 * q + e / 2;
                  hi[b][k] = pack_bf16x2(v[b][e], v[b][e + 1]);
                  lo[b][k] = pack_bf16x2(v[b][e] - __uint_as_float(hi[b][k] << 16),
                                         v[b][e + 1] - __uint_as_float(hi[b][k] & 0xffff0000u));
                }
            }
#pragma unroll
            for (int b = 0; b < 3; ++b)
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                reinterpret_cast<uint4*>(arow + c_hi[b])[v4] =
                    make_uint4(hi[b][4 * v4], hi[b][4 * v4 + 1], hi[b][4 * v4 + 2], hi[b][4 * v4 + 3]);
                if (pair)
                  reinterpret_cast<uint4*>(arow + c_lo[b])[v4] =
                      make_uint4(lo[b][4 * v4], lo[b][4 * v4 + 1], lo[b][4 * v4 + 2], lo[b][4 * v4 + 3]);
              }
          } else {
            // padding tokens: the weight gradients' K runs over whole 64-row blocks
#pragma unroll
            for (int b = 0; b < 3; ++b)
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                reinterpret_cast<uint4*>(arow + c_hi[b])[v4] = make_uint4(0u, 0u, 0u, 0u);
                if (pair) reinterpret_cast<uint4*>(arow + c_lo[b])[v4] = make_uint4(0u, 0u, 0u, 0u);
              }
          }
        }
      } else if (MODE == kModeActivity) {
#pragma unroll 1
        for (int ch = 0; ch < kBN / 32; ++ch) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), r);
          tmem_wait_ld();
          if (ch == kBN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * kBN + ch * 32;
          uint32_t mask = 0;
          if (my_row < M) {
#pragma unroll
            for (int i = 0; i < 32; ++i) mask |= (static_cast<int32_t>(r[i]) > 0 ? 1u : 0u) << i;
          }
          mask = __reduce_or_sync(0xffffffffu, mask);
          if (lane == 0 && mask != 0 && col < p.N) atomicOr(p.active + col / 32, mask);
        }
      } else if (MODE == kModeRelu) {
#pragma unroll 1
        for (int ch = 0; ch < kBN / 32; ++ch) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), r);
          tmem_wait_ld();
          if (ch == kBN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * kBN + ch * 32;
          if (my_row < M && col < p.N) {
            float h[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) h[i] = fmaxf(__uint_as_float(r[i]), 0.0f);
            store_h32(h, p.out + static_cast<size_t>(my_row) * p.ldo, col, p.N, p.h_split != 0);
          }
        }
      } else if (MODE == kModeSlots) {
        // Per row (the thread's TMEM lane) and each of the block's two TwELL
        // tiles: the tile's stored slots, ascending, are walked beside its four
        // 32-column chunks; a half-chunk that holds one of the row's slots is
        // parked in the thread's row of the shared staging buffer and the
        // slot's entry read back from there. A slot whose column is not in its
        // own tile raises TWELL_ERR_INDEX and (second pass) gets a zero record,
        // so that it adds nothing downstream.
        uint32_t* vrow = ebuf + lane * kEpiPitch;
        const bool row_ok = !pre_skip;
        bool bad = false;
        int ptr = 0, n = 0, iq_at = -1;
        size_t base = 0;
        uint4 iq = make_uint4(0u, 0u, 0u, 0u);  // the slot indices iq_at .. iq_at + 7
        // second pass: dh_j and g of the tile's first eight slots, loaded as
        // the tile starts so that the walk does not wait on them one by one
        float dh8[8];
        uint4 g8 = make_uint4(0u, 0u, 0u, 0u);
        auto cur_j = [&]() -> int {  // column of slot ptr (a large value past the last)
          if (ptr >= n) return 0x7fffffff;
          if ((ptr & ~7) != iq_at) {
            iq_at = ptr & ~7;
            iq = *reinterpret_cast<const uint4*>(p.idx + base + iq_at);  // W is a multiple of 8
          }
          const uint32_t w2 = (ptr & 4) ? ((ptr & 2) ? iq.w : iq.z) : ((ptr & 2) ? iq.y : iq.x);
          return static_cast<int16_t>((ptr & 1) ? (w2 >> 16) : (w2 & 0xffffu));
        };
        auto drop = [&]() {  // slot ptr is not in its tile
          bad = true;
          if (p.slots_pass == 1) p.s_rec[base + ptr] = make_float4(0.f, 0.f, 0.f, __int_as_float(my_row));
          ++ptr;
        };
#pragma unroll 1
        for (int k = 0; k < kBN / 32; ++k) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(k * 32), r);
          tmem_wait_ld(r);
          if (k == kBN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int c = n_blk * 2 + (k >> 2);
          if (!row_ok || c >= p.nT) continue;
          if ((k & 3) == 0) {
            while (ptr < n) drop();  // the previous tile's slots past its last column
            const bool second = (k >> 2) != 0;
            base = (static_cast<size_t>(my_row) * p.nT + c) * p.W;
            n = min(max(second ? pre_n[1] : pre_n[0], 0), p.W);
            ptr = 0;
            iq = second ? pre_iq[1] : pre_iq[0];  // the indices of slots 0 .. 7
            iq_at = 0;
            g8 = second ? pre_g8[1] : pre_g8[0];
#pragma unroll
            for (int e = 0; e < 8; ++e) dh8[e] = second ? pre_dh[1][e] : pre_dh[0][e];
          }
          const int tile_hi = (c + 1) * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int wlo = c * 128 + (k & 3) * 32 + 16 * h, whi = wlo + 16;
            bool staged = false;
            while (ptr < n) {
              const int j = cur_j();
              if (j < wlo || j >= tile_hi) {
                drop();  // below this half-chunk (outside the tile, or out of order) or past the tile
                continue;
              }
              if (j >= whi) break;  // a later half-chunk's
              if (!staged) {
#pragma unroll
                for (int e = 0; e < 16; ++e) vrow[e] = r[16 * h + e];
                staged = true;
              }
              const float v = __uint_as_float(vrow[j - wlo]);
              float4* rec = p.s_rec + base + ptr;
              if (p.slots_pass == 0) {
                reinterpret_cast<float*>(rec)[0] = v;  // dh_j, until the second pass
              } else {
                float dh;
                uint32_t gb;
                if (ptr < 8) {
                  dh = dh8[0];
#pragma unroll
                  for (int e = 1; e < 8; ++e) dh = ptr == e ? dh8[e] : dh;
                  const uint32_t w2 = (ptr & 4) ? ((ptr & 2) ? g8.w : g8.z) : ((ptr & 2) ? g8.y : g8.x);
                  gb = (ptr & 1) ? (w2 & 0xffff0000u) : (w2 << 16);
                } else {
                  dh = reinterpret_cast<const float*>(rec)[0];
                  gb = static_cast<uint32_t>(p.vals[base + ptr]) << 16;
                }
                const float g = __uint_as_float(gb);
                *rec = make_float4(g * v, dh * g, dh * v, __int_as_float(my_row));
              }
              ++ptr;
            }
          }
        }
        while (ptr < n) drop();
        if (bad) raise_status(p.dev_status, kDevIndex);
      } else {  // kModeDown, kModeF32: fp32 rows (through the row map when given)
        int orow = my_row;
        bool valid = my_row < M;
        if (valid && p.row_map != nullptr) {
          orow = p.row_map[my_row];
          if (orow < 0 || orow >= p.out_rows) {
            valid = false;
            raise_status(p.dev_status, kDevIndex);
          }
        }
#pragma unroll 1
        for (int ch = 0; ch < kBN / 32; ++ch) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(ch * 32), r);
          tmem_wait_ld();
          if (ch == kBN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
          }
          const int col = n_blk * kBN + ch * 32;
          if (valid && col < p.N) {
            float* dst = p.out_f32 + static_cast<size_t>(orow) * p.ldo + col;
            if (k_splits > 1 || p.accumulate) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                red_add_v4(dst + 4 * v, __uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                           __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            } else {
              uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
              for (int v = 0; v < 8; ++v) d4[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
          }
        }
      }
      tph ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace twell
