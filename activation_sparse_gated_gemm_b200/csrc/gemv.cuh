// Batches of at most 8 tokens on the CUDA cores. A GEMM tile of 128 rows would
// hold 1-8 rows of real data, so the tensor cores would stream the weights at
// a fraction of HBM speed (the split-K tcgen05 path reaches ~30% of DRAM peak at
// T = 1); here the weights stream through registers exactly once with many
// 16-byte loads in flight per SM (32 warps of 512-thread blocks, each lane
// issuing several loads before using any), and the tokens' x rows wait in
// shared memory. Kernels are compiled for 1, 2, 4 and 8 tokens.
//
// gemv_first_kernel: z = x Wg (and u = x Wu when gated) for 32 columns per
// block (two per warp, read in rounds of four loads per lane and matrix),
// then, by mode,
//  - the TwELL pack of ReLU(z) (or of h = ReLU(z) u) in the same kernel
//    (intellectnews.ru "Sakana AI и NVIDIA ... TwELL", section "Формат TwELL
//    вместо классической sparse-упаковки": the format is assembled at the end
//    of the producing pass): a cluster of four blocks covers one 128-column
//    tile and exchanges each token's partial counts through distributed
//    shared memory, so every block writes its slots at their place in
//    ascending column order and the leader writes the count;
//  - the hidden activations of the dense layer (bf16, the library's dense
//    baseline), or, for the rows routed to the dense branch, in fp32.
// gemv_down_kernel: y[rows] += h Wd, one block per (row group of Wd, 256
// columns of d), the grid sized to one wave, each lane keeping a ring of
// eight row loads in flight; partial sums added into y.
// Both need d to be a multiple of 256; other shapes take the small-batch GEMM
// path.
#pragma once

#include <cooperative_groups.h>

#include "ptx.cuh"
#include "sparse_ffn.cuh"

namespace twell {

constexpr int kGemvMaxT = 8;      // tokens per batch on this path
constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvCols = 32;     // columns of z per block (2 per warp)
constexpr int kGemvColsPerWarp = kGemvCols / kGemvWarps;
constexpr int kGemvCluster = 4;   // blocks per 128-column tile in the packing modes
constexpr int kGemvRound = 4;     // gemv_first: 16-byte loads per lane and matrix issued together
constexpr int kGemvRing = 8;      // gemv_down: 16-byte loads in flight per lane
constexpr int kGemvDownCols = 256;
constexpr int kGemvDownMaxRows = 512;  // rows of Wd per block (their h values sit in shared memory)

enum GemvMode : int {
  kGvPackGate = 0,     // TwELL of ReLU(x Wg)
  kGvPackHidden = 1,   // TwELL positions of ReLU(x Wg) > 0, values h = ReLU(x Wg) (x Wu)
  kGvDenseH = 2,       // h = bf16(ReLU(x Wg) (x Wu)) for every token
  kGvDenseRelu = 3,    // h = bf16(ReLU(x W1)) for every token
  kGvBranchH = 4,      // h = ReLU(x Wg) (x Wu) in fp32 for the listed rows
  kGvBranchRelu = 5,   // h = ReLU(x W1) in fp32 for the listed rows
};

__host__ __device__ constexpr bool gv_gated(int mode) {
  return mode == kGvPackHidden || mode == kGvDenseH || mode == kGvBranchH;
}
__host__ __device__ constexpr bool gv_pack(int mode) { return mode == kGvPackGate || mode == kGvPackHidden; }
__host__ __device__ constexpr bool gv_branch(int mode) { return mode == kGvBranchH || mode == kGvBranchRelu; }

struct GemvParams {
  const uint16_t* x;     // [T][d]
  const uint16_t* WgT;   // [f][d]
  const uint16_t* WuT;   // [f][d] (gated modes)
  int T, d, f, nT, W;
  const int* rows;       // branch modes: the tokens rows[i], i < *n_rows
  const int* n_rows;
  int16_t* counts;       // pack modes: the TwELL buffers
  int16_t* idx;
  uint16_t* vals;
  uint16_t* h_bf16;      // dense modes: [T][f]
  float* h_f32;          // branch modes: [T][f], row i for the i-th listed token
  float* y_zero;         // when not null, [T][d] zeroed by this kernel
  int* dev_status;
};

// Token count of the launch (at most NT) and, for the branch modes, the token of slot i.
template <int MODE, int NT>
__device__ __forceinline__ int gv_count(const GemvParams& p) {
  if (gv_branch(MODE)) return min(max(*p.n_rows, 0), min(p.T, NT));
  return min(p.T, NT);
}

// acc[t] += x_t . w over one 16-byte piece (8 bf16) for the first n tokens.
template <int NT>
__device__ __forceinline__ void gv_dot(float (&acc)[NT], const uint4* xs, int dv, int v, int n, const uint4& w) {
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    if (t < n) {
      float a0 = 0.0f, a1 = 0.0f;
      mixdot8(xs[t * dv + v], w, a0, a1);
      acc[t] += a0 + a1;
    }
  }
}

template <int MODE, int NT>
__global__ void __launch_bounds__(kGemvThreads, NT <= 2 ? 2 : 1) gemv_first_kernel(const GemvParams p) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ __align__(16) uint8_t gv_smem[];
  uint4* xs = reinterpret_cast<uint4*>(gv_smem);  // [NT][d/8]
  __shared__ float zs[NT][kGemvCols];
  __shared__ float us[NT][kGemvCols];
  __shared__ int part[kGemvCluster][kGemvMaxT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, dv = p.d / 8;

  if (p.y_zero != nullptr) {
    const size_t n4 = static_cast<size_t>(p.T) * d / 4;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
      reinterpret_cast<float4*>(p.y_zero)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int n = gv_count<MODE, NT>(p);
  if (gv_branch(MODE) && n == 0) return;  // no cluster in the branch modes
  bool bad = false;
  for (int e = threadIdx.x; e < n * dv; e += blockDim.x) {
    const int t = e / dv, k = e - t * dv;
    int r = t;
    if (gv_branch(MODE)) {
      r = p.rows[t];
      if (r < 0 || r >= p.T) {
        bad = true;
        r = -1;
      }
    }
    xs[e] = r >= 0 ? ldg_nc_v4(p.x + static_cast<size_t>(r) * d + k * 8) : make_uint4(0, 0, 0, 0);
  }
  if (bad) raise_status(p.dev_status, kDevIndex);
  __syncthreads();

  const int col0 = gv_pack(MODE) ? (blockIdx.x / kGemvCluster) * 128 + (blockIdx.x % kGemvCluster) * kGemvCols
                                 : blockIdx.x * kGemvCols;
  // Warp w reads weight rows col0 + 2w and + 2w + 1, each in rounds of four
  // 16-byte loads per lane and matrix, all issued before any is used.
#pragma unroll 1
  for (int k = 0; k < kGemvColsPerWarp; ++k) {
    const int lc = warp * kGemvColsPerWarp + k;  // local column
    const int j = col0 + lc;
    float ag[NT], au[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.0f;
    const uint4* rg = reinterpret_cast<const uint4*>(p.WgT + static_cast<size_t>(j) * d);
    const uint4* ru = gv_gated(MODE) ? reinterpret_cast<const uint4*>(p.WuT + static_cast<size_t>(j) * d) : nullptr;
#pragma unroll 1
    for (int base = 0; base < dv; base += kGemvRound * 32) {
      uint4 wg[kGemvRound], wu[kGemvRound];
#pragma unroll
      for (int i = 0; i < kGemvRound; ++i) {
        const int v = base + i * 32 + lane;
        wg[i] = v < dv ? __ldg(rg + v) : make_uint4(0, 0, 0, 0);
        if (gv_gated(MODE)) wu[i] = v < dv ? __ldg(ru + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kGemvRound; ++i) {
        const int v = base + i * 32 + lane;
        if (v < dv) {
          gv_dot<NT>(ag, xs, dv, v, n, wg[i]);
          if (gv_gated(MODE)) gv_dot<NT>(au, xs, dv, v, n, wu[i]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (t < n) {
        float g = ag[t], u = au[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          g += __shfl_xor_sync(0xffffffffu, g, o);
          if (gv_gated(MODE)) u += __shfl_xor_sync(0xffffffffu, u, o);
        }
        if (lane == 0) {
          zs[t][lc] = g;
          us[t][lc] = u;
        }
      }
    }
  }
  __syncthreads();

  if constexpr (gv_pack(MODE)) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int c = blockIdx.x / kGemvCluster;
    uint32_t m = 0;
    float v = 0.0f;
    // warp t packs token t (NT <= kGemvWarps)
    if (warp < n) {
      const float z = zs[warp][lane];
      v = gv_gated(MODE) ? fmaxf(z, 0.0f) * us[warp][lane] : z;
      m = __ballot_sync(0xffffffffu, z > 0.0f);
      if (lane == 0) cluster.map_shared_rank(&part[0][0], 0)[rank * kGemvMaxT + warp] = __popc(m);
    }
    cluster.sync();
    if (warp < n) {
      const int* lead = cluster.map_shared_rank(&part[0][0], 0);
      int off = 0, total = 0;
#pragma unroll
      for (int r = 0; r < kGemvCluster; ++r) {
        const int pc = lead[r * kGemvMaxT + warp];
        off += r < rank ? pc : 0;
        total += pc;
      }
      const size_t base = (static_cast<size_t>(warp) * p.nT + c) * p.W;
      if ((m >> lane) & 1u) {
        const int s = off + __popc(m & ((1u << lane) - 1u));
        if (s < p.W) {
          p.idx[base + s] = static_cast<int16_t>(col0 + lane);
          p.vals[base + s] = f32_to_bf16_bits(v);
        }
      }
      if (rank == 0 && lane == 0) p.counts[static_cast<size_t>(warp) * p.nT + c] = static_cast<int16_t>(total);
    }
    cluster.sync();  // the leader's counts stay readable until every block has read them
  } else {
    for (int e = threadIdx.x; e < n * kGemvCols; e += blockDim.x) {
      const int t = e / kGemvCols, lc2 = e - t * kGemvCols;
      const float z = fmaxf(zs[t][lc2], 0.0f);
      const float h = gv_gated(MODE) ? z * us[t][lc2] : z;
      if (gv_branch(MODE)) {
        p.h_f32[static_cast<size_t>(t) * p.f + col0 + lc2] = h;
      } else {
        p.h_bf16[static_cast<size_t>(t) * p.f + col0 + lc2] = f32_to_bf16_bits(h);
      }
    }
  }
}

struct GemvDownParams {
  const uint16_t* h_bf16;  // [T][f], or
  const float* h_f32;      // [T][f] (row i of the list)
  const uint16_t* Wd;      // [f][d]
  float* y;                // [T][d], zeroed in the rows written
  const int* rows;         // when not null: h row i goes to y row rows[i], i < *n_rows
  const int* n_rows;
  int T, d, f;
  int rows_per_block;      // rows of Wd per block: a multiple of kGemvWarps, at most kGemvDownMaxRows
};

// One block per (rows_per_block rows of Wd, 256 columns of d). Warp w streams
// its contiguous share of the block's rows, lane l owning columns 8l..8l+7 of
// the slice; the warps' partial sums meet in shared memory (column-major so
// the lanes' adds hit distinct banks), then are added into y.
template <int NT>
__global__ void __launch_bounds__(kGemvThreads, NT <= 2 ? 2 : 1) gemv_down_kernel(const GemvDownParams p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float hs[NT][kGemvDownMaxRows];
  __shared__ float acc_s[NT][kGemvDownCols];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = p.rows != nullptr ? min(max(*p.n_rows, 0), min(p.T, NT)) : min(p.T, NT);
  if (n == 0) return;
  const int r0 = blockIdx.x * p.rows_per_block;
  const int nr = min(p.rows_per_block, p.f - r0);
  const int c0 = blockIdx.y * kGemvDownCols;
  for (int e = threadIdx.x; e < n * nr; e += blockDim.x) {
    const int t = e / nr, r = e - t * nr;
    const size_t at = static_cast<size_t>(t) * p.f + r0 + r;
    hs[t][r] = p.h_f32 != nullptr ? p.h_f32[at] : __uint_as_float(static_cast<uint32_t>(p.h_bf16[at]) << 16);
  }
  for (int e = threadIdx.x; e < NT * kGemvDownCols; e += blockDim.x) (&acc_s[0][0])[e] = 0.0f;
  __syncthreads();
  const int col = c0 + lane * 8;
  float a[NT][8];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 8; ++i) a[t][i] = 0.0f;
  const int per = p.rows_per_block / kGemvWarps;
  const int w0 = warp * per, w1 = min(w0 + per, nr);  // the warp's rows, relative to r0
  if (col < p.d && w0 < w1) {
    const uint16_t* src = p.Wd + static_cast<size_t>(r0 + w0) * p.d + col;
    const int cnt = w1 - w0;
    uint4 w[kGemvRing];
#pragma unroll
    for (int i = 0; i < kGemvRing; ++i)
      if (i < cnt) w[i] = ldg_nc_v4(src + static_cast<size_t>(i) * p.d);
    for (int base = 0; base < cnt; base += kGemvRing) {
#pragma unroll
      for (int i = 0; i < kGemvRing; ++i) {
        const int r = base + i;
        if (r < cnt) {
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < n) axpy8(a[t], hs[t][w0 + r], w[i]);
          if (r + kGemvRing < cnt) w[i] = ldg_nc_v4(src + static_cast<size_t>(r + kGemvRing) * p.d);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
    if (t < n) {
#pragma unroll
      for (int i = 0; i < 8; ++i) atomicAdd(&acc_s[t][i * 32 + lane], a[t][i]);
    }
  __syncthreads();
  // threads 0..n*64-1: token t = tid / 64, lane group: 4 columns each
  for (int e = threadIdx.x; e < n * 64; e += blockDim.x) {
    const int t = e / 64, q = e - t * 64;
    const int l = q >> 1, half = q & 1;  // lane l's columns 8l + 4 half .. + 3
    const int cc = c0 + l * 8 + half * 4;
    if (cc >= p.d) continue;
    const int row = p.rows != nullptr ? p.rows[t] : t;
    if (row < 0 || row >= p.T) continue;
    red_add_v4(p.y + static_cast<size_t>(row) * p.d + cc, acc_s[t][(half * 4 + 0) * 32 + l],
               acc_s[t][(half * 4 + 1) * 32 + l], acc_s[t][(half * 4 + 2) * 32 + l],
               acc_s[t][(half * 4 + 3) * 32 + l]);
  }
}

}  // namespace twell
