// Fused sparse step of the TwELL gated FFN, one warp per token:
//   for every stored slot (j, g) of row t:
//       u_j = x_t . Wu[:, j]          (fp32, reduced across the warp)
//       h_j = g * u_j                 (kept in a register, never stored)
//       y_t += h_j * Wd[j, :]         (fp32 accumulators in registers)
// then y_t is stored in fp32 (intellectnews.ru "Sakana AI и NVIDIA ...
// TwELL", section "Слитые CUDA-ядра для инференса и гибрид для обучения":
// several FFN steps in one pass, intermediates not written to global memory).
//
// Lane l owns the 8-element chunks l, l+32, l+64, ... of the d axis, so every
// gather of a weight row is a run of fully coalesced 16-byte loads. x_t and
// y_t live in registers for the whole row.
#pragma once

#include "ptx.cuh"

namespace twell {

struct SparseParams {
  const uint16_t* x;
  const uint16_t* WuT;
  const uint16_t* Wd;
  const int16_t* counts;
  const int16_t* idx;
  const uint16_t* vals;
  const uint8_t* row_ovf;
  float* y;
  int T, d, f, nT, W;
  int skip_ovf;
  int* dev_status;
};

constexpr int kSparseWarps = 8;

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float dot8(const uint4& a, const uint4& b, float acc) {
  acc = fmaf(bf16lo(a.x), bf16lo(b.x), acc);
  acc = fmaf(bf16hi(a.x), bf16hi(b.x), acc);
  acc = fmaf(bf16lo(a.y), bf16lo(b.y), acc);
  acc = fmaf(bf16hi(a.y), bf16hi(b.y), acc);
  acc = fmaf(bf16lo(a.z), bf16lo(b.z), acc);
  acc = fmaf(bf16hi(a.z), bf16hi(b.z), acc);
  acc = fmaf(bf16lo(a.w), bf16lo(b.w), acc);
  acc = fmaf(bf16hi(a.w), bf16hi(b.w), acc);
  return acc;
}

__device__ __forceinline__ void axpy8(float (&y)[8], float h, const uint4& w) {
  y[0] = fmaf(h, bf16lo(w.x), y[0]);
  y[1] = fmaf(h, bf16hi(w.x), y[1]);
  y[2] = fmaf(h, bf16lo(w.y), y[2]);
  y[3] = fmaf(h, bf16hi(w.y), y[3]);
  y[4] = fmaf(h, bf16lo(w.z), y[4]);
  y[5] = fmaf(h, bf16hi(w.z), y[5]);
  y[6] = fmaf(h, bf16lo(w.w), y[6]);
  y[7] = fmaf(h, bf16hi(w.w), y[7]);
}

template <int NCH>
__global__ void __launch_bounds__(kSparseWarps * 32) sparse_ffn_warp_kernel(const SparseParams p) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSparseWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  if (p.skip_ovf && p.row_ovf[t]) return;
  const int d = p.d;

  uint4 xr[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int k0 = (i * 32 + lane) * 8;
    xr[i] = (k0 < d) ? ldg_nc_v4(p.x + static_cast<size_t>(t) * d + k0) : make_uint4(0, 0, 0, 0);
  }
  float y[NCH][8];
#pragma unroll
  for (int i = 0; i < NCH; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) y[i][e] = 0.0f;

  bool overflow = false, bad_index = false;
  const int16_t* cnt_row = p.counts + static_cast<size_t>(t) * p.nT;
#pragma unroll 1
  for (int c = 0; c < p.nT; ++c) {
    const int cnt = cnt_row[c];
    if (cnt > p.W) overflow = true;
    const int n = min(max(cnt, 0), p.W);
    const size_t slot0 = (static_cast<size_t>(t) * p.nT + c) * p.W;
#pragma unroll 1
    for (int s0 = 0; s0 < n; s0 += 32) {
      int my_j = 0;
      float my_g = 0.0f;
      if (s0 + lane < n) {
        my_j = p.idx[slot0 + s0 + lane];
        my_g = __uint_as_float(static_cast<uint32_t>(p.vals[slot0 + s0 + lane]) << 16);
      }
      const int ns = min(32, n - s0);
#pragma unroll 1
      for (int s = 0; s < ns; ++s) {
        const int j = __shfl_sync(0xffffffffu, my_j, s);
        const float g = __shfl_sync(0xffffffffu, my_g, s);
        if (static_cast<unsigned>(j) >= static_cast<unsigned>(p.f)) {
          bad_index = true;
          continue;
        }
        const uint16_t* wu = p.WuT + static_cast<size_t>(j) * d;
        const uint16_t* wd = p.Wd + static_cast<size_t>(j) * d;
        uint4 a[NCH], b[NCH];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int k0 = (i * 32 + lane) * 8;
          if (k0 < d) {
            a[i] = ldg_nc_v4(wu + k0);
            b[i] = ldg_nc_v4(wd + k0);
          } else {
            a[i] = make_uint4(0, 0, 0, 0);
            b[i] = make_uint4(0, 0, 0, 0);
          }
        }
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) acc = dot8(xr[i], a[i], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const float h = g * acc;
#pragma unroll
        for (int i = 0; i < NCH; ++i) axpy8(y[i], h, b[i]);
      }
    }
  }
  if (lane == 0) {
    if (overflow && !p.skip_ovf) raise_status(p.dev_status, kDevOverflow);
    if (bad_index) raise_status(p.dev_status, kDevIndex);
  }
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int k0 = (i * 32 + lane) * 8;
    if (k0 < d) {
      float4* dst = reinterpret_cast<float4*>(p.y + static_cast<size_t>(t) * d + k0);
      dst[0] = make_float4(y[i][0], y[i][1], y[i][2], y[i][3]);
      dst[1] = make_float4(y[i][4], y[i][5], y[i][6], y[i][7]);
    }
  }
}

// ---------------------------------------------------------------- routing

// Ascending list of the rows whose overflow flag is set, and its length. One
// block of 1024 threads scans the flags in order, so the list is deterministic.
__global__ void __launch_bounds__(1024) route_kernel(const uint8_t* row_ovf, int T, int* ovf_rows, int* n_ovf) {
  __shared__ int warp_off[32];
  __shared__ int total_s;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int base = 0;
  for (int start = 0; start < T; start += 1024) {
    const int t = start + threadIdx.x;
    const int flag = (t < T && row_ovf[t] != 0) ? 1 : 0;
    const uint32_t m = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_off[warp] = __popc(m);
    __syncthreads();
    if (warp == 0) {
      const int v = warp_off[lane];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      warp_off[lane] = incl - v;
      if (lane == 31) total_s = incl;
    }
    __syncthreads();
    if (flag) ovf_rows[base + warp_off[warp] + __popc(m & ((1u << lane) - 1u))] = t;
    base += total_s;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_ovf = base;
}

// out[i, :] = x[rows[i], :] for i < *n_rows (clamped to T, the room in rows and out).
__global__ void gather_rows_kernel(const uint16_t* x, int d, const int* rows, const int* n_rows, int T,
                                   uint16_t* out, int* dev_status) {
  const int n = min(max(*n_rows, 0), T);
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int r = rows[i];
    if (r < 0 || r >= T) {
      if (threadIdx.x == 0) raise_status(dev_status, kDevIndex);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * d);
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i) * d);
    for (int k = threadIdx.x; k < d / 8; k += blockDim.x) dst[k] = src[k];
  }
}

// TwELL -> dense bf16: one warp per (row, tile) writes the tile's 128 columns
// as zeros, then scatters the stored slots.
__global__ void __launch_bounds__(256) unpack_kernel(const int16_t* counts, const int16_t* idx, const uint16_t* vals,
                                                     int T, int nT, int W, int f, uint16_t* g, int* dev_status) {
  const int lane = threadIdx.x & 31;
  const long long wid = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (wid >= static_cast<long long>(T) * nT) return;
  const int t = static_cast<int>(wid / nT);
  const int c = static_cast<int>(wid - static_cast<long long>(t) * nT);
  uint16_t* row = g + static_cast<size_t>(t) * f + static_cast<size_t>(c) * 128;
  *reinterpret_cast<uint2*>(row + lane * 4) = make_uint2(0u, 0u);
  __syncwarp();
  const int n = min(max(static_cast<int>(counts[wid]), 0), W);
  bool bad = false;
  for (int s = lane; s < n; s += 32) {
    const int j = idx[wid * W + s] - c * 128;
    if (j < 0 || j >= 128) {
      bad = true;
      continue;
    }
    row[j] = vals[wid * W + s];
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(dev_status, kDevIndex);
}

}  // namespace twell
