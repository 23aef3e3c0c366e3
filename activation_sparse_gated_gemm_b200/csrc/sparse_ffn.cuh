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
// gather of a weight row is a run of fully coalesced 16-byte loads.
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
  // Column tiles per work unit. A unit of all nT tiles stores y_t; smaller
  // units (used when T is small, to spread one token over several warps) add
  // their partial y_t into y, which must then hold zeros.
  int unit_tiles;
  // sparse_small_kernel only: when route_n is set, block (0, 0) also routes
  // the batch (T <= 8): route_flags[t] = (some tile of row t counts more than
  // W), route_rows = the flagged rows ascending, *route_n = their number.
  uint8_t* route_flags;
  int* route_rows;
  int* route_n;
  // sparse_ffn_warp_kernel: when set (a zeroed int), every warp of the grid
  // draws its next work unit from this one counter instead of from its
  // block's share, so that blocks whose tokens hold more slots do not set the
  // kernel's end.
  int* work_next;
  int* dev_status;
};

// Warps per block of the sparse kernel, as many as the register budget of one
// block per SM allows: the up+down kernel holds x chunks, y and two weight
// rows; the down-only kernel needs no x.
constexpr int sparse_warps_for(int nch, bool down_only) {
  return down_only ? (nch <= 6 ? 16 : (nch <= 9 ? 12 : 8)) : (nch <= 6 ? 12 : 8);
}

// Read-only 16-byte load through the non-coherent path. Left as an ordinary
// (non-volatile) operation so the compiler may issue it as early as its
// address is known.
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// y[2k], y[2k+1] += h * (w_lo, w_hi) with one packed fp32x2 fma per pair.
__device__ __forceinline__ void ffma2(float& y0, float& y1, float h, uint32_t w) {
  asm("{\n\t.reg .b64 yy, hh, ww;\n\t"
      "mov.b64 yy, {%0, %1};\n\t"
      "mov.b64 hh, {%2, %2};\n\t"
      "mov.b64 ww, {%3, %4};\n\t"
      "fma.rn.f32x2 yy, hh, ww, yy;\n\t"
      "mov.b64 {%0, %1}, yy;\n\t}"
      : "+f"(y0), "+f"(y1)
      : "f"(h), "f"(__uint_as_float(w << 16)), "f"(__uint_as_float(w & 0xffff0000u)));
}
__device__ __forceinline__ void axpy8(float (&y)[8], float h, const uint4& w) {
  ffma2(y[0], y[1], h, w.x);
  ffma2(y[2], y[3], h, w.y);
  ffma2(y[4], y[5], h, w.z);
  ffma2(y[6], y[7], h, w.w);
}

// acc += sum over 8 bf16 pairs of a_i * b_i, each product exact and added with
// one rounding (mixed-precision fma with bf16 sources and an fp32 addend).
__device__ __forceinline__ void mixdot8(const uint4& a, const uint4& b, float& acc0, float& acc1) {
  asm("{\n\t.reg .b16 a0, a1, a2, a3, a4, a5, a6, a7, b0, b1, b2, b3, b4, b5, b6, b7;\n\t"
      "mov.b32 {a0, a1}, %2; mov.b32 {a2, a3}, %3; mov.b32 {a4, a5}, %4; mov.b32 {a6, a7}, %5;\n\t"
      "mov.b32 {b0, b1}, %6; mov.b32 {b2, b3}, %7; mov.b32 {b4, b5}, %8; mov.b32 {b6, b7}, %9;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %0; fma.rn.f32.bf16 %1, a1, b1, %1;\n\t"
      "fma.rn.f32.bf16 %0, a2, b2, %0; fma.rn.f32.bf16 %1, a3, b3, %1;\n\t"
      "fma.rn.f32.bf16 %0, a4, b4, %0; fma.rn.f32.bf16 %1, a5, b5, %1;\n\t"
      "fma.rn.f32.bf16 %0, a6, b6, %0; fma.rn.f32.bf16 %1, a7, b7, %1;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w));
}

// y[0..8) += h * w[0..8) with h and w in bf16: mixed-precision fma (exact
// bf16 x bf16 product, one fp32 rounding), no unpacking of w.
__device__ __forceinline__ void axpy8_bf16(float (&y)[8], uint16_t h, const uint4& w) {
  asm("{\n\t.reg .b16 w0, w1, w2, w3, w4, w5, w6, w7;\n\t"
      "mov.b32 {w0, w1}, %9; mov.b32 {w2, w3}, %10; mov.b32 {w4, w5}, %11; mov.b32 {w6, w7}, %12;\n\t"
      "fma.rn.f32.bf16 %0, %8, w0, %0; fma.rn.f32.bf16 %1, %8, w1, %1;\n\t"
      "fma.rn.f32.bf16 %2, %8, w2, %2; fma.rn.f32.bf16 %3, %8, w3, %3;\n\t"
      "fma.rn.f32.bf16 %4, %8, w4, %4; fma.rn.f32.bf16 %5, %8, w5, %5;\n\t"
      "fma.rn.f32.bf16 %6, %8, w6, %6; fma.rn.f32.bf16 %7, %8, w7, %7;\n\t}"
      : "+f"(y[0]), "+f"(y[1]), "+f"(y[2]), "+f"(y[3]), "+f"(y[4]), "+f"(y[5]), "+f"(y[6]), "+f"(y[7])
      : "h"(h), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w));
}

template <int NCH>
__device__ __forceinline__ void load_row(uint4 (&w)[NCH], const uint16_t* row, int lane, int d) {
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int k0 = (i * 32 + lane) * 8;
    w[i] = (k0 < d) ? ldg_nc_v4(row + k0) : make_uint4(0, 0, 0, 0);
  }
}

// Stored slots of one token, flattened: entry = column index | bf16 value << 16.
constexpr int kListCap = 1024;  // entries per warp; a group of kListCap / W tiles always fits

__device__ __forceinline__ float entry_g(uint32_t e) { return __uint_as_float(e & 0xffff0000u); }
__device__ __forceinline__ int entry_j(uint32_t e) { return static_cast<int>(e & 0xffffu); }

// Persistent blocks, one per SM, each walking a contiguous range of tokens
// with its warps drawing tokens from a shared counter. Per token, x_t is parked in shared memory and y_t (fp32) stays in
// registers. The token's stored slots are first copied, tile group by tile
// group, into a flat list in shared memory (counts of 32 tiles per load, a warp
// prefix sum for the offsets, 16-byte slot loads), so no dependent load chain
// is paid per tile. The list is then consumed in batches of 32 entries in two
// passes: every u_j = x_t . Wu[:, j] (lane s keeps h_s = g_s * u_s), then every
// y_t += h_s * Wd[j_s, :]. In both passes two weight rows alternate, so the
// gather of entry s+1 is in flight while entry s is computed.
//
// DOWN_ONLY: the stored values already are the hidden activations h (the up
// projection ran on the tensor cores); only the second pass runs and x is not
// read.
template <int NCH, int WARPS, bool DOWN_ONLY>
__global__ void __launch_bounds__(WARPS * 32, 1) sparse_ffn_warp_kernel(const SparseParams p) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ uint4 smem_dyn[];  // xs: [WARPS][NCH * 32] uint4, then lists
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int d = p.d;
  uint4* xs = smem_dyn + warp * NCH * 32;
  uint32_t* list = reinterpret_cast<uint32_t*>(smem_dyn + WARPS * NCH * 32) + warp * kListCap;
  const int group_tiles = max(1, kListCap / p.W);
  bool overflow = false, bad_index = false;
  // x_t, y_t and the pack pass through once: evict them first, keep the weight rows
  const uint64_t stream_pol = l2_evict_first_policy();
  // Block b owns the contiguous tokens [t_begin, t_end); its warps take them
  // one at a time from a shared counter, so a warp that drew light tokens
  // keeps working while another finishes a heavy one. With work_next every
  // warp of the grid takes them from that one counter instead.
  __shared__ int next_unit;
  const int units_per_token = (p.nT + p.unit_tiles - 1) / p.unit_tiles;
  const bool partial = units_per_token > 1;
  const long long n_units = static_cast<long long>(p.T) * units_per_token;
  const int u_begin = static_cast<int>(n_units * blockIdx.x / gridDim.x);
  const int u_end = p.work_next != nullptr ? static_cast<int>(n_units)
                                           : static_cast<int>(n_units * (blockIdx.x + 1) / gridDim.x);
  if (threadIdx.x == 0) next_unit = u_begin;
  __syncthreads();
#pragma unroll 1
  for (;;) {
    int u = 0;
    if (lane == 0) u = p.work_next != nullptr ? atomicAdd(p.work_next, 1) : atomicAdd(&next_unit, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= u_end) break;
    const int t = u / units_per_token;
    const int c_first = (u - t * units_per_token) * p.unit_tiles;
    const int c_last = min(p.nT, c_first + p.unit_tiles);
    if (p.skip_ovf && p.row_ovf[t]) continue;
    __syncwarp();
    if (!DOWN_ONLY) {
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int k0 = (i * 32 + lane) * 8;
        xs[i * 32 + lane] = (k0 < d) ? ldg_stream_v4(p.x + static_cast<size_t>(t) * d + k0, stream_pol)
                                     : make_uint4(0, 0, 0, 0);
      }
    }
    float y[NCH][8];
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) y[i][e] = 0.0f;

#pragma unroll 1
    for (int c0 = c_first; c0 < c_last; c0 += group_tiles) {
      const int c1 = min(c_last, c0 + group_tiles);
      // ---- flatten the slots of tiles [c0, c1) into list[0, total)
      int total = 0;
#pragma unroll 1
      for (int cb = c0; cb < c1; cb += 32) {
        const int c = cb + lane;
        int n = 0;
        if (c < c1) {
          const int cnt = p.counts[static_cast<size_t>(t) * p.nT + c];
          if (cnt > p.W) overflow = true;
          n = min(max(cnt, 0), p.W);
        }
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int off = total + incl - n;
        total += __shfl_sync(0xffffffffu, incl, 31);
        const size_t base = (static_cast<size_t>(t) * p.nT + c) * p.W;
        for (int k = 0; k < n; k += 8) {
          // 8 slots at a time; slots past n are read but not used (k + 8 <= W)
          const uint4 iv = ldg_stream_v4(p.idx + base + k, stream_pol);
          const uint4 vv = ldg_stream_v4(p.vals + base + k, stream_pol);
          const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
          const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (k + e < n) {
              const uint32_t jj = (e & 1) ? (iw[e >> 1] >> 16) : (iw[e >> 1] & 0xffffu);
              const uint32_t gg = (e & 1) ? (vw[e >> 1] & 0xffff0000u) : (vw[e >> 1] << 16);
              uint32_t ent = jj | gg;
              if (static_cast<int>(static_cast<int16_t>(jj)) < 0 || static_cast<int>(jj) >= p.f) {
                bad_index = true;
                ent = 0;  // column 0 with value 0: contributes nothing
              }
              list[off + k + e] = ent;
            }
          }
        }
      }
      __syncwarp();
      // ---- consume the list
#pragma unroll 1
      for (int s0 = 0; s0 < total; s0 += 32) {
        const int ns = min(32, total - s0);
        const uint32_t my_e = (lane < ns) ? list[s0 + lane] : 0u;
        const int my_j = entry_j(my_e);
        const float my_g = entry_g(my_e);
        // pass 1: up projections
        float my_h = DOWN_ONLY ? my_g : 0.0f;
        uint4 wa[NCH], wb[NCH];
        if (!DOWN_ONLY)
          load_row<NCH>(wa, p.WuT + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, 0)) * d, lane, d);
#pragma unroll 1
        for (int s = 0; s < (DOWN_ONLY ? 0 : ns); s += 2) {
          if (s + 1 < ns)
            load_row<NCH>(wb, p.WuT + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 1)) * d, lane, d);
          {
            float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
            for (int i = 0; i < NCH; i += 2) {
              mixdot8(xs[i * 32 + lane], wa[i], a0, a1);
              if (i + 1 < NCH) mixdot8(xs[(i + 1) * 32 + lane], wa[i + 1], a2, a3);
            }
            float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == s) my_h = my_g * acc;
          }
          if (s + 1 < ns) {
            if (s + 2 < ns)
              load_row<NCH>(wa, p.WuT + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 2)) * d, lane, d);
            float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
            for (int i = 0; i < NCH; i += 2) {
              mixdot8(xs[i * 32 + lane], wb[i], a0, a1);
              if (i + 1 < NCH) mixdot8(xs[(i + 1) * 32 + lane], wb[i + 1], a2, a3);
            }
            float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == s + 1) my_h = my_g * acc;
          }
        }
        // pass 2: down projection, h never leaves the registers. When the
        // stored value already is h (a bf16), the mixed-precision fma takes it
        // and the bf16 weights directly.
        const uint32_t my_hb = my_e >> 16;
        load_row<NCH>(wa, p.Wd + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, 0)) * d, lane, d);
#pragma unroll 1
        for (int s = 0; s < ns; s += 2) {
          if (s + 1 < ns)
            load_row<NCH>(wb, p.Wd + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 1)) * d, lane, d);
          if (DOWN_ONLY) {
            const uint16_t hb = static_cast<uint16_t>(__shfl_sync(0xffffffffu, my_hb, s));
#pragma unroll
            for (int i = 0; i < NCH; ++i) axpy8_bf16(y[i], hb, wa[i]);
          } else {
            const float h = __shfl_sync(0xffffffffu, my_h, s);
#pragma unroll
            for (int i = 0; i < NCH; ++i) axpy8(y[i], h, wa[i]);
          }
          if (s + 1 < ns) {
            if (s + 2 < ns)
              load_row<NCH>(wa, p.Wd + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 2)) * d, lane, d);
            if (DOWN_ONLY) {
              const uint16_t hb = static_cast<uint16_t>(__shfl_sync(0xffffffffu, my_hb, s + 1));
#pragma unroll
              for (int i = 0; i < NCH; ++i) axpy8_bf16(y[i], hb, wb[i]);
            } else {
              const float h = __shfl_sync(0xffffffffu, my_h, s + 1);
#pragma unroll
              for (int i = 0; i < NCH; ++i) axpy8(y[i], h, wb[i]);
            }
          }
        }
      }
      __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int k0 = (i * 32 + lane) * 8;
      if (k0 < d) {
        float* dst = p.y + static_cast<size_t>(t) * d + k0;
        if (partial) {
          red_add_stream_v4(dst, y[i][0], y[i][1], y[i][2], y[i][3], stream_pol);
          red_add_stream_v4(dst + 4, y[i][4], y[i][5], y[i][6], y[i][7], stream_pol);
        } else {
          st_stream_v4(dst, y[i][0], y[i][1], y[i][2], y[i][3], stream_pol);
          st_stream_v4(dst + 4, y[i][4], y[i][5], y[i][6], y[i][7], stream_pol);
        }
      }
    }
  }
  // each lane saw the counts of its own tiles
  if (__any_sync(0xffffffffu, overflow) && lane == 0 && !p.skip_ovf) raise_status(p.dev_status, kDevOverflow);
  if (__any_sync(0xffffffffu, bad_index) && lane == 0) raise_status(p.dev_status, kDevIndex);
}

// The sparse step of a batch of at most 8 tokens (d a multiple of 256): one
// warp per stored slot, so that a token's few slots are all in flight at once
// instead of queueing behind one another in the warps of its column tiles.
// Block (b, t) takes slots b*8 + warp, stepping by gridDim.x * 8, of token t
// (numbered across its tiles by a prefix of the stored counts); a warp loads
// the slot's Wd row (and, for the gate form, its WuT row, u = x_t . Wu[:, j]
// and h = g u), adds h Wd[j, :] into the block's copy of y_t in shared memory,
// and the block adds that copy into y (which holds zeros in the rows written).
// A token with a tile above W is left to the dense branch when skip_ovf is
// set (found from its counts here); block (0, 0) also writes the routing of
// the batch when asked, which saves the routing launch.
constexpr int kSmallSparseWarps = 8;
constexpr int kSmallSparseMaxTiles = 256;  // f <= 32767

template <int NCH, bool DOWN_ONLY>
__global__ void __launch_bounds__(kSmallSparseWarps * 32) sparse_small_kernel(const SparseParams p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int pre[kSmallSparseMaxTiles + 1];
  __shared__ int over_s;
  __shared__ float ys[NCH * 256];  // y_t, element (i*32 + l)*8 + e at i*256 + e*32 + l
  __shared__ uint4 xs[DOWN_ONLY ? 1 : NCH * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.y;
  // x_t and the zeroed copy of y_t do not wait for the counts
  if (!DOWN_ONLY)
    for (int e = threadIdx.x; e < NCH * 32; e += blockDim.x)
      xs[e] = ldg_nc_v4(p.x + static_cast<size_t>(t) * p.d + e * 8);
  for (int e = threadIdx.x; e < NCH * 256; e += blockDim.x) ys[e] = 0.0f;
  bool bad_index = false;
  if (warp == 0) {
    bool overflow = false;
    int run = 0;
    for (int cb = 0; cb < p.nT; cb += 32) {
      const int c = cb + lane;
      int n = 0;
      if (c < p.nT) {
        const int cnt = p.counts[static_cast<size_t>(t) * p.nT + c];
        if (cnt > p.W) overflow = true;
        n = min(max(cnt, 0), p.W);
      }
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (c < p.nT) pre[c] = run + incl - n;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    overflow = __any_sync(0xffffffffu, overflow);
    if (lane == 0) {
      pre[p.nT] = run;
      over_s = overflow ? 1 : 0;
      if (overflow && !p.skip_ovf) raise_status(p.dev_status, kDevOverflow);
    }
  } else if (warp == 1 && p.route_n != nullptr && blockIdx.x == 0 && t == 0) {
    int n_over = 0;
    for (int r = 0; r < p.T; ++r) {
      bool o = false;
      for (int c = lane; c < p.nT; c += 32) o |= p.counts[static_cast<size_t>(r) * p.nT + c] > p.W;
      o = __any_sync(0xffffffffu, o);
      if (lane == 0) {
        p.route_flags[r] = o ? 1 : 0;
        if (o) p.route_rows[n_over] = r;
      }
      n_over += o ? 1 : 0;
    }
    if (lane == 0) *p.route_n = n_over;
  }
  __syncthreads();
  if (p.skip_ovf && over_s) return;  // the dense branch computes this row
  const int total = pre[p.nT];
  if (blockIdx.x * kSmallSparseWarps >= total) return;  // no slot for this block
  const int stride = gridDim.x * kSmallSparseWarps;
#pragma unroll 1
  for (int s = blockIdx.x * kSmallSparseWarps + warp; s < total; s += stride) {
    // the tile holding slot s: the last c with pre[c] <= s
    int lo = 0, hi = p.nT - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= s) lo = mid; else hi = mid - 1;
    }
    const size_t at = (static_cast<size_t>(t) * p.nT + lo) * p.W + (s - pre[lo]);
    const int j = p.idx[at];
    if (j < 0 || j >= p.f) {
      bad_index = true;
      continue;
    }
    const uint16_t gb = p.vals[at];
    uint4 wd[NCH];
    load_row<NCH>(wd, p.Wd + static_cast<size_t>(j) * p.d, lane, p.d);
    float h = __uint_as_float(static_cast<uint32_t>(gb) << 16);
    if (!DOWN_ONLY) {
      uint4 wu[NCH];
      load_row<NCH>(wu, p.WuT + static_cast<size_t>(j) * p.d, lane, p.d);
      float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
      for (int i = 0; i < NCH; ++i) mixdot8(xs[i * 32 + lane], wu[i], a0, a1);
      float u = a0 + a1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
      h *= u;
    }
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const uint32_t w4[4] = {wd[i].x, wd[i].y, wd[i].z, wd[i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float w = (e & 1) ? bf16hi(w4[e >> 1]) : bf16lo(w4[e >> 1]);
        atomicAdd(&ys[i * 256 + e * 32 + lane], h * w);
      }
    }
  }
  if (__any_sync(0xffffffffu, bad_index) && lane == 0) raise_status(p.dev_status, kDevIndex);
  __syncthreads();
  // y_t += the block's copy, four columns per thread and step
  float* yt = p.y + static_cast<size_t>(t) * p.d;
  for (int q = threadIdx.x; q < NCH * 64; q += blockDim.x) {
    const int k0 = q * 4;                    // columns k0..k0+3
    const int i = k0 >> 8, l = (k0 >> 3) & 31, e0 = k0 & 7;
    red_add_v4(yt + k0, ys[i * 256 + (e0 + 0) * 32 + l], ys[i * 256 + (e0 + 1) * 32 + l],
               ys[i * 256 + (e0 + 2) * 32 + l], ys[i * 256 + (e0 + 3) * 32 + l]);
  }
}

// The dense branch's hidden activations of the overflowing rows in the tiles
// that did not overflow: all of their nonzeros are in the pack (as bf16 h), so
// the slot's row of H gets them over zeros, with a zero remainder (the tiles
// that overflowed were written, exact, by the gate+up GEMM). Slot s holds row
// slot_row[s]; the slot's row of y is zeroed for the branch's partial sums.
// One warp per (slot, tile): its lanes load the tile's stored slots side by
// side into the tile's 128 units in shared memory, then lane l writes units
// 4l..4l+3.
__global__ void __launch_bounds__(256) ovf_fill_kernel(const int16_t* counts, const int16_t* idx, const uint16_t* vals,
                                                       int nT, int W, int f, const int* slot_row, const int* n_slots,
                                                       uint16_t* H, float* y, int d) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ __align__(16) uint16_t tile_h[8][128];
  const int lane = threadIdx.x & 31;
  uint16_t* th = tile_h[threadIdx.x >> 5];
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long n = static_cast<long long>(max(*n_slots, 0)) * nT;
  for (long long u = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n; u += warps) {
    const int sl = static_cast<int>(u / nT), c = static_cast<int>(u - static_cast<long long>(sl) * nT);
    const int t = slot_row[sl];
    if (c == 0) {
      float4* yr = reinterpret_cast<float4*>(y + static_cast<size_t>(t) * d);
      for (int k = lane; k < d / 4; k += 32) yr[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const size_t at = static_cast<size_t>(t) * nT + c;
    const int cnt = counts[at];
    if (cnt > W) continue;  // written by the gate+up GEMM (warp-uniform)
    *reinterpret_cast<uint2*>(th + 4 * lane) = make_uint2(0u, 0u);
    __syncwarp();
    for (int k = lane; k < cnt; k += 32) {
      const int j = static_cast<int>(idx[at * W + k]) - c * 128;
      if (j >= 0 && j < 128) th[j] = vals[at * W + k];
    }
    __syncwarp();
    const uint2 h = *reinterpret_cast<const uint2*>(th + 4 * lane);
    __syncwarp();  // the next pair's zeros overwrite these units
    uint16_t* hrow = H + static_cast<size_t>(sl) * 2 * f;
    *reinterpret_cast<uint2*>(hrow + c * 128 + 4 * lane) = h;
    *reinterpret_cast<uint2*>(hrow + f + c * 128 + 4 * lane) = make_uint2(0u, 0u);
  }
}

// y[t, :] = 0 for the rows the sparse step will write (all rows, or those
// without the overflow flag when overflow rows are skipped).
__global__ void zero_rows_kernel(float* y, int T, int d, const uint8_t* row_ovf, int skip_ovf) {
  griddep_launch_dependents();
  griddep_wait();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    if (skip_ovf && row_ovf[t]) continue;
    float4* row = reinterpret_cast<float4*>(y + static_cast<size_t>(t) * d);
    for (int k = threadIdx.x; k < d / 4; k += blockDim.x) row[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ---------------------------------------------------------------- routing

// Ascending list of the rows whose overflow flag is set, and its length. One
// block of 1024 threads; per round each thread owns 16 consecutive flags
// (read with one 16-byte load when they are in range), counts its own, and a
// block-wide scan gives every thread the position of its first flagged row,
// so the list comes out in ascending order.
//
// With xo given (small batches), the same block then gathers the listed rows
// of x into xo and zeroes them in y_zero, which saves the separate gather
// launch of the dense branch.
__global__ void __launch_bounds__(1024) route_kernel(const uint8_t* row_ovf, int T, int* ovf_rows, int* n_ovf,
                                                     const uint16_t* x, int d, uint16_t* xo, float* y_zero) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int warp_off[32];
  __shared__ int total_s;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const bool vec_ok = (reinterpret_cast<uintptr_t>(row_ovf) & 15u) == 0;
  int base = 0;
  for (int start = 0; start < T; start += 1024 * 16) {
    const int t0 = start + threadIdx.x * 16;
    uint32_t bits = 0;  // bit k: row t0 + k is flagged
    if (vec_ok && t0 + 16 <= T) {
      const uint4 v = *reinterpret_cast<const uint4*>(row_ovf + t0);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 16; ++k) bits |= ((w[k >> 2] >> (8 * (k & 3))) & 0xffu ? 1u : 0u) << k;
    } else {
      for (int k = 0; k < 16; ++k)
        if (t0 + k < T && row_ovf[t0 + k] != 0) bits |= 1u << k;
    }
    const int mine = __popc(bits);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_off[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = warp_off[lane];
      int wi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      warp_off[lane] = wi - v;
      if (lane == 31) total_s = wi;
    }
    __syncthreads();
    int pos = base + warp_off[warp] + incl - mine;
    while (bits != 0) {
      const int k = __ffs(bits) - 1;
      bits &= bits - 1u;
      ovf_rows[pos++] = t0 + k;
    }
    base += total_s;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_ovf = base;
  if (xo == nullptr) return;
  __syncthreads();  // the list written above is read back by the whole block
  const int vecs = d / 8;
  for (int e = threadIdx.x; e < base * vecs; e += 1024) {
    const int i = e / vecs, k = e - i * vecs;
    const int r = ovf_rows[i];
    reinterpret_cast<uint4*>(xo + static_cast<size_t>(i) * d)[k] =
        reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * d)[k];
    float4* yz = reinterpret_cast<float4*>(y_zero + static_cast<size_t>(r) * d);
    yz[2 * k] = make_float4(0.f, 0.f, 0.f, 0.f);
    yz[2 * k + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// out[i, :] = x[rows[i], :] for i < *n_rows (clamped to T, the room in rows and
// out); when y_zero is given, also y_zero[rows[i], :] = 0 (the dense branch may
// add split partial sums into those rows). With pad_rows > 0 (the room in out,
// at least T), rows from n up to the next multiple of 64 are zeroed, so a
// GEMM whose K runs over out's rows in blocks of 64 reads zeros past n.
__global__ void gather_rows_kernel(const uint16_t* x, int d, const int* rows, const int* n_rows, int T,
                                   uint16_t* out, float* y_zero, int* dev_status, int pad_rows = 0) {
  griddep_launch_dependents();
  griddep_wait();
  const int n = min(max(*n_rows, 0), T);
  if (pad_rows > 0) {
    const int pad_end = min((n + 63) / 64 * 64, pad_rows);
    for (int i = n + blockIdx.x; i < pad_end; i += gridDim.x) {
      uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i) * d);
      for (int k = threadIdx.x; k < d / 8; k += blockDim.x) dst[k] = make_uint4(0, 0, 0, 0);
    }
  }
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int r = rows[i];
    if (r < 0 || r >= T) {
      if (threadIdx.x == 0) raise_status(dev_status, kDevIndex);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * d);
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i) * d);
    for (int k = threadIdx.x; k < d / 8; k += blockDim.x) dst[k] = src[k];
    if (y_zero != nullptr) {
      float4* yz = reinterpret_cast<float4*>(y_zero + static_cast<size_t>(r) * d);
      for (int k = threadIdx.x; k < d / 4; k += blockDim.x) yz[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// TwELL -> dense bf16: one warp per (row, tile) writes the tile's 128 columns
// as zeros, then scatters the stored slots.
__global__ void __launch_bounds__(256) unpack_kernel(const int16_t* counts, const int16_t* idx, const uint16_t* vals,
                                                     int T, int nT, int W, int f, uint16_t* g, int* dev_status) {
  griddep_launch_dependents();
  griddep_wait();
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

// ---------------------------------------------------------------- union of a row tile

// Per tile of 128 rows (one block): the hidden units that the tile's rows that
// fit (overflow rows skipped when skip_ovf) activate -- the union of their
// stored columns -- in ascending order, and the tile's hidden values over that
// union, for the down projection on the tensor cores (kModeUnion):
//   kb_tile[m]                 K blocks of 64 the tile runs (>= 1)
//   union_rows[m][0..64 kb)    the union, padded with unit 0
//   H[128 m + r][0..64 kb)     bf16 hidden value of row r at each union unit, 0 elsewhere
// (row stride `stride` for both). A stored index outside its own column tile
// raises TWELL_ERR_INDEX and is left out; a count above W raises
// TWELL_ERR_OVERFLOW unless overflow rows are skipped.
struct UnionParams {
  const int16_t* counts;
  const int16_t* idx;
  const uint16_t* vals;
  const uint8_t* row_ovf;
  int T, f, nT, W, skip_ovf;
  int* kb_tile;
  int* union_rows;
  uint16_t* H;
  int stride;
  int* dev_status;
};

__global__ void __launch_bounds__(256) union_prep_kernel(const UnionParams p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint32_t bits[1024];  // f <= 32767: at most 1024 words
  __shared__ int wpre[1024];
  __shared__ int warp_sum[8];
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = p.f / 32;
  const int t0 = m * 128;
  for (int w = tid; w < nwords; w += blockDim.x) bits[w] = 0u;
  __syncthreads();
  bool bad = false, overflow = false;
  // 1. the union: one thread per (row, column tile)
  for (int i = tid; i < 128 * p.nT; i += blockDim.x) {
    const int r = i / p.nT, c = i - r * p.nT;
    const int t = t0 + r;
    if (t >= p.T || (p.skip_ovf && p.row_ovf[t])) continue;
    const size_t at = static_cast<size_t>(t) * p.nT + c;
    if (p.counts[at] > p.W) overflow = true;
    const int n = min(max(static_cast<int>(p.counts[at]), 0), p.W);
    for (int s = 0; s < n; ++s) {
      const int j = p.idx[at * p.W + s];
      if (j < c * 128 || j >= c * 128 + 128) {
        bad = true;
        continue;
      }
      atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  // 2. exclusive prefix of the words' popcounts (each thread a run of words)
  const int per = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bits[w]);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
  for (int k = 0; k < static_cast<int>(blockDim.x / 32); ++k) {
    before += k < warp ? warp_sum[k] : 0;
    total += warp_sum[k];
  }
  int run = before + incl - mine;
  for (int w = w0; w < w1; ++w) {
    wpre[w] = run;
    run += __popc(bits[w]);
  }
  const int kb = max(1, (total + 63) / 64);
  const int kpad = kb * 64;
  if (tid == 0) p.kb_tile[m] = kb;
  // 3. the union list, padded with unit 0
  int* ur = p.union_rows + static_cast<size_t>(m) * p.stride;
  for (int w = w0; w < w1; ++w) {
    uint32_t b = bits[w];
    int pos = wpre[w];
    while (b != 0u) {
      const int k = __ffs(b) - 1;
      b &= b - 1u;
      ur[pos++] = w * 32 + k;
    }
  }
  for (int i = total + tid; i < kpad; i += blockDim.x) ur[i] = 0;
  // 4. the tile's hidden values over the union: zeros, then the stored slots
  uint16_t* hb = p.H + static_cast<size_t>(t0) * p.stride;
  const int vpr = kpad / 8;  // 16-byte vectors per row
  for (int i = tid; i < 128 * vpr; i += blockDim.x) {
    const int r = i / vpr, v = i - r * vpr;
    reinterpret_cast<uint4*>(hb + static_cast<size_t>(r) * p.stride)[v] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();  // every zero is written before any value lands on it
  for (int i = tid; i < 128 * p.nT; i += blockDim.x) {
    const int r = i / p.nT, c = i - r * p.nT;
    const int t = t0 + r;
    if (t >= p.T || (p.skip_ovf && p.row_ovf[t])) continue;
    const size_t at = static_cast<size_t>(t) * p.nT + c;
    const int n = min(max(static_cast<int>(p.counts[at]), 0), p.W);
    for (int s = 0; s < n; ++s) {
      const int j = p.idx[at * p.W + s];
      if (j < c * 128 || j >= c * 128 + 128) continue;
      const int pos = wpre[j >> 5] + __popc(bits[j >> 5] & ((1u << (j & 31)) - 1u));
      hb[static_cast<size_t>(r) * p.stride + pos] = p.vals[at * p.W + s];
    }
  }
  if (__syncthreads_or(bad) && tid == 0) raise_status(p.dev_status, kDevIndex);
  if (__syncthreads_or(overflow) && tid == 0 && !p.skip_ovf) raise_status(p.dev_status, kDevOverflow);
}

// ---------------------------------------------------------------- compaction

// One block of 1024 threads (f / 32 <= 1024 bitmap words): col_map[0..f_live)
// = the set bits of `active` in ascending order, col_map[f_live..f) = -1,
// *f_live = their number.
__global__ void __launch_bounds__(1024) compact_columns_kernel(const uint32_t* __restrict__ active, int f,
                                                                int32_t* __restrict__ col_map,
                                                                int32_t* __restrict__ f_live) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int warp_sums[32];
  __shared__ int s_total;
  const int nwords = (f + 31) / 32;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint32_t bits = tid < nwords ? active[tid] : 0u;
  if (tid == nwords - 1 && (f & 31)) bits &= (1u << (f & 31)) - 1u;
  const int n = __popc(bits);
  int incl = n;  // inclusive scan of the popcounts within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {  // warp totals -> exclusive prefixes
    const int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    warp_sums[lane] = wi - w;
  }
  __syncthreads();
  int pos = warp_sums[wid] + incl - n;
  if (tid == 1023) s_total = warp_sums[31] + incl;
  while (bits != 0) {
    const int b = __ffs(bits) - 1;
    bits &= bits - 1u;
    col_map[pos++] = tid * 32 + b;
  }
  __syncthreads();
  for (int i = s_total + tid; i < f; i += 1024) col_map[i] = -1;
  if (tid == 0) *f_live = s_total;
}

// out[i] = W[col_map[i]] for i < min(*f_live, f_out), zero rows after; one
// warp per row, 16-byte copies (d % 64 == 0). Map entries outside [0, f)
// raise TWELL_ERR_INDEX and give a zero row.
__global__ void gather_weight_rows_kernel(const uint16_t* __restrict__ W, int f, int d,
                                          const int32_t* __restrict__ col_map, const int32_t* __restrict__ f_live,
                                          int f_out, uint16_t* __restrict__ out, int* dev_status) {
  griddep_launch_dependents();
  griddep_wait();
  const int n_live = min(max(*f_live, 0), f_out);
  const int lane = threadIdx.x & 31;
  const int vecs = d / 8;  // uint4 per row
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < f_out;
       row += (gridDim.x * blockDim.x) >> 5) {
    int src = -1;
    if (row < n_live) {
      src = col_map[row];
      if (src < 0 || src >= f) {
        if (lane == 0) raise_status(dev_status, kDevIndex);
        src = -1;
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * d);
    if (src < 0) {
      for (int v = lane; v < vecs; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
    } else {
      const uint4* s4 = reinterpret_cast<const uint4*>(W + static_cast<size_t>(src) * d);
      for (int v = lane; v < vecs; v += 32) dst[v] = __ldg(s4 + v);
    }
  }
}

// ---------------------------------------------------------------- small batches

// TwELL pack from fp32 gate pre-activations z [T][f] (the split-K gate GEMM of
// a small batch): one warp per (row, tile), lane l holding columns 4l..4l+3 of
// the tile; the positive ones are placed in ascending column order by a warp
// prefix sum of the per-lane counts. Same output as the GEMM epilogue: the
// true count, the first W (column, bf16 value) slots, the overflow flag (set
// only; row_ovf must start at zero). When y_zero is given, its T x d entries
// are zeroed first (for the sparse step's split-unit partial sums).
__global__ void __launch_bounds__(256) pack_f32_kernel(const float* __restrict__ z, int T, int f, int W,
                                                       int16_t* __restrict__ counts, int16_t* __restrict__ idx,
                                                       uint16_t* __restrict__ vals, uint8_t* __restrict__ row_ovf,
                                                       float* __restrict__ y_zero, int d) {
  griddep_launch_dependents();
  griddep_wait();
  if (y_zero != nullptr) {
    const size_t n4 = static_cast<size_t>(T) * d / 4;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
      reinterpret_cast<float4*>(y_zero)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int nT = f / 128;
  const int lane = threadIdx.x & 31;
  const long long pairs = static_cast<long long>(T) * nT;
  for (long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); w < pairs;
       w += static_cast<long long>(gridDim.x) * 8) {
    const int t = static_cast<int>(w / nT);
    const int c = static_cast<int>(w - static_cast<long long>(t) * nT);
    const float4 v = reinterpret_cast<const float4*>(z + static_cast<size_t>(t) * f + c * 128)[lane];
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) m |= (vv[k] > 0.0f ? 1u : 0u) << k;
    const int n = __popc(m);
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int s = incl - n;
    const size_t slot0 = static_cast<size_t>(w) * W;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if ((m >> k) & 1u) {
        if (s < W) {
          idx[slot0 + s] = static_cast<int16_t>(c * 128 + 4 * lane + k);
          vals[slot0 + s] = f32_to_bf16_bits(vv[k]);
        }
        ++s;
      }
    }
    if (lane == 0) {
      counts[w] = static_cast<int16_t>(total);
      if (total > W) row_ovf[t] = 1;
    }
  }
}

// h [T][f] = bf16(ReLU(z) * u) from zu [T][2f] = [z | u] in fp32 (the first
// half of the dense layer for a small batch), or bf16(ReLU(z)) from z [T][f]
// when not gated.
__global__ void h_from_zu_kernel(const float* __restrict__ zu, int T, int f, int gated, uint16_t* __restrict__ h) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t per_row = static_cast<size_t>(f) / 4;
  const size_t n = static_cast<size_t>(T) * per_row;
  const size_t ldz = gated ? 2 * static_cast<size_t>(f) : static_cast<size_t>(f);
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t t = i / per_row, q = i - t * per_row;
    const float4 z = reinterpret_cast<const float4*>(zu + t * ldz)[q];
    const float4 u = gated ? reinterpret_cast<const float4*>(zu + t * ldz + f)[q] : make_float4(1.f, 1.f, 1.f, 1.f);
    uint2 o;
    o.x = pack_bf16x2(fmaxf(z.x, 0.f) * u.x, fmaxf(z.y, 0.f) * u.y);
    o.y = pack_bf16x2(fmaxf(z.z, 0.f) * u.z, fmaxf(z.w, 0.f) * u.w);
    reinterpret_cast<uint2*>(h + t * f)[q] = o;
  }
}

// ---------------------------------------------------------------- zeroing

// Up to three byte ranges set to zero by one launch (in place of memsets,
// which would interrupt the chain of dependent launches).
struct ZeroRanges {
  void* p[3];
  size_t n[3];
};

__global__ void zero_ranges_kernel(ZeroRanges r) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nth = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (int k = 0; k < 3; ++k) {
    uint8_t* b = static_cast<uint8_t*>(r.p[k]);
    const size_t n = r.n[k];
    if (b == nullptr || n == 0) continue;
    const size_t head = min(n, (16 - (reinterpret_cast<uintptr_t>(b) & 15)) & 15);
    const size_t body = (n - head) / 16;
    for (size_t i = tid; i < head; i += nth) b[i] = 0;
    uint4* b4 = reinterpret_cast<uint4*>(b + head);
    for (size_t i = tid; i < body; i += nth) b4[i] = make_uint4(0, 0, 0, 0);
    for (size_t i = head + body * 16 + tid; i < n; i += nth) b[i] = 0;
  }
}

}  // namespace twell
