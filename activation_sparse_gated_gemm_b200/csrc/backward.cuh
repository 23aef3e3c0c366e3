// Backward pass of the TwELL gated FFN through the hybrid format
// (intellectnews.ru "Sakana AI и NVIDIA ... TwELL", section "Слитые CUDA-ядра
// для инференса и гибрид для обучения": in training, rows that are sparse
// enough use the compact format, rows with many active units a dense branch).
//
// With g = ReLU(z), h = g * u and an upstream gradient dy:
//   dh_j = dy . Wd[j, :], du_j = dh_j g_j, dz_j = dh_j u_j   (only where z_j > 0)
//   dx   = sum_j dz_j Wg[:, j] + du_j Wu[:, j]
//   dWd[j, :] = sum_t h_tj dy_t, dWu[:, j] = sum_t du_tj x_t, dWg[:, j] = sum_t dz_tj x_t
//
// Rows that fit the ELL width take three passes over their stored units:
//   0. dh = dy . Wd^T and u = x . Wu^T on the tensor cores (plain dense
//      contractions: cheaper than gathering a Wd and a Wu row per slot), and
//      per stored slot the record {h, du, dz, token} from u_j, dh_j and the
//      stored g (in the GEMMs' epilogues, or by bwd_records_kernel from the
//      full products for small batches);
//   1b. per token (one warp per token, like the forward's fused kernel): dx_t
//      by two row axpys with du_j, dz_j from the records;
//   2. per hidden unit: the records are sorted by column (count, scan, scatter
//      of whole 16-byte records) and one warp per (unit, 256-wide slice of d)
//      reads its unit's records in order and sums h dy_t, du x_t, dz x_t into
//      the three weight-gradient rows.
// Rows that overflow take the dense branch on the tensor cores (the GEMM
// modes kModeZU, kModeBwdDh and kModeDown), which adds their share to the
// weight gradients afterwards.
#pragma once

#include "sparse_ffn.cuh"

namespace twell {

struct BwdParams {
  const uint16_t* x;   // [rows][d] bf16
  const uint16_t* WgT;
  const uint16_t* WuT;
  const float* dh;        // [rows][f] fp32: dy . Wd^T
  const int16_t* counts;  // TwELL of these rows (the forward's gate pack)
  const int16_t* idx;
  const uint16_t* vals;
  const uint8_t* row_ovf;  // rows with the flag set are skipped
  int rows;
  int d, f, nT, W;
  float* dx;      // [rows][d] fp32
  float4* s_rec;  // per stored slot [rows][nT][W]: {h, du, dz, token (int bits)}
  // dx pass: which of dz Wg^T (bit 0) and du Wu^T (bit 1) it sums, and
  // whether it adds them to dx instead of storing them
  int dx_mats;
  int dx_accumulate;
  // dx pass: when set (a zeroed int), every warp of the grid takes its next
  // token from this one counter instead of from its block's share
  int* next_row_global;
  int* dev_status;
};

// Warps per block of the per-token dx pass, which holds dx_t and two weight
// rows in registers.
constexpr int bwd_dx_warps(int nch) { return nch <= 4 ? 16 : (nch <= 7 ? 12 : 8); }

constexpr size_t bwd_dx_smem_bytes(int nch) { return static_cast<size_t>(bwd_dx_warps(nch)) * kListCap * 6; }

// acc += c_s * M[j_s, :] for the entries s < ns (c_s on lane s), with the same
// two-buffer gather.
template <int NCH>
__device__ __forceinline__ void bwd_axpy_pass(float (&acc)[NCH][8], const uint16_t* M, int my_j, float my_c, int ns,
                                              int lane, int d) {
  uint4 wa[NCH], wb[NCH];
  load_row<NCH>(wa, M + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, 0)) * d, lane, d);
#pragma unroll 1
  for (int s = 0; s < ns; s += 2) {
    if (s + 1 < ns) load_row<NCH>(wb, M + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 1)) * d, lane, d);
    const float c0 = __shfl_sync(0xffffffffu, my_c, s);
#pragma unroll
    for (int i = 0; i < NCH; ++i) axpy8(acc[i], c0, wa[i]);
    if (s + 1 < ns) {
      if (s + 2 < ns)
        load_row<NCH>(wa, M + static_cast<size_t>(__shfl_sync(0xffffffffu, my_j, s + 2)) * d, lane, d);
      const float c1 = __shfl_sync(0xffffffffu, my_c, s + 1);
#pragma unroll
      for (int i = 0; i < NCH; ++i) axpy8(acc[i], c1, wb[i]);
    }
  }
}

// Flattens the stored slots of row t, tiles [c0, c1), into list (column |
// bf16 g << 16) and lpos (the slot's position in the row's [nT][W] block, bit
// 15 set for an out-of-range column, which is then read as column 0 and must
// contribute nothing). Returns the number of entries; 8 slots per 16-byte load.
__device__ __forceinline__ int bwd_build_list(const BwdParams& p, int t, int c0, int c1, uint32_t* list,
                                              uint16_t* lpos, int lane, bool& bad_index) {
  int total = 0;
#pragma unroll 1
  for (int cb = c0; cb < c1; cb += 32) {
    const int c = cb + lane;
    int n = 0;
    if (c < c1) n = min(max(static_cast<int>(p.counts[static_cast<size_t>(t) * p.nT + c]), 0), p.W);
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
      // slots past n are read but not used (k + 8 <= W)
      const uint4 iv = ldg_nc_v4(p.idx + base + k);
      const uint4 vv = ldg_nc_v4(p.vals + base + k);
      const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
      const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (k + e < n) {
          const uint32_t jj = (e & 1) ? (iw[e >> 1] >> 16) : (iw[e >> 1] & 0xffffu);
          const uint32_t gg = (e & 1) ? (vw[e >> 1] & 0xffff0000u) : (vw[e >> 1] << 16);
          uint32_t ent = jj | gg;
          uint16_t pos = static_cast<uint16_t>(c * p.W + k + e);  // < 2^15: nT * W <= 255 * 128
          if (static_cast<int>(static_cast<int16_t>(jj)) < 0 || static_cast<int>(jj) >= p.f) {
            bad_index = true;
            ent = 0;
            pos |= 0x8000u;
          }
          list[off + k + e] = ent;
          lpos[off + k + e] = pos;
        }
      }
    }
  }
  return total;
}

// Tokens are handed out one at a time from a per-block counter over the
// block's contiguous share of the rows, or from one counter for the grid.
__device__ __forceinline__ int bwd_next_row(int* next_row, int lane) {
  int t = 0;
  if (lane == 0) t = atomicAdd(next_row, 1);
  return __shfl_sync(0xffffffffu, t, 0);
}

// The dx pass, one warp per token that fits: dx_t = sum over its stored slots of
// dz_j Wg[:, j] + du_j Wu[:, j], with du_j, dz_j from the slots' records and
// dx_t in registers (two alternating weight-row buffers, as in the forward).
template <int NCH, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) bwd_dx_kernel(const BwdParams p) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ uint4 bwd_smem[];
  __shared__ int next_row;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int d = p.d;
  uint32_t* list = reinterpret_cast<uint32_t*>(bwd_smem) + warp * kListCap;
  uint16_t* lpos = reinterpret_cast<uint16_t*>(reinterpret_cast<uint32_t*>(bwd_smem) + WARPS * kListCap) +
                   warp * kListCap;
  const int group_tiles = max(1, kListCap / p.W);
  bool bad_index = false;
  const int r_end = p.next_row_global != nullptr
                        ? p.rows
                        : static_cast<int>(static_cast<long long>(p.rows) * (blockIdx.x + 1) / gridDim.x);
  if (threadIdx.x == 0) next_row = static_cast<int>(static_cast<long long>(p.rows) * blockIdx.x / gridDim.x);
  __syncthreads();
#pragma unroll 1
  for (;;) {
    const int t = bwd_next_row(p.next_row_global != nullptr ? p.next_row_global : &next_row, lane);
    if (t >= r_end) break;
    if (p.row_ovf[t]) continue;
    float acc[NCH][8];
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;
    const size_t slot_row = static_cast<size_t>(t) * p.nT * p.W;
#pragma unroll 1
    for (int c0 = 0; c0 < p.nT; c0 += group_tiles) {
      __syncwarp();
      const int total = bwd_build_list(p, t, c0, min(p.nT, c0 + group_tiles), list, lpos, lane, bad_index);
      __syncwarp();
#pragma unroll 1
      for (int s0 = 0; s0 < total; s0 += 32) {
        const int ns = min(32, total - s0);
        const int my_j = lane < ns ? entry_j(list[s0 + lane]) : 0;
        const uint16_t my_pos = lane < ns ? lpos[s0 + lane] : 0x8000u;
        float my_du = 0.0f, my_dz = 0.0f;
        if ((my_pos & 0x8000u) == 0) {
          const float4 rec = p.s_rec[slot_row + my_pos];
          my_du = rec.y;
          my_dz = rec.z;
        }
        if (p.dx_mats & 1) bwd_axpy_pass<NCH>(acc, p.WgT, my_j, my_dz, ns, lane, d);
        if (p.dx_mats & 2) bwd_axpy_pass<NCH>(acc, p.WuT, my_j, my_du, ns, lane, d);
      }
    }
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int k0 = (i * 32 + lane) * 8;
      if (k0 < d) {
        float4* dst = reinterpret_cast<float4*>(p.dx + static_cast<size_t>(t) * d + k0);
        if (p.dx_accumulate) {
          const float4 a = dst[0], b = dst[1];
          acc[i][0] += a.x; acc[i][1] += a.y; acc[i][2] += a.z; acc[i][3] += a.w;
          acc[i][4] += b.x; acc[i][5] += b.y; acc[i][6] += b.z; acc[i][7] += b.w;
        }
        dst[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        dst[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
      }
    }
  }
  if (__any_sync(0xffffffffu, bad_index) && lane == 0) raise_status(p.dev_status, kDevIndex);
}

// ---------------------------------------------------------------- by column

// The stored slots of one pass, as the column sort sees them.
// The records of the rows that fit from dense u = x . Wu^T and dh = dy . Wd^T
// ([rows][f] fp32 each, from two tensor-core GEMMs) instead of a dot product
// over a gathered Wu row per stored slot: each stored slot (j, g) gets
// {h = g u_j, du = dh_j g, dz = dh_j u_j, t}. Eight lanes per (row, tile), four
// consecutive tiles per warp, the lanes of a tile taking its slots side by side
// (a thread per tile walking its slots one after another took 0.12 ms at the
// 0.5B layer). A stored index outside its own column tile raises
// TWELL_ERR_INDEX and gets a zero record, so that it adds nothing downstream.
__global__ void __launch_bounds__(256) bwd_records_kernel(const BwdParams p, const float* __restrict__ u) {
  griddep_launch_dependents();
  griddep_wait();
  bool bad = false;
  const int lane = threadIdx.x & 31;
  const long long pairs = static_cast<long long>(p.rows) * p.nT;
  const long long groups = (pairs + 3) / 4;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long g = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < groups;
       g += nw) {
    const long long i = g * 4 + (lane >> 3);
    if (i >= pairs) continue;
    const int t = static_cast<int>(i / p.nT);
    if (p.row_ovf[t]) continue;
    const int n = min(max(static_cast<int>(p.counts[i]), 0), p.W);
    const size_t base = static_cast<size_t>(i) * p.W;
    const float* urow = u + static_cast<size_t>(t) * p.f;
    const float* dhrow = p.dh + static_cast<size_t>(t) * p.f;
    const int c = static_cast<int>(i - static_cast<long long>(t) * p.nT);
    for (int k = lane & 7; k < n; k += 8) {
      const int j = p.idx[base + k];
      const float gv = __uint_as_float(static_cast<uint32_t>(p.vals[base + k]) << 16);
      if (j < c * 128 || j >= (c + 1) * 128 || j >= p.f) {
        bad = true;
        p.s_rec[base + k] = make_float4(0.f, 0.f, 0.f, __int_as_float(t));
        continue;
      }
      const float uj = __ldg(urow + j), dh = __ldg(dhrow + j);
      p.s_rec[base + k] = make_float4(gv * uj, dh * gv, dh * uj, __int_as_float(t));
    }
  }
  if (bad) raise_status(p.dev_status, kDevIndex);
}

struct SlotSource {
  const int16_t* counts;
  const int16_t* idx;
  const float4* rec;  // the slots' records (read by the scatter)
  const uint8_t* row_ovf;  // rows with the flag set are skipped when skip_ovf
  int rows;
  const int* rows_dev;
  int nT, W, f;
  int skip_ovf;
};

__device__ __forceinline__ int source_rows(const SlotSource& s) {
  return s.rows_dev != nullptr ? min(max(*s.rows_dev, 0), s.rows) : s.rows;
}

// SCATTER == false: colcnt[j] += number of slots with column j.
// SCATTER == true: each slot's record is copied to list[colptr[j] +
// cursor[j]++] (the order inside a column is that of the atomics). Eight
// lanes per (row, tile), four consecutive tiles per warp, the lanes of a tile
// taking its slots side by side (a warp per tile left most lanes idle at the
// configured densities).
template <bool SCATTER>
__global__ void bwd_columns_kernel(SlotSource src, int* colcnt, const int* colptr, float4* list) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int rows = source_rows(src);
  const long long pairs = static_cast<long long>(rows) * src.nT;
  const long long groups = (pairs + 3) / 4;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long g = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < groups;
       g += nw) {
    const long long w = g * 4 + (lane >> 3);
    if (w >= pairs) continue;
    const int t = static_cast<int>(w / src.nT);
    if (src.skip_ovf && src.row_ovf[t]) continue;
    const int n = min(max(static_cast<int>(src.counts[w]), 0), src.W);
    for (int k = lane & 7; k < n; k += 8) {
      const size_t slot = static_cast<size_t>(w) * src.W + k;
      const int j = src.idx[slot];
      if (j < 0 || j >= src.f) continue;
      if (SCATTER) {
        const int pos = colptr[j] + atomicAdd(colcnt + j, 1);
        list[pos] = src.rec[slot];
      } else {
        atomicAdd(colcnt + j, 1);
      }
    }
  }
}

// colptr[j] = sum of colcnt[0..j) for j <= f, and colcnt is reset to zero (it
// then serves as the scatter cursor). One block of 1024 threads.
__global__ void __launch_bounds__(1024) bwd_column_scan_kernel(int* colcnt, int f, int* colptr) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < f; base += 1024) {
    const int j = base + tid;
    const int v = j < f ? colcnt[j] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int w = warp_sums[lane];
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      warp_sums[lane] = wi - w;
    }
    __syncthreads();
    const int excl = carry + warp_sums[wid] + incl - v;
    if (j < f) {
      colptr[j] = excl;
      colcnt[j] = 0;
    }
    __syncthreads();
    if (tid == 1023) carry = excl + v;
    __syncthreads();
  }
  if (tid == 0) colptr[f] = carry;
}

struct WgradParams {
  const float4* list;  // slot records {h, du, dz, token} sorted by column
  const int* colptr;
  const uint16_t* x0;
  const uint16_t* dy0;
  int f, d;
  float* dWgT;  // [f][d] fp32, fully written
  float* dWuT;
  float* dWd;
};

// One warp per (hidden unit j, 256-wide slice of d): lane l owns 8 consecutive
// elements of the slice; the unit's slots are read 32 at a time (lane e
// fetches entry e's scalars and row), then broadcast one by one. The warps run
// slice by slice (every unit of slice 0 first), so the x and dy columns being
// gathered at any time are one or two slices of them (T x 512 bytes each),
// which stay in L2; unit by unit, every warp in flight touched all of x and
// dy.
__global__ void __launch_bounds__(256) bwd_wgrad_kernel(const WgradParams p) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int slices = (p.d + 255) / 256;
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(p.f) * slices) return;
  const int sl = static_cast<int>(w / p.f);
  const int j = static_cast<int>(w - static_cast<long long>(sl) * p.f);
  const int k0 = sl * 256 + lane * 8;
  const bool mine = k0 < p.d;
  float ag[8], au[8], ad[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) ag[e] = au[e] = ad[e] = 0.0f;
  const int e0 = p.colptr[j], e1 = p.colptr[j + 1];
  // a batch of 32 records staged in shared memory, read back by broadcast
  __shared__ float4 srec_all[8][32];
  float4* srec = srec_all[threadIdx.x >> 5];
#pragma unroll 1
  for (int b = e0; b < e1; b += 32) {
    const int nb = min(32, e1 - b);
    __syncwarp();
    if (lane < nb) srec[lane] = p.list[b + lane];
    __syncwarp();
#pragma unroll 2
    for (int s = 0; s < nb; ++s) {
      const float4 rec = srec[s];
      if (mine) {
        const size_t off = static_cast<size_t>(__float_as_int(rec.w)) * p.d + k0;
        const uint4 xv = ldg_nc_v4(p.x0 + off);
        const uint4 dv = ldg_nc_v4(p.dy0 + off);
        axpy8(ad, rec.x, dv);
        axpy8(au, rec.y, xv);
        axpy8(ag, rec.z, xv);
      }
    }
  }
  if (mine) {
    const size_t o = static_cast<size_t>(j) * p.d + k0;
    float4* g4 = reinterpret_cast<float4*>(p.dWgT + o);
    float4* u4 = reinterpret_cast<float4*>(p.dWuT + o);
    float4* d4 = reinterpret_cast<float4*>(p.dWd + o);
    g4[0] = make_float4(ag[0], ag[1], ag[2], ag[3]);
    g4[1] = make_float4(ag[4], ag[5], ag[6], ag[7]);
    u4[0] = make_float4(au[0], au[1], au[2], au[3]);
    u4[1] = make_float4(au[4], au[5], au[6], au[7]);
    d4[0] = make_float4(ad[0], ad[1], ad[2], ad[3]);
    d4[1] = make_float4(ad[4], ad[5], ad[6], ad[7]);
  }
}

// Tensor-core forms: the records of the rows that fit, written as token-major
// rows a2[t][4f] = [dz | du | dz_lo | du_lo] (bf16 value, then the bf16
// remainder v - bf16(v); zeros where no slot is stored, and for the rows that
// overflow), the layout of the overflow rows' dense branch, so that one GEMM
// against [Wg; Wu] (read twice along K) gives dx for every token. WITH_H: rows
// a2[t][6f] that also hold [h | h_lo], from which the weight-gradient GEMMs
// read dz, du and h with the tokens as K (an MN-major A operand). One warp per
// (row, tile): its lanes load the tile's slots side by side and drop their
// values into the tile's 128 units in shared memory, then lane l writes units
// 4l..4l+3, so every byte of the block is written once with 8-byte stores that
// a warp makes contiguous (a memset of the block and 2-byte scattered stores
// into it took 0.27 ms at the 0.5B layer; a slot-by-slot walk by every lane,
// 0.22 ms).
template <bool WITH_H>
__global__ void __launch_bounds__(256) bwd_dense_rows_kernel(SlotSource src, uint16_t* __restrict__ a2) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int kVals = WITH_H ? 3 : 2;
  __shared__ __align__(16) float tile_vals[8][3][128];  // per warp: dz, du, h of the tile's units
  const int lane = threadIdx.x & 31;
  float (*tv)[128] = tile_vals[threadIdx.x >> 5];
  const long long pairs = static_cast<long long>(src.rows) * src.nT;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const size_t f = static_cast<size_t>(src.f);
  for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < pairs;
       w += nw) {
    const int t = static_cast<int>(w / src.nT);
    const int c = static_cast<int>(w - static_cast<long long>(t) * src.nT);
#pragma unroll
    for (int b = 0; b < kVals; ++b) *reinterpret_cast<float4*>(&tv[b][4 * lane]) = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();
    if (!src.row_ovf[t]) {
      const int n = min(max(static_cast<int>(src.counts[w]), 0), src.W);
      for (int k = lane; k < n; k += 32) {
        const size_t slot = static_cast<size_t>(w) * src.W + k;
        const int j = static_cast<int>(src.idx[slot]) - c * 128;
        if (j >= 0 && j < 128) {
          const float4 rec = src.rec[slot];
          tv[0][j] = rec.z;
          tv[1][j] = rec.y;
          if (WITH_H) tv[2][j] = rec.x;
        }
      }
    }
    __syncwarp();
    float v[3][4];
#pragma unroll
    for (int b = 0; b < kVals; ++b) {
      const float4 q = *reinterpret_cast<const float4*>(&tv[b][4 * lane]);
      v[b][0] = q.x;
      v[b][1] = q.y;
      v[b][2] = q.z;
      v[b][3] = q.w;
    }
    __syncwarp();  // the next pair's zeros overwrite these units
    uint16_t* row = a2 + static_cast<size_t>(t) * (WITH_H ? 6 : 4) * f + static_cast<size_t>(c) * 128 + 4 * lane;
#pragma unroll
    for (int b = 0; b < kVals; ++b) {
      const uint32_t h01 = pack_bf16x2(v[b][0], v[b][1]), h23 = pack_bf16x2(v[b][2], v[b][3]);
      const uint32_t l01 = pack_bf16x2(v[b][0] - __uint_as_float(h01 << 16), v[b][1] - __uint_as_float(h01 & 0xffff0000u));
      const uint32_t l23 = pack_bf16x2(v[b][2] - __uint_as_float(h23 << 16), v[b][3] - __uint_as_float(h23 & 0xffff0000u));
      // value and remainder columns: dz 0 and 2f, du f and 3f, h 4f and 5f
      const size_t hi_col = b < 2 ? b * f : 4 * f, lo_col = b < 2 ? (2 + b) * f : 5 * f;
      *reinterpret_cast<uint2*>(row + hi_col) = make_uint2(h01, h23);
      *reinterpret_cast<uint2*>(row + lo_col) = make_uint2(l01, l23);
    }
  }
}

}  // namespace twell
