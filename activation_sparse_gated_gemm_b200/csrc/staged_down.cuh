// Down projection from a TwELL of hidden activations, staged through shared
// memory:
//     y[t, :] = sum over the stored slots (j, h) of row t of  h * Wd[j, :]
// (intellectnews.ru "Sakana AI и NVIDIA: TwELL ...", section "Слитые CUDA-ядра
// для инференса и гибрид для обучения": the sparse step reads only the stored
// units; here the hidden values h were already formed by the tensor-core
// epilogue, so only the down projection is left).
//
// The per-token kernel of sparse_ffn.cuh gathers a whole row of Wd from L2 for
// every stored slot; at large batches that runs at the L2 gather rate, and the
// same rows are fetched again for every token that activates the unit. Here a
// block owns a group of G tokens and a 128-column slice of d and walks Wd in
// chunks of 256 rows (two column tiles). TMA copies each chunk's slice into
// shared memory once for the whole group, and every stored slot of the group's
// tokens then reads its 256-byte piece of the row from shared memory. The
// accumulators of the group's tokens stay in registers for the whole walk: a
// warp owns G/15 tokens, a lane four columns of each.
//
// Two small kernels prepare the walk once per token group (all slices of the
// group share it): staged_order_kernel deals the group's tokens to the warps
// in a snake order of their stored-slot totals, so every warp gets about the
// same work; staged_lists_kernel writes, per group and chunk, each warp's
// stored slots as one flat run of 32-bit entries (row within the chunk, bf16 h
// in the high half), token after token, with the offset of every token's run.
#pragma once

#include "ptx.cuh"
#include "sparse_ffn.cuh"

namespace twell {

// 15 consumer warps and the producer make 16 warps, four per SM sub-partition,
// so each thread may hold 128 registers (64 of them accumulators).
constexpr int kStgWarps = 15;                        // consumer warps per block
constexpr int kStgThreads = (kStgWarps + 1) * 32;    // plus one TMA producer warp
constexpr int kStgCols = 128;                        // d columns per unit; a lane owns 4
constexpr int kStgRows = 256;                        // Wd rows per chunk
constexpr int kStgTiles = kStgRows / 128;            // column tiles per chunk
constexpr int kStgStages = 3;                        // chunks in flight per block
constexpr int kStgStageBytes = kStgRows * kStgCols * 2;
constexpr int kStgMaxTpw = 16;                       // tokens per warp, at most
constexpr int kStgMaxG = kStgWarps * kStgMaxTpw;     // tokens per group, at most
constexpr int kStgSmemBytes = kStgStages * kStgStageBytes + 1024 + 1024;  // + barriers, alignment

struct StagedParams {
  const int16_t* counts;
  const int16_t* idx;
  const uint16_t* vals;
  const uint8_t* row_ovf;
  float* y;
  int* pos_tok;     // [ngroups][G]: token at each warp position (warp w owns w*tpw .. w*tpw+tpw-1), or -1
  int* offs;        // [ngroups][nC][G+1]: start of each position's run in the (group, chunk) list
  uint32_t* list;   // entries; group g, chunk k at g*G*nT*W + Gg*(k*kStgTiles)*W
  int T, d, f, nT, W;
  int G, tpw, ngroups, nC, nsl;
  int skip_ovf;
  int* dev_status;
};

__device__ __forceinline__ size_t staged_list_base(const StagedParams& p, int g, int k) {
  const int t0 = g * p.G;
  const int Gg = min(p.G, p.T - t0);
  return static_cast<size_t>(t0) * p.nT * p.W + static_cast<size_t>(Gg) * (k * kStgTiles) * p.W;
}

// One block of 256 threads per token group: each token's number of stored
// slots (0 for a skipped overflow row, -1 past the batch), a rank by that
// number (descending, ties by position), and the snake deal over the consumer
// warps: rank r goes to round r / 15 of warp r % 15, or of warp 14 - r % 15 in
// odd rounds.
__global__ void __launch_bounds__(256) staged_order_kernel(const StagedParams p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int key[kStgMaxG];
  const int g = blockIdx.x;
  const int t0 = g * p.G;
  const int Gg = min(p.G, p.T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool overflow = false;
  for (int i = warp; i < p.G; i += 8) {
    int sum = -1;
    if (i < Gg) {
      const int t = t0 + i;
      if (p.skip_ovf && p.row_ovf[t]) {
        sum = 0;
      } else {
        int s = 0;
        for (int c = lane; c < p.nT; c += 32) {
          const int cnt = p.counts[static_cast<size_t>(t) * p.nT + c];
          if (cnt > p.W) overflow = true;
          s += min(max(cnt, 0), p.W);
        }
        sum = __reduce_add_sync(0xffffffffu, s);
      }
    }
    if (lane == 0) key[i] = sum;
  }
  __syncthreads();
  const int i = threadIdx.x;
  if (i < p.G) {
    const int ki = key[i];
    int r = 0;
    for (int j = 0; j < p.G; ++j) {
      const int kj = key[j];
      r += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
    }
    const int round = r / kStgWarps, m = r - round * kStgWarps;
    const int w = (round & 1) ? kStgWarps - 1 - m : m;
    const bool live = i < Gg && !(p.skip_ovf && p.row_ovf[t0 + i]);
    p.pos_tok[static_cast<size_t>(g) * p.G + w * p.tpw + round] = live ? t0 + i : -1;
  }
  if (__any_sync(0xffffffffu, overflow) && lane == 0 && !p.skip_ovf) raise_status(p.dev_status, kDevOverflow);
}

// One block of 256 threads per (chunk, token group); thread i is warp position
// i. It counts its token's slots in the chunk's tiles, takes its offset from a
// block-wide prefix sum, and writes its entries. A stored index outside its
// own column tile (or outside [0, f)) raises TWELL_ERR_INDEX and is written as
// an entry that adds nothing.
__global__ void __launch_bounds__(256) staged_lists_kernel(const StagedParams p) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int warp_sum[8];
  const int k = blockIdx.x, g = blockIdx.y;
  const int c0 = k * kStgTiles;
  const int c1 = min(p.nT, c0 + kStgTiles);
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  int t = -1;
  int n[kStgTiles];
#pragma unroll
  for (int c = 0; c < kStgTiles; ++c) n[c] = 0;
  if (i < p.G) {
    t = p.pos_tok[static_cast<size_t>(g) * p.G + i];
    if (t >= 0) {
#pragma unroll
      for (int c = 0; c < kStgTiles; ++c)
        if (c0 + c < c1) n[c] = min(max(static_cast<int>(p.counts[static_cast<size_t>(t) * p.nT + c0 + c]), 0), p.W);
    }
  }
  int tot = 0;
#pragma unroll
  for (int c = 0; c < kStgTiles; ++c) tot += n[c];
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_sum[w];
  const int off = before + incl - tot;
  int* ob = p.offs + (static_cast<size_t>(g) * p.nC + k) * (p.G + 1);
  if (i < p.G) ob[i] = off;
  if (i == p.G - 1) ob[p.G] = off + tot;
  uint32_t* out = p.list + staged_list_base(p, g, k) + off;
  bool bad = false;
  int o = 0;
#pragma unroll
  for (int c = 0; c < kStgTiles; ++c) {
    const int nc = n[c];
    const size_t base = (static_cast<size_t>(t) * p.nT + c0 + c) * p.W;
    for (int s0 = 0; s0 < nc; s0 += 8) {
      // 8 slots per 16-byte load; s0 + 8 <= W since W is a multiple of 8
      const uint4 iv = ldg_nc_v4(p.idx + base + s0);
      const uint4 vv = ldg_nc_v4(p.vals + base + s0);
      const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
      const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (s0 + e < nc) {
          const uint32_t jj = (e & 1) ? (iw[e >> 1] >> 16) : (iw[e >> 1] & 0xffffu);
          const uint32_t hh = (e & 1) ? (vw[e >> 1] & 0xffff0000u) : (vw[e >> 1] << 16);
          const int r = static_cast<int>(static_cast<int16_t>(jj)) - c0 * 128;  // row within the chunk
          uint32_t ent = static_cast<uint32_t>(r) | hh;
          if (r < c * 128 || r >= (c + 1) * 128) {
            bad = true;
            ent = 0;  // row 0 with h = 0: adds nothing
          }
          out[o++] = ent;
        }
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(p.dev_status, kDevIndex);
}

// y[0..4) += h * w[0..4): h the high half of an entry, w four bf16 of a row.
__device__ __forceinline__ void axpy4_bf16(float (&y)[4], uint32_t ent, uint32_t w01, uint32_t w23) {
  asm("{\n\t.reg .b16 h, hl, w0, w1, w2, w3;\n\t"
      "mov.b32 {hl, h}, %4;\n\t"
      "mov.b32 {w0, w1}, %5; mov.b32 {w2, w3}, %6;\n\t"
      "fma.rn.f32.bf16 %0, h, w0, %0; fma.rn.f32.bf16 %1, h, w1, %1;\n\t"
      "fma.rn.f32.bf16 %2, h, w2, %2; fma.rn.f32.bf16 %3, h, w3, %3;\n\t}"
      : "+f"(y[0]), "+f"(y[1]), "+f"(y[2]), "+f"(y[3])
      : "r"(ent), "r"(w01), "r"(w23));
}

// The consumer warps' walk (warps 0-14 of staged_down_kernel).
__device__ __forceinline__ void staged_consume(const StagedParams& p, uint8_t* smem, uint64_t* full, uint64_t* empty,
                                               volatile int* abort_flag, int n_chunks, int warp, int lane) {
  const int tpw = p.tpw;
  float acc[kStgMaxTpw][4];
#pragma unroll
  for (int q = 0; q < kStgMaxTpw; ++q)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[q][c] = 0.0f;

  // chunk m of the stream: unit u = blockIdx.x + (m / nC) * grid, chunk k = m % nC
  auto offs_of = [&](int m) -> int {
    if (m >= n_chunks) return 0;
    const int u = static_cast<int>(blockIdx.x) + (m / p.nC) * static_cast<int>(gridDim.x);
    const int k = m - (m / p.nC) * p.nC;
    const int g = u / p.nsl;
    const int* ob = p.offs + (static_cast<size_t>(g) * p.nC + k) * (p.G + 1) + warp * tpw;
    return lane <= tpw ? __ldg(ob + lane) : 0;
  };
  auto list_of = [&](int m) -> const uint32_t* {
    const int u = static_cast<int>(blockIdx.x) + (m / p.nC) * static_cast<int>(gridDim.x);
    const int k = m - (m / p.nC) * p.nC;
    return p.list + staged_list_base(p, u / p.nsl, k);
  };
  // first 32 entries of this warp's run in chunk m, lane l holding entry l
  auto first_of = [&](int m, int o) -> uint32_t {
    const int beg = __shfl_sync(0xffffffffu, o, 0);
    const int end = __shfl_sync(0xffffffffu, o, tpw);
    if (m >= n_chunks) return 0u;
    return beg + lane < end ? __ldg(list_of(m) + beg + lane) : 0u;
  };

  bool ok = true;
  int my_tok = -1;
  int o_cur = offs_of(0);
  int o_n1 = offs_of(1);
  uint32_t e_cur = first_of(0, o_cur);
#pragma unroll 1
  for (int m = 0; m < n_chunks; ++m) {
    const int s = m % kStgStages;
    const uint32_t ph = static_cast<uint32_t>(m / kStgStages) & 1u;
    const int u = static_cast<int>(blockIdx.x) + (m / p.nC) * static_cast<int>(gridDim.x);
    const int k = m - (m / p.nC) * p.nC;
    const int g = u / p.nsl;
    const int sl = u - g * p.nsl;
    if (k == 0) my_tok = lane < tpw ? __ldg(p.pos_tok + static_cast<size_t>(g) * p.G + warp * tpw + lane) : -1;
    // next chunks' offsets and first entries, loaded while this chunk is consumed
    const int o_n2 = offs_of(m + 2);
    const uint32_t e_n1 = first_of(m + 1, o_n1);
    if (!mbar_wait(&full[s], ph, abort_flag)) {
      ok = false;
      break;
    }
    const uint8_t* buf = smem + s * kStgStageBytes + lane * 8;
    const uint32_t* lst = list_of(m);
    int pos = __shfl_sync(0xffffffffu, o_cur, 0);
    const int wend = __shfl_sync(0xffffffffu, o_cur, tpw);
    int bbase = pos;
    uint32_t ecur = e_cur;
    uint32_t enext = bbase + 32 + lane < wend ? __ldg(lst + bbase + 32 + lane) : 0u;
#pragma unroll
    for (int q = 0; q < kStgMaxTpw; ++q) {
      if (q < tpw) {
        const int end = __shfl_sync(0xffffffffu, o_cur, q + 1);
#pragma unroll 1
        while (pos < end) {
          if (pos - bbase == 32) {
            bbase += 32;
            ecur = enext;
            enext = bbase + 32 + lane < wend ? __ldg(lst + bbase + 32 + lane) : 0u;
          }
          const int i0 = pos - bbase;
          const int take = min(end - pos, 32 - i0);
          // Four slots at a time: their broadcasts, then their shared-memory
          // reads, then the math, so the reads' latencies overlap. The low 8
          // bits of an entry address a row of the 256-row stage: always
          // inside it.
          int i = 0;
#pragma unroll 1
          for (; i + 4 <= take; i += 4) {
            uint32_t e[4];
            uint2 w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) e[j] = __shfl_sync(0xffffffffu, ecur, i0 + i + j);
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const uint2*>(buf + ((e[j] & 0xffu) << 8));
#pragma unroll
            for (int j = 0; j < 4; ++j) axpy4_bf16(acc[q], e[j], w[j].x, w[j].y);
          }
#pragma unroll 1
          for (; i < take; ++i) {
            const uint32_t e = __shfl_sync(0xffffffffu, ecur, i0 + i);
            const uint2 w = *reinterpret_cast<const uint2*>(buf + ((e & 0xffu) << 8));
            axpy4_bf16(acc[q], e, w.x, w.y);
          }
          pos += take;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (k == p.nC - 1) {
      const int col = sl * kStgCols + lane * 4;
#pragma unroll
      for (int q = 0; q < kStgMaxTpw; ++q) {
        if (q < tpw) {
          const int t = __shfl_sync(0xffffffffu, my_tok, q);
          if (t >= 0 && col < p.d)
            *reinterpret_cast<float4*>(p.y + static_cast<size_t>(t) * p.d + col) =
                make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[q][c] = 0.0f;
      }
    }
    o_cur = o_n1;
    o_n1 = o_n2;
    e_cur = e_n1;
  }
  if (!ok) {
    *abort_flag = 1;
    if (lane == 0) raise_status(p.dev_status, kDevTimeout);
  }
}

// Persistent: block b takes the units b, b + grid, ... (unit = token group x
// column slice) and walks their chunks as one stream through kStgStages
// shared-memory stages. Warp 15 issues the TMA copies; warps 0-14 consume.
__global__ void __launch_bounds__(kStgThreads, 1)
    staged_down_kernel(const __grid_constant__ CUtensorMap wd_map, const StagedParams p) {
  griddep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStgStages * kStgStageBytes);
  uint64_t* empty = full + kStgStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStgStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStgWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kStgWarps && lane == 0) tma_prefetch_desc(&wd_map);
  __syncthreads();
  griddep_wait();

  const int units = p.ngroups * p.nsl;
  const int my_units = units > static_cast<int>(blockIdx.x)
                           ? (units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                 static_cast<int>(gridDim.x)
                           : 0;
  const int n_chunks = my_units * p.nC;

  // the producer's record of its copies, for the drain on the abort path
  uint32_t issued = 0, issued_par = 0;
  if (warp == kStgWarps) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      bool ok = true;
      for (int m = 0; m < n_chunks; ++m) {
        const int s = m % kStgStages;
        const uint32_t ph = static_cast<uint32_t>(m / kStgStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int u = static_cast<int>(blockIdx.x) + (m / p.nC) * static_cast<int>(gridDim.x);
        const int k = m - (m / p.nC) * p.nC;
        const int sl = u % p.nsl;
        mbar_arrive_expect_tx(&full[s], kStgStageBytes);
        tma_load_2d(smem + s * kStgStageBytes, &wd_map, &full[s], sl * kStgCols, k * kStgRows);
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(p.dev_status, kDevTimeout);
      }
    }
  } else {
    staged_consume(p, smem, full, empty, abort_flag, n_chunks, warp, lane);
  }
  // Every thread gets here (all waits are bounded). After an abort, let the
  // copies still in flight land before the block's shared memory goes away.
  __syncthreads();
  if (*abort_flag && issued != 0) {
    for (int s = 0; s < kStgStages; ++s)
      if (issued & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, kDrainTimeoutNs);
  }
}

}  // namespace twell
