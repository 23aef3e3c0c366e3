// C ABI of the TwELL sparse gated FFN (declared in include/twell.h): argument
// checks, TMA tensor maps and kernel launches. Host code only; the kernels
// live in umma_gemm.cuh and sparse_ffn.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "twell.h"
#include "backward.cuh"
#include "gemv.cuh"
#include "sparse_ffn.cuh"
#include "umma_gemm.cuh"

namespace {

using namespace twell;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ device

struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 ok, 2 unsupported
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

twell_status current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TWELL_ERR_CUDA;
  DeviceInfo& info = g_dev[dev];
  int st = info.state.load(std::memory_order_acquire);
  if (st == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return TWELL_ERR_CUDA;
    info.num_sms = sms;
    st = (major == 10 && minor == 0) ? 1 : 2;
    info.state.store(st, std::memory_order_release);
  }
  if (st != 1) return TWELL_ERR_DEVICE;
  *dev_out = dev;
  *sms_out = info.num_sms;
  return TWELL_OK;
}

// ------------------------------------------------------------------ TMA maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major bf16 matrix [outer][inner] with 128-byte swizzled boxes of
// box_inner x box_outer elements.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ checks

twell_status check_shape(int T, int d, int f) {
  if (T < 0) return TWELL_ERR_SHAPE;
  if (d < 64 || d > 4096 || d % 64 != 0) return TWELL_ERR_SHAPE;
  if (f < 128 || f > 32767 || f % 128 != 0) return TWELL_ERR_SHAPE;
  return TWELL_OK;
}

twell_status check_tw(const twell_t* tw, int T, int f) {
  if (tw == nullptr) return TWELL_ERR_NULL;
  if (tw->T != T || tw->f != f || tw->tile != 128) return TWELL_ERR_SHAPE;
  if (tw->W < 8 || tw->W > 128 || tw->W % 8 != 0) return TWELL_ERR_SHAPE;
  if (T > 0) {
    if (!tw->counts || !tw->idx || !tw->vals || !tw->row_ovf) return TWELL_ERR_NULL;
    if (!aligned16(tw->counts) || !aligned16(tw->idx) || !aligned16(tw->vals) || !aligned16(tw->row_ovf))
      return TWELL_ERR_ALIGN;
  }
  return TWELL_OK;
}

twell_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr) return TWELL_ERR_NULL;
  for (const void* p : ps)
    if (!aligned16(p)) return TWELL_ERR_ALIGN;
  return TWELL_OK;
}

#define TW_TRY(expr)                    \
  do {                                  \
    twell_status _s = (expr);           \
    if (_s != TWELL_OK) return _s;      \
  } while (0)

twell_status cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return TWELL_OK;
  (void)cudaGetLastError();
  return TWELL_ERR_CUDA;
}

// ------------------------------------------------------------------ launches

// Every kernel is launched as a programmatic dependent of the previous work in
// the stream: its blocks may start (and run their private setup) while that
// work finishes; each kernel waits for it before touching shared data.
template <typename... KArgs, typename... Args>
twell_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_ok(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
}

// The same, with the grid cut into clusters of `cluster` consecutive blocks.
template <typename... KArgs, typename... Args>
twell_status launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, int cluster, cudaStream_t s,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_ok(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
}

// Zero up to three device byte ranges with one dependent launch.
twell_status zero_async(cudaStream_t s, int sms, void* p0, size_t n0, void* p1 = nullptr, size_t n1 = 0,
                        void* p2 = nullptr, size_t n2 = 0) {
  ZeroRanges r{{p0, p1, p2}, {n0, n1, n2}};
  const size_t most = std::max(n0, std::max(n1, n2)) / 16 + 1;
  const int blocks = static_cast<int>(std::min<size_t>((most + 255) / 256, 2 * static_cast<size_t>(sms)));
  return launch(zero_ranges_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, s, r);
}

template <int MODE>
twell_status launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                         int grid, cudaStream_t s) {
  auto kern = umma_gemm_kernel<MODE>;
  TW_TRY(cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes)));
  TW_TRY(launch(kern, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, s, a, b0, b1, p));
  return cuda_ok(cudaGetLastError());
}

int gemm_grid(int M, int N, int tile_n, int sms) {
  const long long tiles = static_cast<long long>((M + kBM - 1) / kBM) * ((N + tile_n - 1) / tile_n);
  return static_cast<int>(tiles < sms ? (tiles > 0 ? tiles : 1) : sms);
}

// With slot_of_row set, the GEMM also writes the exact ReLU(z) of every
// overflowing (row, tile) into ovf_h at the row's compact slot (see GemmParams),
// and the int after *ovf_n (the sparse step's work counter) is zeroed with it;
// work_next alone: that counter is zeroed beside the overflow flags.
twell_status gate_pack_impl(const uint16_t* x, const uint16_t* WgT, int T, int d, int f, const twell_t* tw,
                            int32_t* dev_status, cudaStream_t s, int sms, const int* M_dev = nullptr,
                            int* slot_of_row = nullptr, int* slot_row = nullptr, int* ovf_n = nullptr,
                            uint16_t* ovf_h = nullptr, int* work_next = nullptr) {
  if (work_next != nullptr && slot_of_row == nullptr) {
    TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T), work_next, 4));
  } else if (slot_of_row != nullptr) {
    TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T), slot_of_row, static_cast<size_t>(T) * 4, ovf_n, 8));
  } else {
    TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T)));
  }
  CUtensorMap ma, mb;
  if (!make_map(&ma, x, d, T, kBK, kBM) || !make_map(&mb, WgT, d, f, kBK, kBN)) return TWELL_ERR_CUDA;
  GemmParams p{};
  p.M = T;
  p.M_dev = M_dev;
  p.N = f;
  p.K = d;
  p.counts = tw->counts;
  p.idx = tw->idx;
  p.vals = tw->vals;
  p.row_ovf = tw->row_ovf;
  p.nT = f / 128;
  p.W = tw->W;
  p.slot_of_row = slot_of_row;
  p.slot_row = slot_row;
  p.ovf_n = ovf_n;
  p.ovf_h = ovf_h;
  p.dev_status = dev_status;
  return launch_gemm<kModeTwell>(ma, mb, mb, p, M_dev ? sms : gemm_grid(T, f, kBN, sms), s);
}

// Gate and up GEMM in one pass; TwELL of the gate pattern holding h = z * u.
// With slot_of_row set, the GEMM also writes the exact h of every overflowing
// (row, tile) into ovf_h at the row's compact slot (see GemmParams), and the
// int after *ovf_n (the sparse step's work counter) is zeroed with it.
twell_status gate_up_pack_impl(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, int T, int d, int f,
                               const twell_t* tw, int32_t* dev_status, cudaStream_t s, int sms,
                               int* slot_of_row = nullptr, int* slot_row = nullptr, int* ovf_n = nullptr,
                               uint16_t* ovf_h = nullptr) {
  if (slot_of_row != nullptr) {
    TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T), slot_of_row, static_cast<size_t>(T) * 4, ovf_n, 8));
  } else {
    TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T)));
  }
  CUtensorMap ma, mg, mu;
  if (!make_map(&ma, x, d, T, kBK, kBM) || !make_map(&mg, WgT, d, f, kBK, 128) || !make_map(&mu, WuT, d, f, kBK, 128))
    return TWELL_ERR_CUDA;
  GemmParams p{};
  p.M = T;
  p.N = f;
  p.K = d;
  p.counts = tw->counts;
  p.idx = tw->idx;
  p.vals = tw->vals;
  p.row_ovf = tw->row_ovf;
  p.nT = f / 128;
  p.W = tw->W;
  p.slot_of_row = slot_of_row;
  p.slot_row = slot_row;
  p.ovf_n = ovf_n;
  p.ovf_h = ovf_h;
  p.dev_status = dev_status;
  return launch_gemm<kModeTwellHidden>(ma, mg, mu, p, gemm_grid(T, f, 128, sms), s);
}

// Whether the sparse step spreads tokens over several warps (with partial
// sums added into a zeroed y): when the batch has fewer tokens than twice the
// resident warps.
bool sparse_splits_units(int T, int d, bool down_only, int sms) {
  const int nch = (d + 255) / 256;
  return static_cast<long long>(T) * 2 < static_cast<long long>(sparse_warps_for(nch, down_only)) * sms;
}

template <int NCH, bool DOWN_ONLY>
twell_status launch_sparse_n(SparseParams p, int sms, cudaStream_t s, bool y_zeroed) {
  constexpr int kWarps = sparse_warps_for(NCH, DOWN_ONLY);
  // With fewer tokens than resident warps, a token's column tiles are spread
  // over several warps whose partial sums are added into a zeroed y (rows that
  // the sparse step skips are rewritten by the dense branch afterwards).
  const long long warps_resident = static_cast<long long>(kWarps) * sms;
  p.unit_tiles = p.nT;
  if (static_cast<long long>(p.T) * 2 < warps_resident) {
    const long long want_units = warps_resident;  // about one unit per resident warp
    const long long per_token = std::max(1LL, std::min<long long>(p.nT, want_units / std::max(1, p.T)));
    p.unit_tiles = static_cast<int>((p.nT + per_token - 1) / per_token);
    if (p.unit_tiles < p.nT && !y_zeroed) {
      TW_TRY(launch(zero_rows_kernel, dim3(std::min(p.T, 4 * sms)), dim3(256), 0, s, p.y, p.T, p.d, p.row_ovf, p.skip_ovf));
      TW_TRY(cuda_ok(cudaGetLastError()));
    }
  }
  const long long units = static_cast<long long>(p.T) * ((p.nT + p.unit_tiles - 1) / p.unit_tiles);
  const int blocks = static_cast<int>(std::min<long long>((units + kWarps - 1) / kWarps, sms));
  const size_t smem = static_cast<size_t>(kWarps) * (NCH * 32 * sizeof(uint4) + kListCap * sizeof(uint32_t));
  auto kern = sparse_ffn_warp_kernel<NCH, kWarps, DOWN_ONLY>;
  // always opt in: the static shared memory adds to the dynamic size
  TW_TRY(cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))));
  TW_TRY(launch(kern, dim3(blocks), dim3(kWarps * 32), smem, s, p));
  return cuda_ok(cudaGetLastError());
}

template <bool DOWN_ONLY>
twell_status sparse_launch(const SparseParams& p, int d, int sms, cudaStream_t s, bool y_zeroed) {
  // (the launcher decides how a token's column tiles are split over warps)
  switch ((d + 255) / 256) {
    case 1: return launch_sparse_n<1, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 2: return launch_sparse_n<2, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 3: return launch_sparse_n<3, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 4: return launch_sparse_n<4, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 5: return launch_sparse_n<5, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 6: return launch_sparse_n<6, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 7: return launch_sparse_n<7, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 8: return launch_sparse_n<8, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 9: return launch_sparse_n<9, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 10: return launch_sparse_n<10, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 11: return launch_sparse_n<11, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 12: return launch_sparse_n<12, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 13: return launch_sparse_n<13, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 14: return launch_sparse_n<14, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 15: return launch_sparse_n<15, DOWN_ONLY>(p, sms, s, y_zeroed);
    case 16: return launch_sparse_n<16, DOWN_ONLY>(p, sms, s, y_zeroed);
    default: return TWELL_ERR_SHAPE;
  }
}

twell_status sparse_impl(const uint16_t* x, const uint16_t* WuT, const uint16_t* Wd, int T, int d, int f,
                         const twell_t* tw, int skip, float* y, int32_t* dev_status, cudaStream_t s, int sms,
                         bool down_only = false, bool y_zeroed = false, int* work_next = nullptr) {
  SparseParams p{};
  p.work_next = work_next;
  p.x = x;
  p.WuT = WuT;
  p.Wd = Wd;
  p.counts = tw->counts;
  p.idx = tw->idx;
  p.vals = tw->vals;
  p.row_ovf = tw->row_ovf;
  p.y = y;
  p.T = T;
  p.d = d;
  p.f = f;
  p.nT = f / 128;
  p.W = tw->W;
  p.skip_ovf = skip ? 1 : 0;
  p.dev_status = dev_status;
  return down_only ? sparse_launch<true>(p, d, sms, s, y_zeroed) : sparse_launch<false>(p, d, sms, s, y_zeroed);
}

// The sparse step of a batch of at most 8 tokens with d a multiple of 256: one
// warp per stored slot (sparse_small_kernel), enough blocks per token for one
// slot per warp when every tile is full, and about two blocks per SM at most.
// The rows of y it writes must hold zeros; overflow rows are skipped.
template <int NCH>
twell_status sparse_small_n(const SparseParams& p, bool down_only, int sms, cudaStream_t s) {
  const long long most = (static_cast<long long>(p.nT) * p.W + kSmallSparseWarps - 1) / kSmallSparseWarps;
  const long long spread = (2LL * sms + p.T - 1) / p.T;
  const dim3 grid(static_cast<unsigned>(std::max(1LL, std::min(most, spread))), static_cast<unsigned>(p.T));
  if (down_only) return launch(sparse_small_kernel<NCH, true>, grid, dim3(kSmallSparseWarps * 32), 0, s, p);
  return launch(sparse_small_kernel<NCH, false>, grid, dim3(kSmallSparseWarps * 32), 0, s, p);
}

twell_status sparse_small_impl(const uint16_t* x, const uint16_t* WuT, const uint16_t* Wd, int T, int d, int f,
                               const twell_t* tw, float* y, int32_t* ovf_rows, int32_t* n_ovf, int32_t* dev_status,
                               cudaStream_t s, int sms, bool down_only) {
  SparseParams p{};
  p.x = x;
  p.WuT = WuT;
  p.Wd = Wd;
  p.counts = tw->counts;
  p.idx = tw->idx;
  p.vals = tw->vals;
  p.row_ovf = tw->row_ovf;
  p.y = y;
  p.T = T;
  p.d = d;
  p.f = f;
  p.nT = f / 128;
  p.W = tw->W;
  p.skip_ovf = 1;
  p.route_flags = tw->row_ovf;
  p.route_rows = ovf_rows;
  p.route_n = n_ovf;
  p.dev_status = dev_status;
  switch (d / 256) {
    case 1: return sparse_small_n<1>(p, down_only, sms, s);
    case 2: return sparse_small_n<2>(p, down_only, sms, s);
    case 3: return sparse_small_n<3>(p, down_only, sms, s);
    case 4: return sparse_small_n<4>(p, down_only, sms, s);
    case 5: return sparse_small_n<5>(p, down_only, sms, s);
    case 6: return sparse_small_n<6>(p, down_only, sms, s);
    case 7: return sparse_small_n<7>(p, down_only, sms, s);
    case 8: return sparse_small_n<8>(p, down_only, sms, s);
    case 9: return sparse_small_n<9>(p, down_only, sms, s);
    case 10: return sparse_small_n<10>(p, down_only, sms, s);
    case 11: return sparse_small_n<11>(p, down_only, sms, s);
    case 12: return sparse_small_n<12>(p, down_only, sms, s);
    case 13: return sparse_small_n<13>(p, down_only, sms, s);
    case 14: return sparse_small_n<14>(p, down_only, sms, s);
    case 15: return sparse_small_n<15>(p, down_only, sms, s);
    default: return sparse_small_n<16>(p, down_only, sms, s);
  }
}

// Down projection from a TwELL of hidden activations (per-token gathers of Wd rows).
twell_status down_impl(const uint16_t* Wd, int T, int d, int f, const twell_t* tw, int skip, float* y,
                       int32_t* dev_status, cudaStream_t s, int sms, int* work_next = nullptr) {
  return sparse_impl(nullptr, nullptr, Wd, T, d, f, tw, skip, y, dev_status, s, sms, true, false, work_next);
}

twell_status dense_down_impl(const uint16_t* h_buf, int M, const int* M_dev, const uint16_t* Wd, int d, int f,
                             bool split, const int* row_map, float* y, int y_rows, int32_t* dev_status,
                             cudaStream_t s, int sms);

// ------------------------------------------------------------------ down projection over tile unions

// Workspace of the union down projection, carved from the hybrid workspace:
// the tiles' hidden-value blocks (H, [num_m * 128][f] bf16), then the tiles'
// union lists ([num_m][f] int32) and K block counts ([num_m] int32).
size_t union_bytes(int T, int f) {
  const size_t num_m = (static_cast<size_t>(T) + kBM - 1) / kBM;
  return round_up(num_m * kBM * f * 2, 256) + round_up(num_m * f * 4, 256) + round_up(num_m * 4, 256);
}

// y (rows that fit) = per 128-row tile, the tile's hidden values over its
// union of stored units times those rows of Wd, on the tensor cores.
twell_status union_down_impl(const uint16_t* Wd, int T, int d, int f, const twell_t* tw, int skip, float* y,
                             void* ws, int32_t* dev_status, cudaStream_t s, int sms) {
  const int num_m = (T + kBM - 1) / kBM;
  char* w = static_cast<char*>(ws);
  UnionParams u{};
  u.counts = tw->counts;
  u.idx = tw->idx;
  u.vals = tw->vals;
  u.row_ovf = tw->row_ovf;
  u.T = T;
  u.f = f;
  u.nT = f / 128;
  u.W = tw->W;
  u.skip_ovf = skip ? 1 : 0;
  u.H = reinterpret_cast<uint16_t*>(w);
  u.union_rows = reinterpret_cast<int*>(w + round_up(static_cast<size_t>(num_m) * kBM * f * 2, 256));
  u.kb_tile = u.union_rows + round_up(static_cast<size_t>(num_m) * f * 4, 256) / 4;
  u.stride = f;
  u.dev_status = dev_status;
  TW_TRY(launch(union_prep_kernel, dim3(num_m), dim3(256), 0, s, u));
  // A: the H blocks in 128 x 64 boxes; B: Wd rows one at a time (gather4 takes four)
  CUtensorMap ma, mb;
  if (!make_map(&ma, u.H, f, static_cast<uint64_t>(num_m) * kBM, kBK, kBM) || !make_map(&mb, Wd, d, f, 64, 1))
    return TWELL_ERR_CUDA;
  GemmParams p{};
  p.M = T;
  p.N = d;
  p.K = f;
  p.out_f32 = y;
  p.ldo = d;
  p.out_rows = T;
  p.k_splits_max = 1;
  p.kb_tile = u.kb_tile;
  p.union_rows = u.union_rows;
  p.union_stride = f;
  p.dev_status = dev_status;
  return launch_gemm<kModeUnion>(ma, mb, mb, p, gemm_grid(T, d, kBN, sms), s);
}

// Dense FFN over A rows (x itself, or gathered overflow rows): h = ReLU(A Wg) * (A Wu), or
// h = ReLU(A Wg) for the non-gated layer (WuT null), into h_buf, then
// out[row_map[i]] = h[i] Wd (row_map null: identity). With split, h_buf is [M][2f] holding
// bf16(h) and the bf16 remainder, and the down GEMM runs K = 2f.
twell_status dense_impl(const uint16_t* a_rows, int M, const int* M_dev, const uint16_t* WgT, const uint16_t* WuT,
                        const uint16_t* Wd, int d, int f, uint16_t* h_buf, bool split, const int* row_map,
                        float* y, int y_rows, int32_t* dev_status, cudaStream_t s, int sms) {
  const int hk = split ? 2 * f : f;
  const bool gated = WuT != nullptr;
  const int tile_n = gated ? 128 : kBN;  // h columns per output tile of the first GEMM
  CUtensorMap ma, mg, mu;
  if (!make_map(&ma, a_rows, d, M, kBK, kBM) || !make_map(&mg, WgT, d, f, kBK, tile_n) ||
      (gated && !make_map(&mu, WuT, d, f, kBK, 128)))
    return TWELL_ERR_CUDA;
  GemmParams p1{};
  p1.M = M;
  p1.M_dev = M_dev;
  p1.N = f;
  p1.K = d;
  p1.out = h_buf;
  p1.ldo = hk;
  p1.h_split = split ? 1 : 0;
  p1.dev_status = dev_status;
  const int g1 = M_dev ? sms : gemm_grid(M, f, tile_n, sms);
  if (gated) {
    TW_TRY(launch_gemm<kModeGateUp>(ma, mg, mu, p1, g1, s));
  } else {
    TW_TRY(launch_gemm<kModeRelu>(ma, mg, mg, p1, g1, s));
  }
  return dense_down_impl(h_buf, M, M_dev, Wd, d, f, split, row_map, y, y_rows, dev_status, s, sms);
}

// Second half of the dense layer: out[row_map[i]] = h[i] Wd (row_map null: identity), h_buf
// [M][f] bf16, or [M][2f] (h and its bf16 remainder) with split.
twell_status dense_down_impl(const uint16_t* h_buf, int M, const int* M_dev, const uint16_t* Wd, int d, int f,
                             bool split, const int* row_map, float* y, int y_rows, int32_t* dev_status,
                             cudaStream_t s, int sms) {
  const int hk = split ? 2 * f : f;
  CUtensorMap mh, md;
  if (!make_map(&mh, h_buf, hk, M, kBK, kBM) || !make_map(&md, Wd, d, f, 64, kBK)) return TWELL_ERR_CUDA;
  GemmParams p2{};
  p2.M = M;
  p2.M_dev = M_dev;
  p2.N = d;
  p2.K = hk;
  p2.k_wrap = split ? f : 0;
  p2.out_f32 = y;
  p2.ldo = d;
  p2.row_map = row_map;
  p2.out_rows = y_rows;
  // The routed rows of y were zeroed by the gather. The full-batch dense
  // baseline splits K only when its output tiles cannot fill the GPU, after
  // zeroing y.
  p2.k_splits_max = 1;
  if (row_map != nullptr) {
    p2.k_splits_max = 32;
    p2.split_waves = 1;  // the gather zeroed every routed row
  } else if (static_cast<long long>((M + kBM - 1) / kBM) * ((d + kBN - 1) / kBN) * 2 <= sms) {
    TW_TRY(zero_async(s, sms, y, static_cast<size_t>(M) * d * sizeof(float)));
    p2.k_splits_max = 32;
  }
  p2.dev_status = dev_status;
  // a split K needs the whole grid: the kernel derives the splits from it
  const int g2 = (M_dev != nullptr || p2.k_splits_max > 1) ? sms : gemm_grid(M, d, kBN, sms);
  return launch_gemm<kModeDown>(mh, md, md, p2, g2, s);
}


// ------------------------------------------------------------------ small batches

// ------------------------------------------------------------------ batches of <= 8 tokens

// The GEMV path: at most 8 tokens and d a multiple of 256.
bool gemv_batch(int T, int d) { return T <= kGemvMaxT && d % 256 == 0; }

// Tokens the kernels are compiled for: the batch rounded up to 1, 2, 4 or 8
// (the branch modes read their row count on the device and take 8).
int gemv_nt(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8; }

template <int MODE, int NT>
twell_status gemv_first_nt(const GemvParams& p, cudaStream_t s) {
  auto kern = gemv_first_kernel<MODE, NT>;
  const size_t smem = static_cast<size_t>(NT) * p.d * 2;
  TW_TRY(cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))));
  if (gv_pack(MODE))
    return launch_cluster(kern, dim3(p.nT * kGemvCluster), dim3(kGemvThreads), smem, kGemvCluster, s, p);
  return launch(kern, dim3(p.f / kGemvCols), dim3(kGemvThreads), smem, s, p);
}

template <int MODE>
twell_status gemv_first(const GemvParams& p, cudaStream_t s) {
  switch (gv_branch(MODE) ? kGemvMaxT : gemv_nt(p.T)) {
    case 1: return gemv_first_nt<MODE, 1>(p, s);
    case 2: return gemv_first_nt<MODE, 2>(p, s);
    case 4: return gemv_first_nt<MODE, 4>(p, s);
    default: return gemv_first_nt<MODE, kGemvMaxT>(p, s);
  }
}

// The down GEMV's grid: one block per 256 columns of d times row groups, about
// two blocks per SM in all (one wave), each group a multiple of 8 rows.
twell_status gemv_down(GemvDownParams p, int nt, cudaStream_t s, int sms) {
  const int slices = (p.d + kGemvDownCols - 1) / kGemvDownCols;
  const int groups = std::max(1, (2 * sms + slices - 1) / slices);
  int rpb = (p.f + groups - 1) / groups;
  rpb = std::min(kGemvDownMaxRows, std::max(kGemvWarps, (rpb + kGemvWarps - 1) / kGemvWarps * kGemvWarps));
  p.rows_per_block = rpb;
  const dim3 grid(static_cast<unsigned>((p.f + rpb - 1) / rpb), static_cast<unsigned>(slices));
  switch (nt) {
    case 1: return launch(gemv_down_kernel<1>, grid, dim3(kGemvThreads), 0, s, p);
    case 2: return launch(gemv_down_kernel<2>, grid, dim3(kGemvThreads), 0, s, p);
    case 4: return launch(gemv_down_kernel<4>, grid, dim3(kGemvThreads), 0, s, p);
    default: return launch(gemv_down_kernel<kGemvMaxT>, grid, dim3(kGemvThreads), 0, s, p);
  }
}

GemvParams gemv_params(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, int T, int d, int f,
                       int32_t* dev_status) {
  GemvParams p{};
  p.x = x;
  p.WgT = WgT;
  p.WuT = WuT;
  p.T = T;
  p.d = d;
  p.f = f;
  p.nT = f / 128;
  p.dev_status = dev_status;
  return p;
}

// Hybrid forward of a batch of <= 8 tokens: the pack from the GEMV (which also
// zeroes y), the sparse step with one warp per stored slot (down only when the
// pack holds hidden values), which also routes the batch from the counts, and
// the dense branch as
// GEMVs over the listed rows with fp32 hidden activations (h_buf: [T][f] fp32).
// mode: 0 gated (gate pack, fused up+down), 1 gated with hidden values, 2 non-gated.
twell_status gemv_hybrid(int mode, const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, const uint16_t* Wd,
                         int T, int d, int f, const twell_t* tw, float* y, int32_t* ovf_rows, int32_t* n_ovf,
                         float* h_buf, int32_t* dev_status, cudaStream_t s, int sms) {
  GemvParams p = gemv_params(x, WgT, mode == 1 ? WuT : nullptr, T, d, f, dev_status);
  p.W = tw->W;
  p.counts = tw->counts;
  p.idx = tw->idx;
  p.vals = tw->vals;
  p.y_zero = y;
  if (mode == 1) {
    TW_TRY(gemv_first<kGvPackHidden>(p, s));
  } else {
    TW_TRY(gemv_first<kGvPackGate>(p, s));
  }
  TW_TRY(sparse_small_impl(x, WuT, Wd, T, d, f, tw, y, ovf_rows, n_ovf, dev_status, s, sms, mode != 0));
  // the dense branch over the listed rows, hidden activations in fp32
  GemvParams b = gemv_params(x, WgT, mode == 2 ? nullptr : WuT, T, d, f, dev_status);
  b.rows = ovf_rows;
  b.n_rows = n_ovf;
  b.h_f32 = h_buf;
  if (mode == 2) {
    TW_TRY(gemv_first<kGvBranchRelu>(b, s));
  } else {
    TW_TRY(gemv_first<kGvBranchH>(b, s));
  }
  GemvDownParams q{};
  q.h_f32 = h_buf;
  q.Wd = Wd;
  q.y = y;
  q.rows = ovf_rows;
  q.n_rows = n_ovf;
  q.T = T;
  q.d = d;
  q.f = f;
  TW_TRY(gemv_down(q, kGemvMaxT, s, sms));
  return cuda_ok(cudaGetLastError());
}

// Dense layer of a batch of <= 8 tokens: h (bf16, in h_buf [T][f]) from the
// GEMV, which also zeroes y, then y += h Wd. gated: ReLU(x Wg) (x Wu), else ReLU(x W1).
twell_status gemv_dense(bool gated, const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, const uint16_t* Wd,
                        int T, int d, int f, float* y, uint16_t* h_buf, int32_t* dev_status, cudaStream_t s,
                        int sms) {
  GemvParams p = gemv_params(x, WgT, gated ? WuT : nullptr, T, d, f, dev_status);
  p.h_bf16 = h_buf;
  p.y_zero = y;
  if (gated) {
    TW_TRY(gemv_first<kGvDenseH>(p, s));
  } else {
    TW_TRY(gemv_first<kGvDenseRelu>(p, s));
  }
  GemvDownParams q{};
  q.h_bf16 = h_buf;
  q.Wd = Wd;
  q.y = y;
  q.T = T;
  q.d = d;
  q.f = f;
  TW_TRY(gemv_down(q, gemv_nt(T), s, sms));
  return cuda_ok(cudaGetLastError());
}

// Batches up to this many tokens whose gate GEMM has too few output tiles to
// fill the GPU take the small-batch path: the gate GEMM splits K over the whole
// grid into fp32 pre-activations, and a separate kernel packs them.
constexpr int kSmallT = 512;

bool small_batch(int T, int N, int tile_n, int sms) {
  const long long tiles = static_cast<long long>((T + kBM - 1) / kBM) * ((N + tile_n - 1) / tile_n);
  return T <= kSmallT && tiles * 2 <= sms;
}

// C[M][ldo] += A[M][K] B[N][K]^T in fp32 with K split over the whole grid; C's
// first N columns of rows < M must hold zeros.
twell_status f32_gemm_impl(const uint16_t* A, int M, const uint16_t* B, int N, int K, float* C, int ldo,
                           int32_t* dev_status, cudaStream_t s, int sms) {
  // a batch of fewer than 128 rows loads only its rows of A
  const int a_rows = std::min(kBM, (M + 7) / 8 * 8);
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, K, M, kBK, a_rows) || !make_map(&mb, B, K, N, kBK, kBN)) return TWELL_ERR_CUDA;
  GemmParams p{};
  p.a_box_rows = a_rows;
  p.M = M;
  p.N = N;
  p.K = K;
  p.out_f32 = C;
  p.ldo = ldo;
  p.out_rows = M;
  p.k_splits_max = 32;
  p.dev_status = dev_status;
  return launch_gemm<kModeF32>(ma, mb, mb, p, sms, s);
}

// The gate pack of a small batch: split-K gate GEMM into zbuf ([T][f] fp32,
// caller's scratch), then one warp per (row, tile) packs it; y is zeroed on
// the way when y_zero is given.
twell_status small_gate_pack_impl(const uint16_t* x, const uint16_t* WgT, int T, int d, int f, const twell_t* tw,
                                  float* zbuf, float* y_zero, int32_t* dev_status, cudaStream_t s, int sms) {
  TW_TRY(zero_async(s, sms, tw->row_ovf, static_cast<size_t>(T), zbuf, static_cast<size_t>(T) * f * sizeof(float)));
  TW_TRY(f32_gemm_impl(x, T, WgT, f, d, zbuf, f, dev_status, s, sms));
  const long long warps = static_cast<long long>(T) * (f / 128);
  const int blocks = static_cast<int>(std::min<long long>((warps + 7) / 8, 4LL * sms));
  TW_TRY(launch(pack_f32_kernel, dim3(blocks), dim3(256), 0, s, zbuf, T, f, tw->W, tw->counts, tw->idx, tw->vals, tw->row_ovf, y_zero, d));
  return cuda_ok(cudaGetLastError());
}

// Dense branch: gather x[rows[i]] into xo, dense FFN (gated, or non-gated when WuT is
// null) into ho, scatter to y.
twell_status dense_rows_impl(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, const uint16_t* Wd,
                             int T, int d, int f, const int32_t* rows, const int32_t* n_rows, float* y,
                             uint16_t* xo, uint16_t* ho, int32_t* dev_status, cudaStream_t s, int sms) {
  TW_TRY(launch(gather_rows_kernel, dim3(sms * 2), dim3(256), 0, s, x, d, rows, n_rows, T, xo, y, dev_status, 0));
  TW_TRY(cuda_ok(cudaGetLastError()));
  return dense_impl(xo, T, n_rows, WgT, WuT, Wd, d, f, ho, true, rows, y, T, dev_status, s, sms);
}

#include "backward_host.cuh"

}  // namespace

// ====================================================================== C ABI

extern "C" {

twell_status twell_gate_pack(const uint16_t* x, const uint16_t* WgT, int T, int d, int f, const twell_t* tw,
                             int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return gate_pack_impl(x, WgT, T, d, f, tw, dev_status, static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_sparse_ffn(const uint16_t* x, const uint16_t* WuT, const uint16_t* Wd, int T, int d, int f,
                              const twell_t* tw, int skip_overflow_rows, float* y, int32_t* dev_status,
                              void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WuT, Wd, y, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return sparse_impl(x, WuT, Wd, T, d, f, tw, skip_overflow_rows, y, dev_status, static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_ffn_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, const uint16_t* Wd,
                               int T, int d, int f, const twell_t* tw, float* y, int32_t* dev_status,
                               void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, y, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TW_TRY(gate_pack_impl(x, WgT, T, d, f, tw, dev_status, s, sms));
  return sparse_impl(x, WuT, Wd, T, d, f, tw, 0, y, dev_status, s, sms);
}

twell_status twell_gate_up_pack(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, int T, int d, int f,
                                const twell_t* tw, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return gate_up_pack_impl(x, WgT, WuT, T, d, f, tw, dev_status, static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_sparse_down(const uint16_t* Wd, int T, int d, int f, const twell_t* tw, int skip_overflow_rows,
                               float* y, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({Wd, y, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return down_impl(Wd, T, d, f, tw, skip_overflow_rows, y, dev_status, static_cast<cudaStream_t>(stream), sms);
}

size_t twell_sparse_down_union_workspace_bytes(int T, int d, int f) {
  (void)d;
  if (T <= 0 || f < 128) return 0;
  return union_bytes(T, f);
}

twell_status twell_sparse_down_union(const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                                     int skip_overflow_rows, float* y, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({Wd, y, dev_status}));
  if (workspace == nullptr || workspace_bytes < union_bytes(T, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return union_down_impl(Wd, T, d, f, tw, skip_overflow_rows, y, workspace, dev_status,
                         static_cast<cudaStream_t>(stream), sms);
}

// The union form measured slower than the per-token kernel at every
// configured layer (0.5B, 1.5B and 2B), so the hybrid forwards never take it.
int twell_hybrid_down_is_union(int T, int d, int f, size_t workspace_bytes) {
  (void)T;
  (void)d;
  (void)f;
  (void)workspace_bytes;
  return 0;
}

namespace {

// The dense branch over the compact slots that the pack GEMM claimed for the
// routed rows (their overflowing tiles' exact h already in ho): the other
// tiles' h from the pack (a bf16 value and a zero remainder), the rows of y
// zeroed, then y[slot_row[s]] = [h | h_lo][s] [Wd; Wd].
twell_status slot_branch_impl(const twell_t* tw, const uint16_t* Wd, int T, int d, int f, const int* slot_row,
                              const int* n_slots, uint16_t* ho, float* y, int32_t* dev_status, cudaStream_t s,
                              int sms) {
  const long long pairs = static_cast<long long>(T) * (f / 128);
  TW_TRY(launch(ovf_fill_kernel, dim3(static_cast<unsigned>(std::max(1LL, std::min<long long>((pairs + 7) / 8, 4LL * sms)))),
                dim3(256), 0, s, static_cast<const int16_t*>(tw->counts), static_cast<const int16_t*>(tw->idx),
                static_cast<const uint16_t*>(tw->vals), f / 128, tw->W, f, slot_row, n_slots, ho, y, d));
  TW_TRY(cuda_ok(cudaGetLastError()));
  return dense_down_impl(ho, T, n_slots, Wd, d, f, true, slot_row, y, T, dev_status, s, sms);
}

}  // namespace

twell_status twell_ffn_hybrid_forward_tc_up(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                            const uint16_t* Wd, int T, int d, int f, const twell_t* tw, float* y,
                                            int32_t* ovf_rows, int32_t* n_ovf, void* workspace,
                                            size_t workspace_bytes, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, y, ovf_rows, n_ovf, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_hybrid_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* xo = static_cast<uint16_t*>(workspace);
  uint16_t* ho = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                             round_up(static_cast<size_t>(T) * d * 2, 256));
  if (gemv_batch(T, d)) return gemv_hybrid(1, x, WgT, WuT, Wd, T, d, f, tw, y, ovf_rows, n_ovf,
                                        reinterpret_cast<float*>(ho), dev_status, s, sms);
  // The dense branch takes its hidden activations from the gate+up GEMM (the
  // overflowing tiles, exact) and the pack (the others): no second gate and up
  // GEMM over the routed rows. The x-gather region holds the slot tables.
  int* slot_of_row = reinterpret_cast<int*>(xo);
  int* slot_row = slot_of_row + T;
  int* n_slots = slot_row + T;
  TW_TRY(gate_up_pack_impl(x, WgT, WuT, T, d, f, tw, dev_status, s, sms, slot_of_row, slot_row, n_slots, ho));
  TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, s, tw->row_ovf, T, ovf_rows, n_ovf, static_cast<const uint16_t*>(nullptr), 0, static_cast<uint16_t*>(nullptr), static_cast<float*>(nullptr)));
  TW_TRY(cuda_ok(cudaGetLastError()));
  TW_TRY(down_impl(Wd, T, d, f, tw, 1, y, dev_status, s, sms, n_slots + 1));
  return slot_branch_impl(tw, Wd, T, d, f, slot_row, n_slots, ho, y, dev_status, s, sms);
}

twell_status twell_route(const twell_t* tw, int32_t* ovf_rows, int32_t* n_ovf, void* stream) {
  if (tw == nullptr) return TWELL_ERR_NULL;
  TW_TRY(check_tw(tw, tw->T, tw->f));
  TW_TRY(check_ptrs({ovf_rows, n_ovf}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, static_cast<cudaStream_t>(stream), tw->row_ovf, tw->T, ovf_rows, n_ovf, static_cast<const uint16_t*>(nullptr), 0, static_cast<uint16_t*>(nullptr), static_cast<float*>(nullptr)));
  return cuda_ok(cudaGetLastError());
}

size_t twell_hybrid_workspace_bytes(int T, int d, int f) {
  if (T <= 0 || d <= 0 || f <= 0) return 0;
  return round_up(static_cast<size_t>(T) * d * 2, 256) + round_up(static_cast<size_t>(T) * f * 4, 256);
}

twell_status twell_ffn_hybrid_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, int T, int d, int f, const twell_t* tw, float* y,
                                      int32_t* ovf_rows, int32_t* n_ovf, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, y, ovf_rows, n_ovf, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_hybrid_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* xo = static_cast<uint16_t*>(workspace);
  uint16_t* ho = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                             round_up(static_cast<size_t>(T) * d * 2, 256));
  if (gemv_batch(T, d)) return gemv_hybrid(0, x, WgT, WuT, Wd, T, d, f, tw, y, ovf_rows, n_ovf,
                                        reinterpret_cast<float*>(ho), dev_status, s, sms);
  if (small_batch(T, f, kBN, sms)) {
    // the h region of the dense branch is free until that branch runs
    const bool zero_y = sparse_splits_units(T, d, false, sms);
    TW_TRY(small_gate_pack_impl(x, WgT, T, d, f, tw, reinterpret_cast<float*>(ho), zero_y ? y : nullptr,
                                dev_status, s, sms));
    TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, s, tw->row_ovf, T, ovf_rows, n_ovf, x, d, xo, y));
    TW_TRY(cuda_ok(cudaGetLastError()));
    TW_TRY(sparse_impl(x, WuT, Wd, T, d, f, tw, 1, y, dev_status, s, sms, false, zero_y));
    return dense_impl(xo, T, n_ovf, WgT, WuT, Wd, d, f, ho, true, ovf_rows, y, T, dev_status, s, sms);
  }
  // the sparse step's work counter in the h region of the dense branch (free until that branch runs)
  int* work_next = reinterpret_cast<int*>(ho);
  TW_TRY(gate_pack_impl(x, WgT, T, d, f, tw, dev_status, s, sms, nullptr, nullptr, nullptr, nullptr, nullptr,
                        work_next));
  TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, s, tw->row_ovf, T, ovf_rows, n_ovf, static_cast<const uint16_t*>(nullptr), 0, static_cast<uint16_t*>(nullptr), static_cast<float*>(nullptr)));
  TW_TRY(cuda_ok(cudaGetLastError()));
  TW_TRY(sparse_impl(x, WuT, Wd, T, d, f, tw, 1, y, dev_status, s, sms, false, false, work_next));
  return dense_rows_impl(x, WgT, WuT, Wd, T, d, f, ovf_rows, n_ovf, y, xo, ho, dev_status, s, sms);
}

twell_status twell_dense_rows_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, int T, int d, int f, const int32_t* rows,
                                      const int32_t* n_rows, float* y, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, rows, n_rows, y, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_hybrid_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  uint16_t* xo = static_cast<uint16_t*>(workspace);
  uint16_t* ho = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                             round_up(static_cast<size_t>(T) * d * 2, 256));
  return dense_rows_impl(x, WgT, WuT, Wd, T, d, f, rows, n_rows, y, xo, ho, dev_status,
                         static_cast<cudaStream_t>(stream), sms);
}

size_t twell_dense_workspace_bytes(int T, int d, int f) {
  (void)d;
  if (T <= 0 || f <= 0) return 0;
  // h [T][f] bf16, and for small batches the fp32 pre-activations [T][2f]
  const size_t small = T <= kSmallT ? round_up(static_cast<size_t>(T) * f * 8, 256) : 0;
  return round_up(static_cast<size_t>(T) * f * 2, 256) + small;
}

twell_status twell_dense_ffn_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                     const uint16_t* Wd, int T, int d, int f, float* y, void* workspace,
                                     size_t workspace_bytes, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, y, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_dense_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* h = static_cast<uint16_t*>(workspace);
  if (gemv_batch(T, d)) return gemv_dense(true, x, WgT, WuT, Wd, T, d, f, y, h, dev_status, s, sms);
  if (small_batch(T, f, 128, sms)) {
    // z and u with K split over the whole grid, then h = bf16(ReLU(z) * u)
    float* zu = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up(static_cast<size_t>(T) * f * 2, 256));
    TW_TRY(zero_async(s, sms, zu, static_cast<size_t>(T) * f * 8));
    TW_TRY(f32_gemm_impl(x, T, WgT, f, d, zu, 2 * f, dev_status, s, sms));
    TW_TRY(f32_gemm_impl(x, T, WuT, f, d, zu + f, 2 * f, dev_status, s, sms));
    const size_t n4 = static_cast<size_t>(T) * f / 4;
    TW_TRY(launch(h_from_zu_kernel, dim3(static_cast<unsigned>(std::min<size_t>((n4 + 255) / 256, 4 * static_cast<size_t>(sms)))), dim3(256), 0, s, zu, T, f, 1, h));
    TW_TRY(cuda_ok(cudaGetLastError()));
    return dense_down_impl(h, T, nullptr, Wd, d, f, false, nullptr, y, T, dev_status, s, sms);
  }
  return dense_impl(x, T, nullptr, WgT, WuT, Wd, d, f, h, false, nullptr, y, T, dev_status, s, sms);
}

twell_status twell_relu_ffn_hybrid_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2, int T, int d,
                                           int f, const twell_t* tw, float* y, int32_t* ovf_rows, int32_t* n_ovf,
                                           void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                           void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, W1T, W2, y, ovf_rows, n_ovf, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_hybrid_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* xo = static_cast<uint16_t*>(workspace);
  uint16_t* ho = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                             round_up(static_cast<size_t>(T) * d * 2, 256));
  // The pack of ReLU(x W1) holds the hidden activations themselves, so the
  // sparse step is the down projection alone.
  if (gemv_batch(T, d)) return gemv_hybrid(2, x, W1T, nullptr, W2, T, d, f, tw, y, ovf_rows, n_ovf,
                                        reinterpret_cast<float*>(ho), dev_status, s, sms);
  if (small_batch(T, f, kBN, sms)) {
    const bool zero_y = sparse_splits_units(T, d, true, sms);
    TW_TRY(small_gate_pack_impl(x, W1T, T, d, f, tw, reinterpret_cast<float*>(ho), zero_y ? y : nullptr,
                                dev_status, s, sms));
    TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, s, tw->row_ovf, T, ovf_rows, n_ovf, x, d, xo, y));
    TW_TRY(cuda_ok(cudaGetLastError()));
    TW_TRY(sparse_impl(nullptr, nullptr, W2, T, d, f, tw, 1, y, dev_status, s, sms, true, zero_y));
    return dense_impl(xo, T, n_ovf, W1T, nullptr, W2, d, f, ho, true, ovf_rows, y, T, dev_status, s, sms);
  }
  // As in the tensor-core-up form, the dense branch takes the routed rows' h
  // from the pack GEMM (the overflowing tiles, exact) and the pack (the
  // others) instead of a second GEMM over them; the x-gather region holds the
  // slot tables.
  int* slot_of_row = reinterpret_cast<int*>(xo);
  int* slot_row = slot_of_row + T;
  int* n_slots = slot_row + T;
  TW_TRY(gate_pack_impl(x, W1T, T, d, f, tw, dev_status, s, sms, nullptr, slot_of_row, slot_row, n_slots, ho));
  TW_TRY(launch(route_kernel, dim3(1), dim3(1024), 0, s, tw->row_ovf, T, ovf_rows, n_ovf, static_cast<const uint16_t*>(nullptr), 0, static_cast<uint16_t*>(nullptr), static_cast<float*>(nullptr)));
  TW_TRY(cuda_ok(cudaGetLastError()));
  TW_TRY(down_impl(W2, T, d, f, tw, 1, y, dev_status, s, sms, n_slots + 1));
  return slot_branch_impl(tw, W2, T, d, f, slot_row, n_slots, ho, y, dev_status, s, sms);
}

twell_status twell_relu_dense_rows_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2, int T, int d,
                                          int f, const int32_t* rows, const int32_t* n_rows, float* y,
                                          void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                          void* stream) {
  TW_TRY(check_shape(T, d, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, W1T, W2, rows, n_rows, y, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_hybrid_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  uint16_t* xo = static_cast<uint16_t*>(workspace);
  uint16_t* ho = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                             round_up(static_cast<size_t>(T) * d * 2, 256));
  return dense_rows_impl(x, W1T, nullptr, W2, T, d, f, rows, n_rows, y, xo, ho, dev_status,
                         static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_relu_dense_ffn_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2, int T, int d,
                                          int f, float* y, void* workspace, size_t workspace_bytes,
                                          int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, W1T, W2, y, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_dense_workspace_bytes(T, d, f)) return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* h = static_cast<uint16_t*>(workspace);
  if (gemv_batch(T, d)) return gemv_dense(false, x, W1T, nullptr, W2, T, d, f, y, h, dev_status, s, sms);
  if (small_batch(T, f, kBN, sms)) {
    float* z = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up(static_cast<size_t>(T) * f * 2, 256));
    TW_TRY(zero_async(s, sms, z, static_cast<size_t>(T) * f * 4));
    TW_TRY(f32_gemm_impl(x, T, W1T, f, d, z, f, dev_status, s, sms));
    const size_t n4 = static_cast<size_t>(T) * f / 4;
    TW_TRY(launch(h_from_zu_kernel, dim3(static_cast<unsigned>(std::min<size_t>((n4 + 255) / 256, 4 * static_cast<size_t>(sms)))), dim3(256), 0, s, z, T, f, 0, h));
    TW_TRY(cuda_ok(cudaGetLastError()));
    return dense_down_impl(h, T, nullptr, W2, d, f, false, nullptr, y, T, dev_status, s, sms);
  }
  return dense_impl(x, T, nullptr, W1T, nullptr, W2, d, f, h, false, nullptr, y, T, dev_status, s, sms);
}

size_t twell_backward_workspace_bytes(int T, int d, int f, int W) {
  if (T <= 0 || d <= 0 || f < 128 || W <= 0) return 0;
  return bwd_carve(nullptr, T, d, f, W).bytes;
}

twell_status twell_ffn_hybrid_backward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                       const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                       const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf, float* dx,
                                       float* dWgT, float* dWuT, float* dWd, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  // slot indices are kept in 31 bits
  if (static_cast<long long>(T) * (f / 128) * tw->W >= (1LL << 31)) return TWELL_ERR_SHAPE;
  TW_TRY(check_ptrs({dWgT, dWuT, dWd, dev_status}));
  if (T == 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = static_cast<size_t>(f) * d * sizeof(float);
    TW_TRY(cuda_ok(cudaMemsetAsync(dWgT, 0, n, s)));
    TW_TRY(cuda_ok(cudaMemsetAsync(dWuT, 0, n, s)));
    return cuda_ok(cudaMemsetAsync(dWd, 0, n, s));
  }
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, dy, ovf_rows, n_ovf, dx}));
  if (workspace == nullptr || workspace_bytes < twell_backward_workspace_bytes(T, d, f, tw->W))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  TW_TRY(backward_dx_impl(x, WgT, WuT, Wd, dy, T, d, f, tw, ovf_rows, n_ovf, dx, ws, dev_status, s, sms));
  return backward_dw_impl(x, dy, T, d, f, tw, n_ovf, dWgT, dWuT, dWd, ws, s, sms);
}

twell_status twell_ffn_hybrid_backward_dx(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                          const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                          const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf,
                                          float* dx, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                          void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (static_cast<long long>(T) * (f / 128) * tw->W >= (1LL << 31)) return TWELL_ERR_SHAPE;
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, dy, ovf_rows, n_ovf, dx, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_backward_workspace_bytes(T, d, f, tw->W))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return backward_dx_impl(x, WgT, WuT, Wd, dy, T, d, f, tw, ovf_rows, n_ovf, dx, static_cast<char*>(workspace),
                          dev_status, static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_ffn_hybrid_backward_dx_tc(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                             const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                             const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf,
                                             float* dx, void* workspace, size_t workspace_bytes,
                                             int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (static_cast<long long>(T) * (f / 128) * tw->W >= (1LL << 31)) return TWELL_ERR_SHAPE;
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, dy, ovf_rows, n_ovf, dx, dev_status}));
  if (workspace == nullptr || workspace_bytes < twell_backward_workspace_bytes(T, d, f, tw->W))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return backward_dx_impl(x, WgT, WuT, Wd, dy, T, d, f, tw, ovf_rows, n_ovf, dx, static_cast<char*>(workspace),
                          dev_status, static_cast<cudaStream_t>(stream), sms, true);
}

twell_status twell_ffn_hybrid_backward_dw(const uint16_t* x, const uint16_t* dy, int T, int d, int f,
                                          const twell_t* tw, const int32_t* n_ovf, float* dWgT, float* dWuT,
                                          float* dWd, void* workspace, size_t workspace_bytes, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (static_cast<long long>(T) * (f / 128) * tw->W >= (1LL << 31)) return TWELL_ERR_SHAPE;
  TW_TRY(check_ptrs({dWgT, dWuT, dWd}));
  if (T == 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = static_cast<size_t>(f) * d * sizeof(float);
    TW_TRY(cuda_ok(cudaMemsetAsync(dWgT, 0, n, s)));
    TW_TRY(cuda_ok(cudaMemsetAsync(dWuT, 0, n, s)));
    return cuda_ok(cudaMemsetAsync(dWd, 0, n, s));
  }
  TW_TRY(check_ptrs({x, dy, n_ovf}));
  if (workspace == nullptr || workspace_bytes < twell_backward_workspace_bytes(T, d, f, tw->W))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return backward_dw_impl(x, dy, T, d, f, tw, n_ovf, dWgT, dWuT, dWd, static_cast<char*>(workspace),
                          static_cast<cudaStream_t>(stream), sms);
}

twell_status twell_ffn_hybrid_backward_dw_tc(const uint16_t* x, const uint16_t* dy, int T, int d, int f,
                                             const twell_t* tw, const int32_t* n_ovf, float* dWgT, float* dWuT,
                                             float* dWd, void* workspace, size_t workspace_bytes, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (static_cast<long long>(T) * (f / 128) * tw->W >= (1LL << 31)) return TWELL_ERR_SHAPE;
  TW_TRY(check_ptrs({dWgT, dWuT, dWd}));
  if (T == 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = static_cast<size_t>(f) * d * sizeof(float);
    TW_TRY(cuda_ok(cudaMemsetAsync(dWgT, 0, n, s)));
    TW_TRY(cuda_ok(cudaMemsetAsync(dWuT, 0, n, s)));
    return cuda_ok(cudaMemsetAsync(dWd, 0, n, s));
  }
  TW_TRY(check_ptrs({x, dy, n_ovf}));
  if (workspace == nullptr || workspace_bytes < twell_backward_workspace_bytes(T, d, f, tw->W))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  return backward_dw_tc_impl(x, dy, T, d, f, tw, n_ovf, dWgT, dWuT, dWd, static_cast<char*>(workspace),
                             static_cast<cudaStream_t>(stream), sms);
}

size_t twell_dense_backward_workspace_bytes(int T, int d, int f) {
  (void)d;
  if (T <= 0 || f <= 0) return 0;
  const size_t tp = round_up(static_cast<size_t>(T), 64);
  return round_up(static_cast<size_t>(T) * f * 8, 256)   // [z | u] fp32
         + round_up(tp * f * 6, 256);                     // [dz | du | h] bf16, token-major
}

twell_status twell_dense_ffn_backward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, const uint16_t* dy, int T, int d, int f, float* dx,
                                      float* dWgT, float* dWuT, float* dWd, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_ptrs({dWgT, dWuT, dWd, dev_status}));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    const size_t n = static_cast<size_t>(f) * d * sizeof(float);
    TW_TRY(cuda_ok(cudaMemsetAsync(dWgT, 0, n, s)));
    TW_TRY(cuda_ok(cudaMemsetAsync(dWuT, 0, n, s)));
    return cuda_ok(cudaMemsetAsync(dWd, 0, n, s));
  }
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, dy, dx}));
  if (workspace == nullptr || workspace_bytes < twell_dense_backward_workspace_bytes(T, d, f))
    return TWELL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TWELL_ERR_ALIGN;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  char* ws = static_cast<char*>(workspace);
  const int tp = static_cast<int>(round_up(static_cast<size_t>(T), 64));
  float* zu = reinterpret_cast<float*>(ws);
  uint16_t* a2 = reinterpret_cast<uint16_t*>(ws + round_up(static_cast<size_t>(T) * f * 8, 256));
  CUtensorMap mx, mdy, mg, mu, mwd, ma2, mgT, muT;
  if (!make_map(&mx, x, d, T, kBK, kBM) || !make_map(&mdy, dy, d, T, kBK, kBM) ||
      !make_map(&mg, WgT, d, f, kBK, 128) || !make_map(&mu, WuT, d, f, kBK, 128) ||
      !make_map(&mwd, Wd, d, f, kBK, kBN) || !make_map(&ma2, a2, 3 * f, T, kBK, kBM) ||
      !make_map(&mgT, WgT, d, f, 64, kBK) || !make_map(&muT, WuT, d, f, 64, kBK))
    return TWELL_ERR_CUDA;
  // [z | u] = x [Wg | Wu]; dh = dy Wd^T with dz, du, h (bf16) in the epilogue
  GemmParams q1{};
  q1.M = T;
  q1.N = f;
  q1.K = d;
  q1.out_f32 = zu;
  q1.ldo = 2 * f;
  q1.dev_status = dev_status;
  TW_TRY(launch_gemm<kModeZU>(mx, mg, mu, q1, gemm_grid(T, f, 128, sms), s));
  GemmParams q2{};
  q2.M = T;
  q2.N = f;
  q2.K = d;
  q2.zu = zu;
  q2.a2 = a2;
  q2.t_pad = tp;
  q2.h_split = 0;
  q2.dev_status = dev_status;
  TW_TRY(launch_gemm<kModeBwdDh>(mdy, mwd, mwd, q2, gemm_grid(T, f, kBN, sms), s));
  // dx = [dz | du] [Wg; Wu]^T: K split (into a zeroed dx) only when the tiles cannot fill the GPU
  GemmParams q3{};
  q3.M = T;
  q3.N = d;
  q3.K = 2 * f;
  q3.k_split_b = f;
  q3.out_f32 = dx;
  q3.ldo = d;
  q3.k_splits_max = 1;
  q3.dev_status = dev_status;
  if (static_cast<long long>((T + kBM - 1) / kBM) * ((d + kBN - 1) / kBN) * 2 <= sms) {
    TW_TRY(zero_async(s, sms, dx, static_cast<size_t>(T) * d * sizeof(float)));
    q3.k_splits_max = 32;
  }
  TW_TRY(launch_gemm<kModeDown>(ma2, mgT, muT, q3, q3.k_splits_max > 1 ? sms : gemm_grid(T, d, kBN, sms), s));
  // dWgT = dz^T x, dWuT = du^T x, dWd = h^T dy: the [dz | du | h] block read
  // as an MN-major A operand (units along M, tokens along K; its padding rows
  // hold zeros, and rows of x and dy past T are read as zeros by the tensor
  // maps). As in the hybrid's tensor-core weight gradients, K is split
  // whenever that shortens the last wave of output tiles, the partial sums
  // added into zeroed outputs.
  CUtensorMap maT;
  if (!make_map(&maT, a2, 3 * static_cast<uint64_t>(f), tp, 64, kBK)) return TWELL_ERR_CUDA;
  const uint16_t* bT[3] = {x, x, dy};
  float* outs[3] = {dWgT, dWuT, dWd};
  const size_t wbytes = static_cast<size_t>(f) * d * sizeof(float);
  TW_TRY(zero_async(s, sms, dWgT, wbytes, dWuT, wbytes, dWd, wbytes));  // the split GEMMs add into them
  for (int i = 0; i < 3; ++i) {
    CUtensorMap mb;
    if (!make_map(&mb, bT[i], d, T, 64, kBK)) return TWELL_ERR_CUDA;
    GemmParams q{};
    q.M = f;
    q.N = d;
    q.K = tp;
    q.a_mn_major = 1;
    q.a_col_hi = i * f;
    q.out_f32 = outs[i];
    q.ldo = d;
    q.k_splits_max = 32;
    q.split_waves = 1;
    q.dev_status = dev_status;
    TW_TRY(launch_gemm<kModeDown>(maT, mb, mb, q, sms, s));
  }
  return TWELL_OK;
}

twell_status twell_column_activity(const uint16_t* x, const uint16_t* WgT, int T, int d, int f,
                                   uint32_t* active_bits, int accumulate, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_ptrs({active_bits, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!accumulate) TW_TRY(zero_async(s, sms, active_bits, static_cast<size_t>(f / 32) * 4));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT}));
  CUtensorMap ma, mb;
  if (!make_map(&ma, x, d, T, kBK, kBM) || !make_map(&mb, WgT, d, f, kBK, kBN)) return TWELL_ERR_CUDA;
  GemmParams p{};
  p.M = T;
  p.N = f;
  p.K = d;
  p.active = active_bits;
  p.dev_status = dev_status;
  return launch_gemm<kModeActivity>(ma, mb, mb, p, gemm_grid(T, f, kBN, sms), s);
}

twell_status twell_compact_columns(const uint32_t* active_bits, int f, int32_t* col_map, int32_t* f_live,
                                   void* stream) {
  if (f < 128 || f % 128 != 0 || f > 32767) return TWELL_ERR_SHAPE;
  TW_TRY(check_ptrs({active_bits, col_map, f_live}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  TW_TRY(launch(compact_columns_kernel, dim3(1), dim3(1024), 0, static_cast<cudaStream_t>(stream), active_bits, f, col_map, f_live));
  return cuda_ok(cudaGetLastError());
}

twell_status twell_gather_rows(const uint16_t* W, int f, int d, const int32_t* col_map, const int32_t* f_live,
                               int f_out, uint16_t* W_out, int32_t* dev_status, void* stream) {
  if (f < 128 || f % 128 != 0 || f > 32767 || d < 64 || d % 64 != 0 || d > 4096 || f_out < 1 || f_out > f)
    return TWELL_ERR_SHAPE;
  TW_TRY(check_ptrs({W, col_map, f_live, W_out, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  const int blocks = std::min((f_out + 7) / 8, 4 * sms);
  TW_TRY(launch(gather_weight_rows_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream), W, f, d, col_map, f_live, f_out,
                                                                                  W_out, dev_status));
  return cuda_ok(cudaGetLastError());
}

twell_status twell_unpack(const twell_t* tw, uint16_t* g_dense, int32_t* dev_status, void* stream) {
  if (tw == nullptr) return TWELL_ERR_NULL;
  TW_TRY(check_tw(tw, tw->T, tw->f));
  if (tw->T < 0 || tw->f < 128 || tw->f % 128 != 0 || tw->f > 32767) return TWELL_ERR_SHAPE;
  if (tw->T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({g_dense, dev_status}));
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  const int nT = tw->f / 128;
  const long long warps = static_cast<long long>(tw->T) * nT;
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffLL) return TWELL_ERR_SHAPE;
  TW_TRY(launch(unpack_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream), 
      tw->counts, tw->idx, tw->vals, tw->T, nT, tw->W, tw->f, g_dense, dev_status));
  return cuda_ok(cudaGetLastError());
}

twell_status twell_status_reset(int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return TWELL_ERR_NULL;
  return cuda_ok(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)));
}

twell_status twell_status_get(const int32_t* dev_status, void* stream, int32_t* host_out) {
  if (dev_status == nullptr || host_out == nullptr) return TWELL_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TW_TRY(cuda_ok(cudaMemcpyAsync(host_out, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, s)));
  return cuda_ok(cudaStreamSynchronize(s));
}

const char* twell_status_str(int status) {
  switch (status) {
    case TWELL_OK: return "ok";
    case TWELL_ERR_NULL: return "a required pointer is NULL";
    case TWELL_ERR_SHAPE: return "a size is out of range or the TwELL descriptor does not match";
    case TWELL_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case TWELL_ERR_WORKSPACE: return "workspace missing or too small";
    case TWELL_ERR_CUDA: return "a CUDA call failed";
    case TWELL_ERR_DEVICE: return "the current device is not compute capability 10.0 (B200)";
    case TWELL_ERR_OVERFLOW: return "a row had more nonzeros in a tile than the ELL width (non-hybrid forward)";
    case TWELL_ERR_INDEX: return "a stored column or row index was out of range";
    case TWELL_ERR_TIMEOUT: return "a bounded on-chip wait gave up";
    default: return "unknown status";
  }
}

const char* twell_version(void) { return "twell-b200 0.1"; }

}  // extern "C"

// ====================================================================== no-allocation variant
//
// Some callers cannot hand the library a workspace: code that runs where
// device allocation is not allowed or not wanted (inside a framework that owns
// every byte of device memory through its own pool, a real-time loop that must
// not call the allocator, or a plugin whose host gives it only its inputs and
// outputs). For them the hybrid forward can run on a scratch area that lives in
// the library itself: a fixed array in device memory, created when the module
// is loaded on a device and held until the process exits.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // == TWELL_NOALLOC_SCRATCH_BYTES

// Device-side scratch shared by every call of twell_ffn_hybrid_forward_noalloc
// on a device. In host code this name is only a handle: its device address is
// obtained once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void*> g_noalloc_ptr[kMaxDevices];

// Device address of the scratch for the current device `dev`. It is looked up
// with that device current on the first call that succeeds in doing so and
// kept from then on; a failed lookup is not kept, so the next call tries
// again. (Two threads making their first calls at once may both look it up;
// they get the same address.)
void* noalloc_scratch(int dev) {
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_noalloc_ptr[dev].store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" twell_status twell_ffn_hybrid_forward_noalloc(const uint16_t* x, const uint16_t* WgT,
                                                         const uint16_t* WuT, const uint16_t* Wd, int T, int d,
                                                         int f, const twell_t* tw, float* y, int32_t* ovf_rows,
                                                         int32_t* n_ovf, int32_t* dev_status, void* stream) {
  TW_TRY(check_shape(T, d, f));
  TW_TRY(check_tw(tw, T, f));
  if (T == 0) return TWELL_OK;
  TW_TRY(check_ptrs({x, WgT, WuT, Wd, y, ovf_rows, n_ovf, dev_status}));
  const size_t need = twell_hybrid_workspace_bytes(T, d, f);
  if (need > kNoAllocScratchBytes) return TWELL_ERR_WORKSPACE;
  int dev, sms;
  TW_TRY(current_device(&dev, &sms));
  void* ws = noalloc_scratch(dev);
  if (ws == nullptr) return TWELL_ERR_CUDA;
  return twell_ffn_hybrid_forward(x, WgT, WuT, Wd, T, d, f, tw, y, ovf_rows, n_ovf, ws, need, dev_status, stream);
}
