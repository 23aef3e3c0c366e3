// Host side of the backward pass through the hybrid format: the workspace
// layout and the launch sequences of its two halves (dx, then the weight
// gradients). Included by twell_api.cu inside its internal namespace, after
// the forward's helpers it reuses (launch, zero_async, make_map, gather).
#pragma once

// Workspace of the hybrid backward, carved in this order (each piece 256-byte
// aligned): per-slot records {h, du, dz, token} of the rows that fit
// ([T][nT][W] float4); for the overflow rows, the gathered rows of x and dy
// ([Tp][d] bf16 each, Tp = T rounded up to 64), their [z | u] ([T][2f] fp32;
// before that, dh = dy . Wd^T of every token, [T][f] fp32),
// [dz | du | dz_lo | du_lo | h | h_lo] ([Tp][6f] bf16); the column
// counts/cursors ([f]), column
// offsets ([f + 1]) and the column-sorted records (one float4 per slot of the
// rows that fit); for the tensor-core form of the weight gradients, the rows
// that fit as dense token-major [dz | du | dz_lo | du_lo | h | h_lo] ([T][6f]
// bf16, within a region of 6 f Tp elements).
struct BwdWorkspace {
  float4* rec;
  uint16_t *xo, *dyo;
  float* zu;
  uint16_t* a2;
  int *colcnt, *colptr;
  float4* list;
  int* counters;    // work counters of the dx passes
  uint16_t* dense;  // tensor-core form: the rows that fit, [T][6f] bf16 (dz, du, their remainders, h, its remainder)
  int t_pad;
  size_t bytes;
};

BwdWorkspace bwd_carve(char* base, int T, int d, int f, int W) {
  const size_t nT = static_cast<size_t>(f) / 128;
  const size_t s0 = static_cast<size_t>(T) * nT * W;
  const size_t tp = round_up(static_cast<size_t>(T), 64);
  BwdWorkspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += round_up(bytes, 256);
    return p;
  };
  w.rec = reinterpret_cast<float4*>(take(s0 * 16));
  w.xo = reinterpret_cast<uint16_t*>(take(tp * d * 2));
  w.dyo = reinterpret_cast<uint16_t*>(take(tp * d * 2));
  w.zu = reinterpret_cast<float*>(take(static_cast<size_t>(T) * f * 8));
  w.a2 = reinterpret_cast<uint16_t*>(take(tp * f * 12));
  w.colcnt = reinterpret_cast<int*>(take(static_cast<size_t>(f) * 4));
  w.colptr = reinterpret_cast<int*>(take((static_cast<size_t>(f) + 1) * 4));
  w.list = reinterpret_cast<float4*>(take(s0 * 16));
  w.dense = reinterpret_cast<uint16_t*>(take(3 * static_cast<size_t>(f) * 2 * tp * 2));
  w.counters = reinterpret_cast<int*>(take(16));
  w.t_pad = static_cast<int>(tp);
  w.bytes = off;
  return w;
}

template <int NCH, int WARPS>
twell_status launch_bwd_pass(void (*kern)(BwdParams), size_t smem, const BwdParams& p, int sms, cudaStream_t s) {
  // always opt in: the static shared memory adds to the dynamic size
  TW_TRY(cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))));
  const long long want = (static_cast<long long>(p.rows) + WARPS - 1) / WARPS;
  const int blocks = static_cast<int>(std::max(1LL, std::min<long long>(want, sms)));
  return launch(kern, dim3(blocks), dim3(WARPS * 32), smem, s, p);
}

// Wg and Wu bytes above which the per-token dx pass runs once per matrix.
constexpr size_t kDxSplitBytes = 64u << 20;

// The per-token dx pass of the rows that fit.
template <int NCH>
twell_status launch_bwd_dx_n(const BwdParams& p, int sms, cudaStream_t s) {
  constexpr int kDx = bwd_dx_warps(NCH);
  return launch_bwd_pass<NCH, kDx>(bwd_dx_kernel<NCH, kDx>, bwd_dx_smem_bytes(NCH), p, sms, s);
}

twell_status launch_bwd_dx(const BwdParams& p, int sms, cudaStream_t s) {
  switch ((p.d + 255) / 256) {
    case 1: return launch_bwd_dx_n<1>(p, sms, s);
    case 2: return launch_bwd_dx_n<2>(p, sms, s);
    case 3: return launch_bwd_dx_n<3>(p, sms, s);
    case 4: return launch_bwd_dx_n<4>(p, sms, s);
    case 5: return launch_bwd_dx_n<5>(p, sms, s);
    case 6: return launch_bwd_dx_n<6>(p, sms, s);
    case 7: return launch_bwd_dx_n<7>(p, sms, s);
    case 8: return launch_bwd_dx_n<8>(p, sms, s);
    case 9: return launch_bwd_dx_n<9>(p, sms, s);
    case 10: return launch_bwd_dx_n<10>(p, sms, s);
    case 11: return launch_bwd_dx_n<11>(p, sms, s);
    case 12: return launch_bwd_dx_n<12>(p, sms, s);
    case 13: return launch_bwd_dx_n<13>(p, sms, s);
    case 14: return launch_bwd_dx_n<14>(p, sms, s);
    case 15: return launch_bwd_dx_n<15>(p, sms, s);
    case 16: return launch_bwd_dx_n<16>(p, sms, s);
    default: return TWELL_ERR_SHAPE;
  }
}

// dx, and the per-slot records the weight gradients read, in the workspace. tc_dx: the
// rows that fit get dx from one tensor-core GEMM over their scattered dz, du
// instead of the per-token axpy pass.
twell_status backward_dx_impl(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, const uint16_t* Wd,
                              const uint16_t* dy, int T, int d, int f, const twell_t* tw, const int32_t* ovf_rows,
                              const int32_t* n_ovf, float* dx, char* ws, int32_t* dev_status, cudaStream_t s,
                              int sms, bool tc_dx = false) {
  const int nT = f / 128;
  BwdWorkspace w = bwd_carve(ws, T, d, f, tw->W);
  BwdParams p0{};
  p0.x = x;
  p0.WgT = WgT;
  p0.WuT = WuT;
  p0.dh = w.zu;
  p0.counts = tw->counts;
  p0.idx = tw->idx;
  p0.vals = tw->vals;
  p0.row_ovf = tw->row_ovf;
  p0.rows = T;
  p0.d = d;
  p0.f = f;
  p0.nT = nT;
  p0.W = tw->W;
  p0.dx = dx;
  p0.s_rec = w.rec;
  p0.dev_status = dev_status;
  // 0. the records {h, du, dz, t} of the stored slots of the rows that fit,
  // from dh = dy . Wd^T and u = x Wu^T on the tensor cores (cheaper than a
  // dot product over a gathered weight row per slot).
  const long long dh_tiles = static_cast<long long>((T + kBM - 1) / kBM) * ((f + kBN - 1) / kBN);
  if (dh_tiles >= sms) {
    // The output tiles fill the GPU without splitting K: two GEMMs whose
    // epilogues take only the stored slots' entries, dh_j into the records
    // first, then the records from u_j (dh and u are never written in full).
    const uint16_t* a_op[2] = {dy, x};
    const uint16_t* b_op[2] = {Wd, WuT};
    for (int pass = 0; pass < 2; ++pass) {
      CUtensorMap ma, mb;
      if (!make_map(&ma, a_op[pass], d, T, kBK, kBM) || !make_map(&mb, b_op[pass], d, f, kBK, kBN))
        return TWELL_ERR_CUDA;
      GemmParams q{};
      q.M = T;
      q.N = f;
      q.K = d;
      q.counts = const_cast<int16_t*>(tw->counts);
      q.idx = const_cast<int16_t*>(tw->idx);
      q.vals = const_cast<uint16_t*>(tw->vals);
      q.row_ovf = const_cast<uint8_t*>(tw->row_ovf);
      q.nT = nT;
      q.W = tw->W;
      q.s_rec = w.rec;
      q.slots_pass = pass;
      q.dev_status = dev_status;
      TW_TRY(launch_gemm<kModeSlots>(ma, mb, mb, q, gemm_grid(T, f, kBN, sms), s));
    }
  } else {
    // Small batches: both products in full, fp32 [T][f] in the [z | u] region
    // (free until the overflow rows' dense branch below), with K split over
    // the grid (partial sums added into zeroed rows), then the records.
    float* ubuf = w.zu + static_cast<size_t>(T) * f;
    TW_TRY(zero_async(s, sms, w.zu, static_cast<size_t>(T) * f * 2 * sizeof(float)));
    TW_TRY(f32_gemm_impl(dy, T, Wd, f, d, w.zu, f, dev_status, s, sms));
    TW_TRY(f32_gemm_impl(x, T, WuT, f, d, ubuf, f, dev_status, s, sms));
    const long long pairs = static_cast<long long>(T) * nT;  // four per warp, eight warps per block
    const int rb = static_cast<int>(std::min<long long>((pairs + 31) / 32, 8LL * sms));
    TW_TRY(launch(bwd_records_kernel, dim3(std::max(rb, 1)), dim3(256), 0, s, p0, static_cast<const float*>(ubuf)));
    TW_TRY(cuda_ok(cudaGetLastError()));
  }
  if (!tc_dx) {
    // 1b. dx of the rows that fit, per token. When Wg and Wu together would not
    // stay in L2 beside the streamed rows, one pass per matrix (the second
    // adding into dx) keeps each pass's gathered rows resident.
    // Every warp of a pass takes its tokens from one counter (a zeroed int per
    // pass), so blocks whose tokens hold more slots do not set its end.
    TW_TRY(zero_async(s, sms, w.counters, 8));
    p0.dx_mats = 3;
    p0.next_row_global = w.counters;
    if (2ull * static_cast<size_t>(f) * d * 2 > kDxSplitBytes) {
      p0.dx_mats = 1;
      TW_TRY(launch_bwd_dx(p0, sms, s));
      p0.dx_mats = 2;
      p0.dx_accumulate = 1;
      p0.next_row_global = w.counters + 1;
    }
    TW_TRY(launch_bwd_dx(p0, sms, s));
  }
  if (tc_dx) {
    // 1b. dx of every token = [dz | du | dz_lo | du_lo] [Wg; Wu; Wg; Wu]^T on
    // the tensor cores, the rows that fit scattered token-major into the
    // [z | u] region (dh there is no longer needed), overflow rows left zero
    // (their dx is rewritten below). K is split over the grid, with partial
    // sums added into zeroed rows, when the output tiles cannot fill it (a
    // split that only shortens the last wave measured slower here: the
    // zeroing and the added partial sums of dx cost more than it saves).
    uint16_t* a2all = reinterpret_cast<uint16_t*>(w.zu);
    const long long dx_tiles = static_cast<long long>((T + kBM - 1) / kBM) * ((d + kBN - 1) / kBN);
    if (dx_tiles < sms) TW_TRY(zero_async(s, sms, dx, static_cast<size_t>(T) * d * 4));
    SlotSource src{tw->counts, tw->idx, w.rec, tw->row_ovf, T, nullptr, nT, tw->W, f, 1};
    TW_TRY(launch(bwd_dense_rows_kernel<false>, dim3(8 * sms), dim3(256), 0, s, src, a2all));
    CUtensorMap ma, mgT, muT;
    if (!make_map(&ma, a2all, 4 * f, T, kBK, kBM) || !make_map(&mgT, WgT, d, f, 64, kBK) ||
        !make_map(&muT, WuT, d, f, 64, kBK))
      return TWELL_ERR_CUDA;
    GemmParams q{};
    q.M = T;
    q.N = d;
    q.K = 4 * f;
    q.k_wrap = 2 * f;
    q.k_split_b = f;
    q.out_f32 = dx;
    q.ldo = d;
    q.k_splits_max = 32;
    q.dev_status = dev_status;
    TW_TRY(launch_gemm<kModeDown>(ma, mgT, muT, q, dx_tiles < sms ? sms : gemm_grid(T, d, kBN, sms), s));
  }
  // 2. overflow rows, dense on the tensor cores: gather x and dy (zero the dx
  // rows and the padding rows up to a multiple of 64), recompute [z | u], then
  // dh = dy Wd^T with dz, du, h in its epilogue, then dx = [dz | du] [Wg; Wu]^T
  TW_TRY(launch(gather_rows_kernel, dim3(sms * 2), dim3(256), 0, s, x, d, ovf_rows, n_ovf, T, w.xo, dx, dev_status, w.t_pad));
  TW_TRY(cuda_ok(cudaGetLastError()));
  TW_TRY(launch(gather_rows_kernel, dim3(sms * 2), dim3(256), 0, s, dy, d, ovf_rows, n_ovf, T, w.dyo, nullptr, dev_status, w.t_pad));
  TW_TRY(cuda_ok(cudaGetLastError()));
  CUtensorMap mx, mdy, mg, mu, mwd, ma2, mgT, muT;
  if (!make_map(&mx, w.xo, d, T, kBK, kBM) || !make_map(&mdy, w.dyo, d, T, kBK, kBM) ||
      !make_map(&mg, WgT, d, f, kBK, 128) || !make_map(&mu, WuT, d, f, kBK, 128) ||
      !make_map(&mwd, Wd, d, f, kBK, kBN) || !make_map(&ma2, w.a2, 6 * f, T, kBK, kBM) ||
      !make_map(&mgT, WgT, d, f, 64, kBK) || !make_map(&muT, WuT, d, f, 64, kBK))
    return TWELL_ERR_CUDA;
  GemmParams q1{};
  q1.M = T;
  q1.M_dev = n_ovf;
  q1.N = f;
  q1.K = d;
  q1.out_f32 = w.zu;
  q1.ldo = 2 * f;
  q1.dev_status = dev_status;
  TW_TRY(launch_gemm<kModeZU>(mx, mg, mu, q1, sms, s));
  GemmParams q2{};
  q2.M = T;
  q2.M_dev = n_ovf;
  q2.N = f;
  q2.K = d;
  q2.zu = w.zu;
  q2.a2 = w.a2;
  q2.t_pad = w.t_pad;
  q2.h_split = 1;
  q2.dev_status = dev_status;
  TW_TRY(launch_gemm<kModeBwdDh>(mdy, mwd, mwd, q2, sms, s));
  GemmParams q3{};
  q3.M = T;
  q3.M_dev = n_ovf;
  q3.N = d;
  q3.K = 4 * f;
  q3.k_wrap = 2 * f;
  q3.k_split_b = f;
  q3.out_f32 = dx;
  q3.ldo = d;
  q3.row_map = ovf_rows;
  q3.out_rows = T;
  q3.k_splits_max = 32;  // the gather zeroed these dx rows
  q3.split_waves = 1;
  q3.dev_status = dev_status;
  return launch_gemm<kModeDown>(ma2, mgT, muT, q3, sms, s);
}

twell_status backward_dw_overflow(int d, int f, const int32_t* n_ovf, float* dWgT, float* dWuT, float* dWd,
                                  const BwdWorkspace& w, cudaStream_t s, int sms);

// Weight gradients from the workspace filled by backward_dx_impl.
twell_status backward_dw_impl(const uint16_t* x, const uint16_t* dy, int T, int d, int f, const twell_t* tw,
                              const int32_t* n_ovf, float* dWgT, float* dWuT, float* dWd, char* ws, cudaStream_t s,
                              int sms) {
  const int nT = f / 128;
  BwdWorkspace w = bwd_carve(ws, T, d, f, tw->W);
  // 3. weight gradients of the rows that fit: sort their slots by column, then
  // sum per column (every row of dW is written)
  SlotSource a{tw->counts, tw->idx, w.rec, tw->row_ovf, T, nullptr, nT, tw->W, f, 1};
  TW_TRY(zero_async(s, sms, w.colcnt, static_cast<size_t>(f) * 4));
  const int cblocks = 4 * sms;
  TW_TRY(launch(bwd_columns_kernel<false>, dim3(cblocks), dim3(256), 0, s, a, w.colcnt, w.colptr, w.list));
  TW_TRY(launch(bwd_column_scan_kernel, dim3(1), dim3(1024), 0, s, w.colcnt, f, w.colptr));
  TW_TRY(launch(bwd_columns_kernel<true>, dim3(cblocks), dim3(256), 0, s, a, w.colcnt, w.colptr, w.list));
  TW_TRY(cuda_ok(cudaGetLastError()));
  WgradParams g{};
  g.list = w.list;
  g.colptr = w.colptr;
  g.x0 = x;
  g.dy0 = dy;
  g.f = f;
  g.d = d;
  g.dWgT = dWgT;
  g.dWuT = dWuT;
  g.dWd = dWd;
  const long long warps = static_cast<long long>(f) * ((d + 255) / 256);
  TW_TRY(launch(bwd_wgrad_kernel, dim3(static_cast<unsigned>((warps + 7) / 8)), dim3(256), 0, s, g));
  TW_TRY(cuda_ok(cudaGetLastError()));
  return backward_dw_overflow(d, f, n_ovf, dWgT, dWuT, dWd, w, s, sms);
}

// The overflow rows' share of the weight gradients, on the tensor cores:
// dWgT += dz^T x, dWuT += du^T x, dWd += h^T dy over the gathered rows (K =
// their tokens, as bf16 value and remainder halves).
twell_status backward_dw_overflow(int d, int f, const int32_t* n_ovf, float* dWgT, float* dWuT, float* dWd,
                                  const BwdWorkspace& w, cudaStream_t s, int sms) {
  // A: the overflow rows' [dz | du | dz_lo | du_lo | h | h_lo] block (token-major,
  // read MN-major: units along M, the gathered tokens along K, values then
  // remainders); K sized on the device to the overflow count rounded up to 64
  // (the padding rows of the block and of xo, dyo hold zeros).
  CUtensorMap ma;
  if (!make_map(&ma, w.a2, 6 * static_cast<uint64_t>(f), w.t_pad, 64, kBK)) return TWELL_ERR_CUDA;
  const uint16_t* bT[3] = {w.xo, w.xo, w.dyo};
  float* outs[3] = {dWgT, dWuT, dWd};
  const int col_hi[3] = {0, f, 4 * f}, col_lo[3] = {2 * f, 3 * f, 5 * f};
  for (int i = 0; i < 3; ++i) {
    CUtensorMap mb;
    if (!make_map(&mb, bT[i], d, w.t_pad, 64, kBK)) return TWELL_ERR_CUDA;
    GemmParams q{};
    q.M = f;
    q.N = d;
    q.K = 2 * w.t_pad;
    q.k_wrap = w.t_pad;
    q.k_dev = n_ovf;
    q.k_half = w.t_pad;
    q.a_mn_major = 1;
    q.a_col_hi = col_hi[i];
    q.a_col_lo = col_lo[i];
    q.accumulate = 1;
    q.k_splits_max = 32;
    q.out_f32 = outs[i];
    q.ldo = d;
    q.dev_status = nullptr;
    TW_TRY(launch_gemm<kModeDown>(ma, mb, mb, q, sms, s));
  }
  return TWELL_OK;
}

// Tensor-core form of the weight gradients from the workspace filled by
// backward_dx_impl: the records of the rows that fit are written densely
// (bf16 value and remainder) by token, three GEMMs over all tokens give their
// share, then the overflow rows' GEMMs add theirs.
twell_status backward_dw_tc_impl(const uint16_t* x, const uint16_t* dy, int T, int d, int f, const twell_t* tw,
                                 const int32_t* n_ovf, float* dWgT, float* dWuT, float* dWd, char* ws,
                                 cudaStream_t s, int sms) {
  const int nT = f / 128;
  BwdWorkspace w = bwd_carve(ws, T, d, f, tw->W);
  // The records of the rows that fit, token-major: [dz | du | dz_lo | du_lo |
  // h | h_lo] (6 f bf16 per token, in the region of 6 f t_pad elements that
  // the weight gradients own). The three GEMMs read them as an MN-major A
  // (units along M, tokens along K), so no transposition by unit is needed.
  SlotSource a{tw->counts, tw->idx, w.rec, tw->row_ovf, T, nullptr, nT, tw->W, f, 1};
  uint16_t* rows = w.dense;
  TW_TRY(launch(bwd_dense_rows_kernel<true>, dim3(8 * sms), dim3(256), 0, s, a, rows));
  TW_TRY(cuda_ok(cudaGetLastError()));
  CUtensorMap ma;
  if (!make_map(&ma, rows, 6 * static_cast<uint64_t>(f), T, 64, kBK)) return TWELL_ERR_CUDA;
  // K runs over the tokens twice (values, then remainders); rows of the block,
  // x and dy past T read as zeros. K is split whenever that shortens the last
  // wave of output tiles (e.g. 192 tiles on 148 SMs: three splits, 1.33 waves
  // instead of 2), the partial sums added into zeroed outputs.
  const uint16_t* bT[3] = {x, x, dy};
  float* outs[3] = {dWgT, dWuT, dWd};
  const int col_hi[3] = {0, f, 4 * f}, col_lo[3] = {2 * f, 3 * f, 5 * f};
  const size_t wbytes = static_cast<size_t>(f) * d * sizeof(float);
  TW_TRY(zero_async(s, sms, dWgT, wbytes, dWuT, wbytes, dWd, wbytes));  // the split GEMMs add into them
  for (int i = 0; i < 3; ++i) {
    CUtensorMap mb;
    if (!make_map(&mb, bT[i], d, T, 64, kBK)) return TWELL_ERR_CUDA;
    GemmParams q{};
    q.M = f;
    q.N = d;
    q.K = 2 * w.t_pad;
    q.k_wrap = w.t_pad;  // [value | remainder] halves against the same rows of x (or dy)
    q.a_mn_major = 1;
    q.a_col_hi = col_hi[i];
    q.a_col_lo = col_lo[i];
    q.out_f32 = outs[i];
    q.ldo = d;
    q.k_splits_max = 32;
    q.split_waves = 1;
    TW_TRY(launch_gemm<kModeDown>(ma, mb, mb, q, sms, s));
  }
  return backward_dw_overflow(d, f, n_ovf, dWgT, dWuT, dWd, w, s, sms);
}
