/*
 * twell.h -- C ABI of the TwELL sparse ReLU-gated FFN forward pass (B200, sm_100a).
 *
 * The layer is y = (ReLU(x Wg) * (x Wu)) Wd. Hidden units whose gate is not
 * strictly positive are exact zeros and are skipped: the gate GEMM packs its
 * ReLU output into Tile-wise ELLPACK (TwELL) in its own epilogue, with no
 * separate pack launch and no extra pass over memory, and a fused kernel then
 * computes the up and down projections only for the stored hidden units,
 * keeping the hidden activations on chip. Rows whose nonzeros do not fit the
 * ELL width go to a dense branch.
 *
 * Sources: intellectnews.ru, "Sakana AI и NVIDIA ... TwELL" -- sections
 * "Формат TwELL вместо классической sparse-упаковки" (format, packed at the
 * end of the producing pass), "Слитые CUDA-ядра для инференса и гибрид для
 * обучения" (fused inference kernel; hybrid sparse/dense rows) and
 * "Минимальные изменения в рецепте обучения" (ReLU gate gives exact zeros);
 * gate.com post 20977915, paragraph on TwELL (tiles packed locally by each
 * compute unit).
 *
 * Conventions for every entry point:
 *   - bf16 values travel as uint16_t bit patterns.
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no memory and keeps no per-call state. It is safe to call from
 *     several host threads on distinct buffers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are stream-ordered and never synchronise the host.
 *   - Argument errors are returned synchronously and nothing is launched.
 *     Conditions found on the device (ELL overflow in the non-hybrid forward,
 *     an out-of-range stored index, a bounded wait that gave up) are raised
 *     into the caller's int32 `dev_status` with an atomic max; `dev_status`
 *     is sticky until the caller resets it (twell_status_reset).
 *   - Every pointer must be 16-byte aligned.
 *
 * Shapes: T tokens (T >= 0; T == 0 is a no-op), d = d_model, f = d_ff.
 *   d % 64 == 0, 64 <= d <= 4096; f % 128 == 0, 128 <= f <= 32767;
 *   tile == 128; W % 8 == 0, 8 <= W <= 128.
 *
 * Layouts (row-major):
 *   x   [T][d]   bf16 activations
 *   WgT [f][d]   gate weight, transposed (row j = column j of Wg; this is the
 *                weight of an nn.Linear(d, f))
 *   WuT [f][d]   up weight, transposed likewise
 *   Wd  [f][d]   down weight (row j multiplies hidden unit j)
 *   y   [T][d]   fp32 output (accumulated in fp32 and stored without a final
 *                rounding to bf16; the hidden activations of the dense paths
 *                are held as bf16)
 */
#ifndef TWELL_H
#define TWELL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum twell_status {
  TWELL_OK = 0,
  TWELL_ERR_NULL = 1,        /* a required pointer is NULL */
  TWELL_ERR_SHAPE = 2,       /* a size is outside the ranges above, or tw does not match */
  TWELL_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  TWELL_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the size query */
  TWELL_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed (launch, tensor map) */
  TWELL_ERR_DEVICE = 6,      /* the current device is not compute capability 10.0 */
  /* device-side codes, raised into dev_status */
  TWELL_ERR_OVERFLOW = 16,   /* a row of the non-hybrid forward had a tile count > W */
  TWELL_ERR_INDEX = 17,      /* a stored column index was outside [0, f) */
  TWELL_ERR_TIMEOUT = 18     /* a bounded on-chip wait gave up; outputs are undefined */
} twell_status;

/*
 * TwELL buffers (Tile-wise ELLPACK of ReLU(x Wg)), all caller-owned device memory.
 * The columns are cut into nT = f / tile tiles. For row t and tile c:
 *   counts[t*nT + c]          true number of strictly positive gate values in
 *                             the tile (not capped at W)
 *   idx [(t*nT + c)*W + s]    global column index j (0..f-1) of the s-th
 *                             positive value in ascending column order
 *   vals[(t*nT + c)*W + s]    bf16 (nearest-even) of ReLU(z[t, j])
 * for s < min(count, W). Slots from min(count, W) on are unspecified.
 *   row_ovf[t]                1 iff some tile of row t has count > W, else 0.
 */
typedef struct twell_t {
  int16_t* counts;   /* [T][nT]    */
  int16_t* idx;      /* [T][nT][W] */
  uint16_t* vals;    /* [T][nT][W] bf16 bits */
  uint8_t* row_ovf;  /* [T]        */
  int32_t T, f, tile, W;
} twell_t;

/*
 * Gate GEMM with the TwELL pack in its epilogue (steps: z = x Wg on the tensor
 * cores, ReLU, per-row per-tile compaction; source: the format section above).
 * Writes tw->counts, tw->idx, tw->vals, tw->row_ovf. tw->T, tw->f must equal
 * T, f; tw->tile must be 128.
 */
twell_status twell_gate_pack(const uint16_t* x, const uint16_t* WgT, int T, int d, int f,
                             const twell_t* tw, int32_t* dev_status, void* stream);

/*
 * Fused sparse step alone, on an already packed tw: for each stored slot
 * (j, g) of row t, u_j = x_t . Wu[:, j], h_j = g * u_j, y_t += h_j Wd[j, :]
 * with fp32 accumulation; h never leaves the chip (source: the fused-kernel
 * section above). Rows with row_ovf set are skipped (y rows left untouched)
 * when skip_overflow_rows != 0; otherwise they use their first W slots, their
 * y is undefined and dev_status is raised to TWELL_ERR_OVERFLOW.
 */
twell_status twell_sparse_ffn(const uint16_t* x, const uint16_t* WuT, const uint16_t* Wd,
                              int T, int d, int f, const twell_t* tw, int skip_overflow_rows,
                              float* y, int32_t* dev_status, void* stream);

/*
 * Whole non-hybrid forward: twell_gate_pack, then twell_sparse_ffn without
 * skipping (source: intellectnews.ru "Sakana AI и NVIDIA ... TwELL", section
 * "Слитые CUDA-ядра для инференса и гибрид для обучения": at inference the
 * packed gate output feeds fused kernels that do the rest of the FFN for the
 * stored units only; section "Формат TwELL вместо классической
 * sparse-упаковки": the pack is formed at the end of the gate's own pass).
 * If any row overflows, dev_status becomes TWELL_ERR_OVERFLOW and the y of
 * the overflowing rows is undefined (other rows are correct).
 */
twell_status twell_ffn_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                               const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                               float* y, int32_t* dev_status, void* stream);

/*
 * Variant for mid densities, where the dense up projection on the tensor
 * cores costs less than gathering Wu rows on the CUDA cores (not on the
 * pages; the pages' kernels target H100). One GEMM forms z = x Wg and
 * u = x Wu together ([Wg; Wu] stacked in each MMA); its epilogue packs the
 * positions where z > 0 exactly as twell_gate_pack does (same counts, indices
 * and overflow flags) but stores h_j = bf16(ReLU(z_j) * u_j) in `vals`.
 */
twell_status twell_gate_up_pack(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT, int T, int d,
                                int f, const twell_t* tw, int32_t* dev_status, void* stream);

/*
 * Down projection from a TwELL holding hidden activations (twell_gate_up_pack):
 * y_t = sum over stored slots (j, h) of h * Wd[j, :], fp32 accumulation, fp32
 * y. Overflow handling as in twell_sparse_ffn.
 */
twell_status twell_sparse_down(const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                               int skip_overflow_rows, float* y, int32_t* dev_status, void* stream);

/*
 * The same down projection per 128-row tile over the tile's union of stored
 * units, on the tensor cores (same source as twell_sparse_down; the grouping
 * of rows into tiles and their unions is this library's). For
 * each tile of 128 rows, the units that its rows that fit have stored (the
 * union, ascending) are collected, the tile's hidden values over that union
 * are written as a bf16 block in `workspace`, and y_tile = block . Wd[union, :]
 * runs on tcgen05 with K = the tile's union (the union's rows of Wd gathered
 * into shared memory per K block by TMA, four rows per instruction). y as for
 * twell_sparse_down (fp32 sums of
 * the same exact products, in another order), except that with
 * skip_overflow_rows != 0 the overflow rows' y is written as zeros (the
 * dense branch rewrites it) instead of left untouched; with
 * skip_overflow_rows == 0 they use their first W slots, their y is undefined
 * and dev_status is raised to TWELL_ERR_OVERFLOW. workspace: at least twell_sparse_down_union_workspace_bytes(T, d, f) bytes,
 * 16-byte aligned, caller-owned, overwritten. A stored index outside its own
 * column tile raises TWELL_ERR_INDEX and adds nothing. Two kernel launches.
 * Measured on B200 it is slower than twell_sparse_down at the 0.5B, 1.5B and
 * 2B layers (the row gather is the wall), so the hybrid forwards do not use
 * it.
 */
twell_status twell_sparse_down_union(const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                                     int skip_overflow_rows, float* y, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream);

/* Workspace bytes of twell_sparse_down_union: about (T + 127) * f * 2 (the
 * tiles' hidden-value blocks) plus the tiles' union lists. */
size_t twell_sparse_down_union_workspace_bytes(int T, int d, int f);

/*
 * 1 if twell_ffn_hybrid_forward_tc_up and twell_relu_ffn_hybrid_forward would
 * run their down projection as twell_sparse_down_union for this shape and
 * workspace, 0 if as twell_sparse_down. Always 0: the union form is an
 * explicit entry point only (see above).
 */
int twell_hybrid_down_is_union(int T, int d, int f, size_t workspace_bytes);

/*
 * Hybrid forward of the tensor-core-up variant: twell_gate_up_pack,
 * twell_route, twell_sparse_down of the rows that fit (overflow rows
 * skipped), and the dense branch on ovf_rows. Same arguments and workspace as
 * twell_ffn_hybrid_forward. The dense branch does not recompute the gate and
 * up GEMMs: the gate+up GEMM writes each overflowing (row, tile)'s exact
 * hidden activations h = ReLU(z) u (bf16 value and bf16 remainder) into the
 * workspace at the row's compact slot, the row's other tiles take their
 * nonzeros from the pack (bf16 h, every nonzero of a tile that fits is
 * stored), and one down GEMM adds them times Wd into the zeroed rows of y.
 * Batches of at most 8 tokens (d a multiple of 256) run the GEMV path of
 * twell_ffn_hybrid_forward with the hidden values packed.
 */
twell_status twell_ffn_hybrid_forward_tc_up(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                            const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                                            float* y, int32_t* ovf_rows, int32_t* n_ovf, void* workspace,
                                            size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Routing step of the hybrid route (source: the hybrid paragraph of the
 * fused-kernel section above): ovf_rows[0..n_ovf) = rows with row_ovf set,
 * in ascending order; *n_ovf (device int32) = their number. ovf_rows has T
 * entries of room.
 */
twell_status twell_route(const twell_t* tw, int32_t* ovf_rows, int32_t* n_ovf, void* stream);

/* Bytes of workspace needed by twell_ffn_hybrid_forward and
 * twell_dense_rows_forward (worst case: every row overflows). For batches of
 * 9 to 512 tokens the hybrid forward also uses the hidden-activation part of
 * it for the fp32 gate pre-activations of its split-K gate GEMM, before the
 * dense branch runs; for batches of at most 8 tokens the dense branch keeps its
 * hidden activations there in fp32. */
size_t twell_hybrid_workspace_bytes(int T, int d, int f);

/*
 * Dense branch of the hybrid route alone (source: the hybrid paragraph of the
 * fused-kernel section above): for i < *n_rows (device int32, <= T), row
 * r = rows[i] of y is set to the dense gated FFN of x[r] -- gate recomputed,
 * h = ReLU(x Wg) * (x Wu) on the tensor cores, then h Wd. h is kept as a pair
 * of bf16 values (bf16(h) and the bf16 of the remainder), so the rounding of
 * the hidden activations costs ~2^-16 relative instead of 2^-8; rows routed
 * here have many active units and large outputs. The rows are gathered into
 * `workspace`, which also holds their hidden activations (size:
 * twell_hybrid_workspace_bytes). Rows not listed are untouched. A listed row
 * outside [0, T) is skipped and raises TWELL_ERR_INDEX.
 */
twell_status twell_dense_rows_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, int T, int d, int f, const int32_t* rows,
                                      const int32_t* n_rows, float* y, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Whole hybrid forward = twell_gate_pack, twell_route, twell_sparse_ffn with
 * overflowing rows skipped, and twell_dense_rows_forward on ovf_rows (source:
 * intellectnews.ru "Sakana AI и NVIDIA ... TwELL", section "Слитые CUDA-ядра
 * для инференса и гибрид для обучения": rows whose active units do not fit
 * the sparse format are handled in dense form, the rest sparsely; the pages
 * describe this split for training and this library applies the same rule to
 * the forward pass). Every row of y is written. `workspace` holds the gathered
 * overflow rows and their hidden activations.
 * Batches of at most 8 tokens take a CUDA-core path (a weight GEMM tile would
 * hold 1-8 real rows): the gate is a GEMV whose epilogue makes the pack, four
 * blocks per column tile exchanging their partial counts through distributed
 * shared memory; routing derives the overflow flags from the counts; the dense
 * branch is a pair of GEMVs over the listed rows with fp32 hidden activations.
 * The same holds for twell_ffn_hybrid_forward_tc_up and
 * twell_relu_ffn_hybrid_forward.
 */
twell_status twell_ffn_hybrid_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                                      float* y, int32_t* ovf_rows, int32_t* n_ovf,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream);

/*
 * Hybrid forward without a caller-provided workspace (the paper has no
 * counterpart; this is a convenience of this library).
 *
 * For callers that cannot allocate device memory for a workspace -- code that
 * runs inside a framework that owns all device memory through its own pool,
 * a loop that must never reach the allocator, or a plugin whose host passes it
 * only inputs and outputs. Same arguments and results as
 * twell_ffn_hybrid_forward minus the workspace: the gathered overflow rows and
 * their hidden activations go to a scratch array compiled into the library
 * (TWELL_NOALLOC_SCRATCH_BYTES of device memory, held on every device that
 * loads the library until the process exits). The call itself allocates
 * nothing.
 *   - Size limit: twell_hybrid_workspace_bytes(T, d, f) must not exceed
 *     TWELL_NOALLOC_SCRATCH_BYTES, i.e. roughly T * (2d + 4f) bytes; larger
 *     calls return TWELL_ERR_WORKSPACE and launch nothing.
 *   - The first call on a device looks up the scratch address for that device
 *     (with it current) and keeps it; make that first call before any stream
 *     capture. A lookup that fails is not kept (the call returns
 *     TWELL_ERR_CUDA and the next call tries again). The kept address belongs
 *     to the device's current context: after cudaDeviceReset the library must
 *     not be called again in that process.
 *   - Every call on a device shares the one scratch array, which keeps the last
 *     call's contents (nothing in it needs to start at zero). Calls whose work
 *     overlaps on the GPU -- on different streams, or from several host
 *     threads -- race on it; serialise them.
 */
#define TWELL_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
twell_status twell_ffn_hybrid_forward_noalloc(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                              const uint16_t* Wd, int T, int d, int f, const twell_t* tw,
                                              float* y, int32_t* ovf_rows, int32_t* n_ovf,
                                              int32_t* dev_status, void* stream);

/* Bytes of workspace needed by twell_dense_ffn_forward and
 * twell_relu_dense_ffn_forward: the [T][f] bf16 hidden activations, and for
 * T <= 512 room for the fp32 pre-activations ([T][2f]) of the small-batch path,
 * whose first GEMMs split K over the whole GPU (batches of at most 8 tokens
 * use two CUDA-core GEMVs instead, h in bf16 as in the GEMM path). */
size_t twell_dense_workspace_bytes(int T, int d, int f);

/*
 * Dense ReLU-gated FFN on the tensor cores, no sparsity: one GEMM against
 * [Wg | Wu] with ReLU(z) * u in its epilogue (h stored once as bf16 in
 * workspace, as a standard bf16 layer does), then h Wd. This is the library's
 * own dense baseline for the same layer; its error is that of one bf16
 * rounding of h, |y - y_exact| <= 2^-8 sum_j |h_j Wd[j, :]| plus fp32 sums.
 */
twell_status twell_dense_ffn_forward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                     const uint16_t* Wd, int T, int d, int f, float* y,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream);

/*
 * Non-gated ReLU FFN, y = ReLU(x W1) W2, hybrid forward. The pages note the
 * method also applies to the non-gated layer, with a smaller gain
 * (intellectnews.ru, "Sakana AI и NVIDIA: TwELL ...", section "Ограничения и
 * открытые вопросы").
 *   x [T][d] bf16, W1T [f][d] bf16 (W1 transposed), W2 [f][d] bf16 (row j is
 *   hidden unit j's output vector), y [T][d] fp32: all device pointers,
 *   caller-owned, 16-byte aligned. Shapes and the TwELL buffers as for
 *   twell_ffn_hybrid_forward; workspace of twell_hybrid_workspace_bytes(T, d, f).
 * Steps: the pack of ReLU(x W1) (its stored values are the hidden activations
 * themselves), routing, the per-token down projection of the stored slots for
 * rows that fit (twell_sparse_down), and the dense layer on the tensor cores
 * for overflow rows (hidden values kept as bf16 plus bf16 remainder, as in
 * the gated dense branch). Past the small-batch paths the dense branch does
 * not recompute x W1 over the routed rows: as in
 * twell_ffn_hybrid_forward_tc_up, the pack GEMM writes each overflowing
 * (row, tile)'s exact ReLU(z) into the workspace at the row's compact slot and
 * the row's other tiles take theirs from the pack. Errors as for
 * twell_ffn_hybrid_forward.
 */
twell_status twell_relu_ffn_hybrid_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2,
                                           int T, int d, int f, const twell_t* tw, float* y,
                                           int32_t* ovf_rows, int32_t* n_ovf, void* workspace,
                                           size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * The dense branch of twell_relu_ffn_hybrid_forward on its own: for i <
 * *n_rows, y[rows[i]] = ReLU(x[rows[i]] W1) W2 (rows and n_rows device
 * int32, as twell_route writes them; rows outside [0, T) raise
 * TWELL_ERR_INDEX and are skipped). Workspace and errors as for
 * twell_dense_rows_forward.
 */
twell_status twell_relu_dense_rows_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2,
                                          int T, int d, int f, const int32_t* rows, const int32_t* n_rows,
                                          float* y, void* workspace, size_t workspace_bytes,
                                          int32_t* dev_status, void* stream);

/*
 * Dense non-gated ReLU FFN on the tensor cores (h = ReLU(x W1) stored once as
 * bf16 in a workspace of twell_dense_workspace_bytes(T, d, f), then h W2): the
 * library's own baseline for the non-gated layer; error bound as for
 * twell_dense_ffn_forward.
 */
twell_status twell_relu_dense_ffn_forward(const uint16_t* x, const uint16_t* W1T, const uint16_t* W2,
                                          int T, int d, int f, float* y, void* workspace,
                                          size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Backward pass through the hybrid format (intellectnews.ru, "Sakana AI и
 * NVIDIA: TwELL ...", section "Слитые CUDA-ядра для инференса и гибрид для
 * обучения": in training, rows that are sparse enough use the compact format
 * and rows with many active units a dense branch). For y = (ReLU(x Wg) *
 * (x Wu)) Wd and an upstream gradient dy [T][d] (bf16):
 *   dh_j = dy . Wd[j, :], du_j = dh_j g_j, dz_j = dh_j u_j where z_j > 0
 *   dx [T][d] = dz Wg^T + du Wu^T           (fp32)
 *   dWgT [f][d] = dz^T x, dWuT [f][d] = du^T x, dWd [f][d] = h^T dy   (fp32,
 *   overwritten; the layouts of WgT, WuT and Wd)
 * tw, ovf_rows and n_ovf are the outputs of twell_ffn_hybrid_forward on the
 * same x (the gate form: tw's values are the bf16 gate). dh and u are formed
 * by two tensor-core GEMMs (dy Wd^T and x Wu^T, fp32 sums), whose epilogues
 * keep only the stored slots' entries as each slot's record {h, du, dz}. Rows that fit use
 * their stored slots with the stored bf16 gate g (h = g u), so the result is
 * the method's, within one bf16 rounding per term of the exact gradients;
 * their weight gradients are summed per hidden unit over a column sort of the
 * slots (the order of the terms inside a column is not fixed, so the fp32 sums
 * are not bit-reproducible). Overflow rows take the dense branch on the tensor
 * cores: [z | u] recomputed, dh = dy Wd^T with dz, du, h formed in its
 * epilogue (kept as bf16 plus bf16 remainder), dx = [dz | du] [Wg; Wu]^T, and
 * their share of the weight gradients added by three GEMMs over their tokens.
 * workspace: twell_backward_workspace_bytes(T, d, f, tw->W) bytes (worst case:
 * every row overflows). T == 0 zeroes the weight gradients. Errors as for
 * twell_ffn_hybrid_forward; a stored index outside its own column tile raises
 * TWELL_ERR_INDEX and that slot adds nothing to any gradient. T * (f / 128) *
 * W must stay below 2^31.
 */
size_t twell_backward_workspace_bytes(int T, int d, int f, int W);
twell_status twell_ffn_hybrid_backward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                       const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                       const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf,
                                       float* dx, float* dWgT, float* dWuT, float* dWd, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * The two halves of twell_ffn_hybrid_backward, for callers that want dx early
 * (to go on with the previous layer's backward while the weight gradients are
 * summed, e.g. on another stream ordered after this one). _dx writes dx and
 * leaves per-slot scalars in the workspace; _dw reads them and writes the
 * weight gradients, and must see the same workspace, x, dy, tw and n_ovf,
 * stream-ordered after _dx with nothing in between that writes them.
 */
twell_status twell_ffn_hybrid_backward_dx(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                          const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                          const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf,
                                          float* dx, void* workspace, size_t workspace_bytes,
                                          int32_t* dev_status, void* stream);
twell_status twell_ffn_hybrid_backward_dw(const uint16_t* x, const uint16_t* dy, int T, int d, int f,
                                          const twell_t* tw, const int32_t* n_ovf, float* dWgT, float* dWuT,
                                          float* dWd, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Tensor-core form of twell_ffn_hybrid_backward_dw (same arguments, same
 * workspace, called after twell_ffn_hybrid_backward_dx). At densities where
 * every unit is active for many tokens of a batch, the weight gradients are a
 * dense contraction over the tokens: the records of the rows that fit are
 * written token-major into a dense block [dz | du | h] (each as bf16 value
 * plus bf16 remainder, zeros where no slot is stored) and three tcgen05 GEMMs
 * over all tokens, reading that block with the units along M, form their
 * share; the overflow rows' GEMMs add theirs. The extra error is ~2^-16 of
 * each term; the sums are in fp32, with K (the tokens) split over the GPU
 * where that shortens the GEMMs' last wave, the partial sums added atomically
 * (so not bit-reproducible from run to run).
 */
twell_status twell_ffn_hybrid_backward_dw_tc(const uint16_t* x, const uint16_t* dy, int T, int d, int f,
                                             const twell_t* tw, const int32_t* n_ovf, float* dWgT, float* dWuT,
                                             float* dWd, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Tensor-core form of twell_ffn_hybrid_backward_dx (same arguments, same
 * workspace; twell_ffn_hybrid_backward_dw or _dw_tc may follow it). The
 * records are built as in twell_ffn_hybrid_backward_dx (u and dh for every
 * token by tcgen05 GEMMs), and the rows that fit get their dx from one
 * tcgen05 GEMM instead of the per-token pass: their dz and du are written by
 * token into dense rows
 * [dz | du | dz_lo | du_lo] (bf16 value plus bf16 remainder, zeros elsewhere)
 * and multiplied by [Wg; Wu] read twice along K, the layout the overflow
 * rows' dense branch uses. Pays where the rows hold many stored units (the
 * GEMMs' cost does not fall with density); the extra error is ~2^-16 of each
 * term.
 */
twell_status twell_ffn_hybrid_backward_dx_tc(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                             const uint16_t* Wd, const uint16_t* dy, int T, int d, int f,
                                             const twell_t* tw, const int32_t* ovf_rows, const int32_t* n_ovf,
                                             float* dx, void* workspace, size_t workspace_bytes,
                                             int32_t* dev_status, void* stream);

/*
 * Dense backward of the gated layer on the tensor cores, no sparsity: the
 * library's own baseline for twell_ffn_hybrid_backward. [z | u] = x [Wg | Wu]
 * (fp32), dh = dy Wd^T with dz = dh u [z > 0], du = dh ReLU(z), h = ReLU(z) u
 * formed in that GEMM's epilogue and stored once as bf16 (as a standard bf16
 * layer does), then dx = [dz | du] [Wg; Wu]^T and dWgT = dz^T x, dWuT = du^T x,
 * dWd = h^T dy (fp32, overwritten). Its error is that of one bf16 rounding of
 * dz, du and h: at most 2^-8 of the summed magnitudes of the terms, plus fp32
 * sums. Workspace: twell_dense_backward_workspace_bytes(T, d, f).
 */
size_t twell_dense_backward_workspace_bytes(int T, int d, int f);
twell_status twell_dense_ffn_backward(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                      const uint16_t* Wd, const uint16_t* dy, int T, int d, int f, float* dx,
                                      float* dWgT, float* dWuT, float* dWd, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Dead hidden units (intellectnews.ru, "Sakana AI и NVIDIA: TwELL ...",
 * section "Ограничения и открытые вопросы": under the chosen L1 setting some
 * units die, i.e. are never active). Three calls compact a layer to the units
 * a profile batch activates:
 *
 * twell_column_activity: the gate GEMM z = x Wg on the tensor cores with an
 * epilogue that sets bit j of active_bits ([f / 32] uint32, device) iff
 * z[t, j] > 0 for some row t. accumulate == 0 clears the bitmap first;
 * accumulate != 0 ORs this batch into it (a profile over several batches).
 * T == 0 only clears (or keeps) the bitmap. Shapes as for twell_gate_pack.
 */
twell_status twell_column_activity(const uint16_t* x, const uint16_t* WgT, int T, int d, int f,
                                   uint32_t* active_bits, int accumulate, int32_t* dev_status,
                                   void* stream);

/*
 * twell_compact_columns: col_map[0 .. f_live) = the indices j with bit j of
 * active_bits set, ascending; col_map[f_live .. f) = -1; *f_live (device
 * int32) = their number. col_map is [f] int32 device memory. One block.
 */
twell_status twell_compact_columns(const uint32_t* active_bits, int f, int32_t* col_map, int32_t* f_live,
                                   void* stream);

/*
 * twell_gather_rows: W_out[i, :] = W[col_map[i], :] for i < min(*f_live,
 * f_out) and zero rows for the rest, W [f][d] and W_out [f_out][d] bf16
 * (1 <= f_out <= f). Applied to WgT, WuT and Wd with f_out = f_live rounded
 * up to a multiple of 128 (the caller reads *f_live), it gives the compacted
 * layer: its zero gate rows have z = 0 and are never active, so on the
 * profile batch the layer computes the same y with f_out hidden units. A map
 * entry outside [0, f) raises TWELL_ERR_INDEX and gives a zero row.
 */
twell_status twell_gather_rows(const uint16_t* W, int f, int d, const int32_t* col_map, const int32_t* f_live,
                               int f_out, uint16_t* W_out, int32_t* dev_status, void* stream);

/*
 * TwELL -> dense bf16 g[T][f]: zeros everywhere except the stored slots
 * (slots below min(count, W); overflowing rows unpack only what was stored).
 * The inverse of the packing of intellectnews.ru "Sakana AI и NVIDIA ...
 * TwELL", section "Формат TwELL вместо классической sparse-упаковки" (per row
 * and column tile, the nonzero values with their column indices); for tests
 * and for callers that need the dense hidden activations.
 */
twell_status twell_unpack(const twell_t* tw, uint16_t* g_dense, int32_t* dev_status, void* stream);

/* Zero dev_status (stream-ordered). */
twell_status twell_status_reset(int32_t* dev_status, void* stream);

/* Synchronise `stream` and copy *dev_status to *host_out (blocks the host). */
twell_status twell_status_get(const int32_t* dev_status, void* stream, int32_t* host_out);

/* Static description of a status code. */
const char* twell_status_str(int status);

/* Library version string. */
const char* twell_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TWELL_H */
