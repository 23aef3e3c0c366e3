"""CPU oracle for the TwELL sparse ReLU-gated FFN forward pass.

TEST INFRASTRUCTURE ONLY. Nothing in the library imports this module; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
it. It shares no code with the CUDA path: every step here is written out from
the definitions on the pages, in float64, with numpy's matmul as the only
library primitive.

Sources (three news pages about one release; cited by page and section):

* [P1] intellectnews.ru, "Sakana AI и NVIDIA: TwELL ..." -- sections
  "Формат TwELL вместо классической sparse-упаковки" (the format),
  "Слитые CUDA-ядра для инференса и гибрид для обучения" (fused inference
  kernel; hybrid sparse/dense routing), "Минимальные изменения в рецепте
  обучения" (ReLU in the gate gives exact zeros).
* [P2] gate.com post 20977915 -- paragraph on the TwELL format (tiles packed
  locally by each compute unit).

Readings taken where the pages are silent:

* a hidden unit is active iff its gate pre-activation is strictly positive;
* TwELL keeps, per row and per 128-column tile, the true nonzero count and the
  first W (global column index, bf16 value) pairs in ascending column order;
  slots past min(count, W) are padding (idx -1, value 0 here; unspecified on
  the device);
* the stored value is the ReLU output rounded once to bf16, nearest-even;
* a row overflows iff any of its tiles holds more than W nonzeros, and the
  overflow rows, in ascending order, go to the dense branch;
* the dense branch recomputes the gate for its rows.

Every function here is pinned by ``tests/test_oracle.py`` (closed forms,
exact rational brute force, finite differences, library rounding, hand-derived
fixtures in ``tests/golden``, invariants). The pages print no numeric worked
example, so no pin uses values printed on the pages.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
    "gate_preactivation",
    "gated_ffn",
    "twell_pack",
    "route_rows",
    "twell_unpack",
    "sparse_ffn_from_twell",
    "hybrid_ffn",
    "twell_pack_hidden",
    "sparse_down_from_twell",
    "hybrid_ffn_up_dense",
    "relu_ffn",
    "hybrid_relu_ffn",
    "column_activity",
    "compact_layer",
    "gated_ffn_backward",
    "hybrid_ffn_backward",
    "hybrid_backward_weight_rows",
]


# ---------------------------------------------------------------------------
# bf16 <-> float64


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (a bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16, nearest with ties to even, in one step.

    bf16 keeps 8 significant bits with fp32's exponent range; below 2^-126
    its quantum is fixed at 2^-133. The rounding is done on |x| scaled by the
    quantum of its binade (an exact power-of-two scaling), so no intermediate
    fp32 rounding takes place. Finite inputs only.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)  # a = m * 2^e with m in [0.5, 1)
    q_exp = np.maximum(e.astype(np.int64) - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(a, -q_exp)), q_exp)
    r = np.where(a == 0, 0.0, r)
    bits = (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    sign = np.where(np.signbit(x), np.uint16(0x8000), np.uint16(0))
    return (bits | sign).astype(np.uint16)


# ---------------------------------------------------------------------------
# The layer: y = (ReLU(x Wg) * (x Wu)) Wd   [P1, "Минимальные изменения ..."]


def gate_preactivation(x_bits: np.ndarray, WgT_bits: np.ndarray) -> np.ndarray:
    """z = x . Wg in float64. x is [T, d]; WgT is Wg transposed, [f, d]."""
    return bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(WgT_bits).T


def gated_ffn(x_bits, WgT_bits, WuT_bits, Wd_bits) -> np.ndarray:
    """Dense ReLU-gated FFN in float64: the exact result the sparse path must
    reach, since skipping exact zeros changes nothing mathematically
    [P1, opening paragraphs and "Минимальные изменения ..."].

    x [T,d], WgT [f,d], WuT [f,d], Wd [f,d] as bf16 bits -> y [T,d] float64.
    """
    x = bf16_bits_to_f64(x_bits)
    z = x @ bf16_bits_to_f64(WgT_bits).T
    g = np.maximum(z, 0.0)
    u = x @ bf16_bits_to_f64(WuT_bits).T
    return (g * u) @ bf16_bits_to_f64(Wd_bits)


# ---------------------------------------------------------------------------
# TwELL   [P1, "Формат TwELL ..."; P2, paragraph on TwELL]


def twell_pack(z: np.ndarray, tile: int, W: int) -> dict:
    """Pack ReLU(z) into Tile-wise ELLPACK.

    The columns are cut into tiles of ``tile``; for every (row t, tile c) the
    format holds the number of strictly positive entries (not capped) and
    the first W of them in ascending column order as (global column index,
    bf16 of the value). Padding slots hold idx -1 and value 0.

    Returns counts int16 [T,nT], idx int16 [T,nT,W], vals uint16 [T,nT,W],
    row_ovf uint8 [T] (1 iff some tile of the row has count > W).
    """
    T, f = z.shape
    if f % tile:
        raise ValueError("f must be a multiple of the tile width")
    nT = f // tile
    zt = z.reshape(T, nT, tile)
    active = zt > 0
    counts = active.sum(axis=2)
    rank = np.cumsum(active, axis=2) - 1  # position among the tile's nonzeros
    keep = active & (rank < W)
    t, c, k = np.nonzero(keep)
    s = rank[t, c, k]
    idx = np.full((T, nT, W), -1, dtype=np.int16)
    vals = np.zeros((T, nT, W), dtype=np.uint16)
    idx[t, c, s] = (c * tile + k).astype(np.int16)
    vals[t, c, s] = f64_to_bf16_bits(zt[t, c, k])
    row_ovf = (counts > W).any(axis=1).astype(np.uint8)
    return {"counts": counts.astype(np.int16), "idx": idx, "vals": vals, "row_ovf": row_ovf,
            "tile": tile, "W": W, "f": f}


def route_rows(counts: np.ndarray, W: int) -> np.ndarray:
    """Rows sent to the dense branch: those with a tile holding more nonzeros
    than the ELL width can store [P1, "Слитые CUDA-ядра ... гибрид ..."],
    in ascending row order. Returns int32 [n_ovf]."""
    flagged = (np.asarray(counts) > W).any(axis=1)
    return np.nonzero(flagged)[0].astype(np.int32)


def twell_unpack(counts: np.ndarray, idx: np.ndarray, vals: np.ndarray, f: int) -> np.ndarray:
    """Scatter the stored slots back into a dense bf16 [T, f] matrix (zeros
    elsewhere). Only slots below min(count, W) are read."""
    T, nT, W = idx.shape
    g = np.zeros((T, f), dtype=np.uint16)
    n = np.minimum(np.asarray(counts, dtype=np.int64), W)
    live = np.arange(W)[None, None, :] < n[:, :, None]
    t, c, s = np.nonzero(live)
    g[t, idx[t, c, s].astype(np.int64)] = vals[t, c, s]
    return g


def sparse_ffn_from_twell(tw: dict, x_bits, WuT_bits, Wd_bits, rows=None) -> np.ndarray:
    """The fused sparse inference step, one token at a time, in float64
    [P1, "Слитые CUDA-ядра ..."]: for each stored slot (j, g) of row t,
    u_j = x_t . Wu[:, j], h_j = g * u_j, and y_t accumulates h_j * Wd[j, :].
    g is the stored bf16 value. Returns y for ``rows`` (default: all rows).
    """
    counts, idx, vals = tw["counts"], tw["idx"], tw["vals"]
    T, nT, W = idx.shape
    rows = np.arange(T) if rows is None else np.asarray(rows)
    x = bf16_bits_to_f64(np.asarray(x_bits)[rows])
    WuT = bf16_bits_to_f64(WuT_bits)
    Wd = bf16_bits_to_f64(Wd_bits)
    d = Wd.shape[1]
    y = np.zeros((len(rows), d))
    for r, t in enumerate(rows):
        n = np.minimum(counts[t].astype(np.int64), W)
        js = np.concatenate([idx[t, c, : n[c]] for c in range(nT)]).astype(np.int64)
        if js.size == 0:
            continue
        gs = bf16_bits_to_f64(np.concatenate([vals[t, c, : n[c]] for c in range(nT)]))
        u = WuT[js] @ x[r]
        y[r] = (gs * u) @ Wd[js]
    return y


def hybrid_ffn(x_bits, WgT_bits, WuT_bits, Wd_bits, tile: int, W: int) -> dict:
    """The whole hybrid forward: gate, pack, route; stored slots for rows that
    fit, the dense layer (gate recomputed) for the rows that overflow."""
    z = gate_preactivation(x_bits, WgT_bits)
    tw = twell_pack(z, tile, W)
    ovf = route_rows(tw["counts"], W)
    T = z.shape[0]
    keep = np.setdiff1d(np.arange(T), ovf)
    y = np.zeros((T, np.asarray(Wd_bits).shape[1]))
    if keep.size:
        y[keep] = sparse_ffn_from_twell(tw, x_bits, WuT_bits, Wd_bits, rows=keep)
    if ovf.size:
        y[ovf] = gated_ffn(np.asarray(x_bits)[ovf], WgT_bits, WuT_bits, Wd_bits)
    return {"y": y, "twell": tw, "ovf_rows": ovf, "z": z}


# ---------------------------------------------------------------------------
# Variant with the up projection on the tensor cores: the gate GEMM also forms
# u = x . Wu, and the packed values are the hidden activations h = ReLU(z) * u
# at the same positions; the sparse step is then the down projection alone.
# The positions, counts and routing are those of twell_pack(z).


def twell_pack_hidden(z: np.ndarray, u: np.ndarray, tile: int, W: int) -> dict:
    """TwELL of the pattern of ReLU(z) holding bf16(ReLU(z) * u) as values."""
    tw = twell_pack(z, tile, W)
    T, nT, _ = tw["idx"].shape
    n = np.minimum(tw["counts"].astype(np.int64), W)
    live = np.arange(W)[None, None, :] < n[:, :, None]
    t, c, s = np.nonzero(live)
    j = tw["idx"][t, c, s].astype(np.int64)
    tw["vals"][t, c, s] = f64_to_bf16_bits(np.maximum(z[t, j], 0.0) * u[t, j])
    return tw


def sparse_down_from_twell(tw: dict, Wd_bits, rows=None) -> np.ndarray:
    """y_t = sum over stored slots (j, h) of h * Wd[j, :], in float64."""
    counts, idx, vals = tw["counts"], tw["idx"], tw["vals"]
    T, nT, W = idx.shape
    rows = np.arange(T) if rows is None else np.asarray(rows)
    Wd = bf16_bits_to_f64(Wd_bits)
    y = np.zeros((len(rows), Wd.shape[1]))
    for r, t in enumerate(rows):
        n = np.minimum(counts[t].astype(np.int64), W)
        js = np.concatenate([idx[t, c, : n[c]] for c in range(nT)]).astype(np.int64)
        if js.size:
            hs = bf16_bits_to_f64(np.concatenate([vals[t, c, : n[c]] for c in range(nT)]))
            y[r] = hs @ Wd[js]
    return y


def hybrid_ffn_up_dense(x_bits, WgT_bits, WuT_bits, Wd_bits, tile: int, W: int) -> dict:
    """Hybrid forward of the tensor-core-up variant: rows that fit use the
    stored bf16 hidden values, overflow rows the dense layer."""
    x = bf16_bits_to_f64(x_bits)
    z = x @ bf16_bits_to_f64(WgT_bits).T
    u = x @ bf16_bits_to_f64(WuT_bits).T
    tw = twell_pack_hidden(z, u, tile, W)
    ovf = route_rows(tw["counts"], W)
    T = z.shape[0]
    keep = np.setdiff1d(np.arange(T), ovf)
    y = np.zeros((T, np.asarray(Wd_bits).shape[1]))
    if keep.size:
        y[keep] = sparse_down_from_twell(tw, Wd_bits, rows=keep)
    if ovf.size:
        y[ovf] = gated_ffn(np.asarray(x_bits)[ovf], WgT_bits, WuT_bits, Wd_bits)
    return {"y": y, "twell": tw, "ovf_rows": ovf}


# ---------------------------------------------------------------------------
# Non-gated variant y = ReLU(x . W1) . W2 [P1, "Ограничения и открытые
# вопросы": the method also applies to the non-gated FFN, with a smaller
# gain]. The pack is twell_pack of z = x . W1 and the stored values are the
# hidden activations themselves, so the sparse step is the down projection
# alone (sparse_down_from_twell); overflow rows take the dense layer.


def relu_ffn(x_bits, W1T_bits, W2_bits) -> np.ndarray:
    """Dense non-gated ReLU FFN in float64. W1T is W1 transposed ([f, d]);
    W2 is [f, d] (row j is hidden unit j's output vector)."""
    x = bf16_bits_to_f64(x_bits)
    h = np.maximum(x @ bf16_bits_to_f64(W1T_bits).T, 0.0)
    return h @ bf16_bits_to_f64(W2_bits)


def hybrid_relu_ffn(x_bits, W1T_bits, W2_bits, tile: int, W: int) -> dict:
    """Hybrid forward of the non-gated layer: rows whose tiles fit use the
    stored bf16 ReLU outputs, overflow rows the dense layer."""
    z = gate_preactivation(x_bits, W1T_bits)
    tw = twell_pack(z, tile, W)
    ovf = route_rows(tw["counts"], W)
    T = z.shape[0]
    keep = np.setdiff1d(np.arange(T), ovf)
    y = np.zeros((T, np.asarray(W2_bits).shape[1]))
    if keep.size:
        y[keep] = sparse_down_from_twell(tw, W2_bits, rows=keep)
    if ovf.size:
        y[ovf] = relu_ffn(np.asarray(x_bits)[ovf], W1T_bits, W2_bits)
    return {"y": y, "twell": tw, "ovf_rows": ovf}


# ---------------------------------------------------------------------------
# Dead-column compaction [P1, "Ограничения и открытые вопросы": under the
# chosen L1 setting some hidden units die, i.e. are never active]. A profile
# marks the hidden units that are active for at least one token; the others
# are dropped from Wg, Wu and Wd. The kept units keep their order, and the
# compacted width is padded up to a whole number of tiles with all-zero rows,
# whose gate pre-activation is exactly 0 and so never active.


def column_activity(z: np.ndarray) -> np.ndarray:
    """active[j] = True iff z[t, j] > 0 for some row t (strictly positive)."""
    return np.any(np.asarray(z) > 0, axis=0)


def compact_layer(WgT_bits, WuT_bits, Wd_bits, active: np.ndarray, tile: int) -> dict:
    """Keep the rows j of WgT, WuT and Wd with active[j], in ascending j.
    Returns the compacted matrices ([f_c, d], f_c = the kept count rounded up
    to a multiple of tile, at least one tile; padding rows are zero), col_map
    (original index of each compacted row, -1 for padding) and f_live."""
    live = np.nonzero(np.asarray(active))[0]
    f_live = int(live.size)
    f_c = max(tile, -(-f_live // tile) * tile)
    out = {"f_live": f_live, "f_c": f_c}
    col_map = np.full(f_c, -1, dtype=np.int32)
    col_map[:f_live] = live
    out["col_map"] = col_map
    for name, m in (("WgT", WgT_bits), ("WuT", WuT_bits), ("Wd", Wd_bits)):
        if m is None:
            continue
        m = np.asarray(m)
        c = np.zeros((f_c, m.shape[1]), dtype=m.dtype)
        c[:f_live] = m[live]
        out[name] = c
    return out


# ---------------------------------------------------------------------------
# Backward pass through the hybrid format [P1, "Слитые CUDA-ядра для инференса
# и гибрид для обучения": in training, rows that are sparse enough use the
# compact sparse format, rows with many active units take a dense branch].
# The gradients of y = (ReLU(x Wg) * (x Wu)) Wd for an upstream gradient dy:
#   dh = dy Wd^T, du = dh * g, dz = dh * u * [z > 0] (g = ReLU(z), h = g * u),
#   dWd = h^T dy, dWu^T = du^T x, dWg^T = dz^T x, dx = dz Wg^T + du Wu^T.
# Every term vanishes where z <= 0, so the sparse rows need only their stored
# units. The ReLU derivative at z == 0 is 0 (active iff z > 0).


def gated_ffn_backward(x_bits, WgT_bits, WuT_bits, Wd_bits, dy_bits) -> dict:
    """Dense gradients in float64: dx [T, d], dWgT, dWuT, dWd [f, d]."""
    x = bf16_bits_to_f64(x_bits)
    WgT = bf16_bits_to_f64(WgT_bits)
    WuT = bf16_bits_to_f64(WuT_bits)
    Wd = bf16_bits_to_f64(Wd_bits)
    dy = bf16_bits_to_f64(dy_bits)
    z = x @ WgT.T
    u = x @ WuT.T
    act = z > 0
    g = np.where(act, z, 0.0)
    dh = dy @ Wd.T
    du = dh * g
    dz = np.where(act, dh * u, 0.0)
    return {"dx": dz @ WgT + du @ WuT, "dWgT": dz.T @ x, "dWuT": du.T @ x, "dWd": (g * u).T @ dy}


def hybrid_ffn_backward(x_bits, WgT_bits, WuT_bits, Wd_bits, dy_bits, tile: int, W: int) -> dict:
    """The method's backward: the gate pack and routing of the forward; for a
    row that fits, each stored slot (j, g) with g the stored bf16 value gives
    u_j = x_t . Wu[:, j], dh_j = dy_t . Wd[j, :], h_j = g u_j, du_j = dh_j g,
    dz_j = dh_j u_j; overflow rows take the dense gradients. dx is per row;
    the weight gradients sum both kinds of rows."""
    x = bf16_bits_to_f64(x_bits)
    WgT = bf16_bits_to_f64(WgT_bits)
    WuT = bf16_bits_to_f64(WuT_bits)
    Wd = bf16_bits_to_f64(Wd_bits)
    dy = bf16_bits_to_f64(dy_bits)
    z = x @ WgT.T
    tw = twell_pack(z, tile, W)
    ovf = route_rows(tw["counts"], W)
    T, d = x.shape
    f = WgT.shape[0]
    out = {"dx": np.zeros((T, d)), "dWgT": np.zeros((f, d)), "dWuT": np.zeros((f, d)), "dWd": np.zeros((f, d)),
           "twell": tw, "ovf_rows": ovf}
    counts, idx, vals = tw["counts"], tw["idx"], tw["vals"]
    nT = idx.shape[1]
    is_ovf = np.zeros(T, dtype=bool)
    is_ovf[ovf] = True
    for t in np.nonzero(~is_ovf)[0]:
        n = np.minimum(counts[t].astype(np.int64), W)
        js = np.concatenate([idx[t, c, : n[c]] for c in range(nT)]).astype(np.int64)
        if js.size == 0:
            continue
        g = bf16_bits_to_f64(np.concatenate([vals[t, c, : n[c]] for c in range(nT)]))
        u = WuT[js] @ x[t]
        dh = Wd[js] @ dy[t]
        du, dz = dh * g, dh * u
        out["dx"][t] = dz @ WgT[js] + du @ WuT[js]
        out["dWgT"][js] += dz[:, None] * x[t][None, :]
        out["dWuT"][js] += du[:, None] * x[t][None, :]
        out["dWd"][js] += (g * u)[:, None] * dy[t][None, :]
    if ovf.size:
        dense = gated_ffn_backward(np.asarray(x_bits)[ovf], WgT_bits, WuT_bits, Wd_bits, np.asarray(dy_bits)[ovf])
        out["dx"][ovf] = dense["dx"]
        for k in ("dWgT", "dWuT", "dWd"):
            out[k] += dense[k]
    return out


def hybrid_backward_weight_rows(x_bits, WgT_bits, WuT_bits, Wd_bits, dy_bits, ovf_rows, cols) -> dict:
    """Rows `cols` of the hybrid backward's weight gradients, given the routing
    (ovf_rows) of the whole batch: a row that fits stores every active unit,
    with the bf16 gate, and an overflow row uses the exact gate. Needs only the
    gate, up and down columns `cols`, so it scales to full-size batches."""
    cols = np.asarray(cols)
    x = bf16_bits_to_f64(x_bits)
    dy = bf16_bits_to_f64(dy_bits)
    z = x @ bf16_bits_to_f64(np.asarray(WgT_bits)[cols]).T
    u = x @ bf16_bits_to_f64(np.asarray(WuT_bits)[cols]).T
    dh = dy @ bf16_bits_to_f64(np.asarray(Wd_bits)[cols]).T
    act = z > 0
    g = np.where(act, bf16_bits_to_f64(f64_to_bf16_bits(np.where(act, z, 0.0))), 0.0)
    ovf = np.asarray(ovf_rows, dtype=np.int64)
    g[ovf] = np.where(act[ovf], z[ovf], 0.0)
    du = dh * g
    dz = np.where(act, dh * u, 0.0)
    return {"dWgT": dz.T @ x, "dWuT": du.T @ x, "dWd": (g * u).T @ dy}
