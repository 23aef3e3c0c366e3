"""GPU parity of the backward pass through the hybrid format against the CPU
oracle. The forward (gate form) provides the pack and the routing; each
gradient (dx, dWgT, dWuT, dWd) must satisfy max|g - g_ref| <= 2e-2 * rms(g_ref)
against the oracle's result of the method. Rows that fit are summed in fp32
from the same bf16 values the oracle sums in fp64, so a much tighter
1e-3 * rms is also required; the overflow rows' dense branch holds dz, du and
h as bf16 value plus bf16 remainder (relative error <= 2^-16 per term), so
their share may in addition move by 2^-15 * sum |term|."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import upload
from tests.test_gpu_parity import IDS, SMALL

pytestmark = pytest.mark.gpu

GRADS = ("dx", "dWgT", "dWuT", "dWd")

# Batches whose dh and u output tiles fill the GPU, so that the records come
# from the GEMMs' slot epilogues (the small configurations build them from the
# full products): a ragged last M tile, an odd number of column tiles (the
# last 256-column block holds one tile), d of 3 x 64, heavy rows.
LC = synth.LayerConfig
MID = [
    LC("slots_mid", T=2000, d=256, f=4608, tile=128, W=16, density=0.03, sigma=0.5, heavy_frac=0.05,
       heavy_lo=0.2, heavy_hi=0.35),
    LC("slots_odd_tiles", T=2500, d=192, f=3968, tile=128, W=8, density=0.02, sigma=0.5),
]
MID_IDS = [c.name for c in MID]
TIGHT = 1e-3
CONTRACT = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


def make_dy(T: int, d: int, seed: int) -> np.ndarray:
    return synth.make_dy(T, d, seed)


def forward_backward(L, cfg, dy_bits):
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ovf_rows = torch.empty((T,), dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    dy = tl.to_device_bf16(dy_bits)
    g = {k: torch.full((T if k == "dx" else f, d), float("nan"), dtype=torch.float32, device="cuda")
         for k in GRADS}
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf,
                           g["dx"], g["dWgT"], g["dWuT"], g["dWd"], wsb, st)
    assert tl.status_get(st) == 0
    n = int(n_ovf.item())
    return {k: v.double().cpu().numpy() for k, v in g.items()}, ovf_rows[:n].cpu().numpy()


def assert_grad_close(got: np.ndarray, ref: np.ndarray, name: str, pair_bound=None) -> None:
    assert np.isfinite(got).all(), name
    rms = float(np.sqrt(np.mean(ref**2)))
    err = np.abs(got - ref)
    assert err.max() <= CONTRACT * rms, f"{name}: {err.max():.3e} > {CONTRACT} * rms {rms:.3e}"
    tight = TIGHT * rms + (0.0 if pair_bound is None else pair_bound)
    assert np.all(err <= tight), f"{name}: {float((err / tight).max()):.3f} x the tight bound"


def dense_branch_bounds(L, dy_bits, ovf, rows=None, cols=None, k=2.0**-15) -> dict:
    """k * sum |term| of the rows `ovf` (by default 2^-15, the bf16 value and
    remainder pair's error): per sampled row of dx (zero for other rows) and
    per sampled unit of the weight gradients."""
    F = O.bf16_bits_to_f64
    x, dyv = F(L["x"][ovf]), F(dy_bits[ovf])
    WgT, WuT, Wd = F(L["WgT"]), F(L["WuT"]), F(L["Wd"])
    sel = slice(None) if cols is None else cols
    z, u = x @ WgT[sel].T, x @ WuT[sel].T
    g = np.maximum(z, 0)
    dh = dyv @ Wd[sel].T
    dz, du, h = np.abs(np.where(z > 0, dh * u, 0)), np.abs(dh * g), np.abs(g * u)
    out = {"dWgT": k * dz.T @ np.abs(x), "dWuT": k * du.T @ np.abs(x), "dWd": k * h.T @ np.abs(dyv)}
    if rows is not None:
        bx = np.zeros((len(rows), x.shape[1]))
        pos = {int(r): i for i, r in enumerate(ovf)}
        for i, r in enumerate(rows):
            if int(r) in pos:
                q = pos[int(r)]
                bx[i] = k * (dz[q] @ np.abs(WgT) + du[q] @ np.abs(WuT))
        out["dx"] = bx
    return out


@pytest.mark.parametrize("cfg", SMALL + MID, ids=IDS + MID_IDS)
def test_hybrid_backward(cfg):
    L = synth.make_layer(cfg, seed=0)
    dy = make_dy(cfg.T, cfg.d, 0)
    got, ovf = forward_backward(L, cfg, dy)
    ref = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy, cfg.tile, cfg.W)
    assert np.array_equal(ovf, ref["ovf_rows"])
    b = dense_branch_bounds(L, dy, ovf, rows=np.arange(cfg.T)) if ovf.size else {}
    for k in GRADS:
        assert_grad_close(got[k], ref[k], k, b.get(k))


def test_backward_of_an_all_negative_gate_is_zero():
    cfg = SMALL[1]
    L = dict(synth.make_layer(cfg, seed=0))
    neg = O.bf16_bits_to_f64(L["WgT"]).copy()
    neg[:, -1] = -64.0
    L["WgT"] = O.f64_to_bf16_bits(neg)
    got, ovf = forward_backward(L, cfg, make_dy(cfg.T, cfg.d, 1))
    assert ovf.size == 0
    for k in GRADS:
        assert not np.any(got[k]), k


@pytest.mark.parametrize("name", ["0.5b", "2b"])
def test_full_size_hybrid_backward(name):
    """Full layer size: dx on sampled rows and on overflow rows, the weight
    gradients on sampled hidden units (oracle restricted to those units)."""
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    dy = make_dy(cfg.T, cfg.d, 2)
    got, ovf = forward_backward(L, cfg, dy)
    rng = np.random.default_rng(3)
    rows = np.union1d(np.sort(rng.choice(cfg.T, size=128, replace=False)), ovf[:32])
    ref_rows = O.hybrid_ffn_backward(L["x"][rows], L["WgT"], L["WuT"], L["Wd"], dy[rows], cfg.tile, cfg.W)
    ovf_in = np.intersect1d(rows, ovf)  # the sampled rows that took the dense branch
    bx = dense_branch_bounds(L, dy, ovf_in, rows=rows) if ovf_in.size else {}
    assert_grad_close(got["dx"][rows], ref_rows["dx"], "dx", bx.get("dx"))
    cols = np.sort(rng.choice(cfg.f, size=48, replace=False))
    ref_cols = O.hybrid_backward_weight_rows(L["x"], L["WgT"], L["WuT"], L["Wd"], dy, ovf, cols)
    bw = dense_branch_bounds(L, dy, ovf, cols=cols) if ovf.size else {}
    for k in ("dWgT", "dWuT", "dWd"):
        assert_grad_close(got[k][cols], ref_cols[k], k, bw.get(k))


def test_split_backward_matches_the_oracle():
    """dx first, weight gradients afterwards, through the two-call form."""
    cfg = SMALL[4]  # heavy tokens: both passes have work
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 4)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ovf_rows = torch.empty((T,), dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    dy = tl.to_device_bf16(dy_bits)
    dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
    dW = [torch.empty((f, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward_dx(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf, dx, wsb, st)
    tl.ffn_hybrid_backward_dw(dev["x"], dy, tw, n_ovf, dW[0], dW[1], dW[2], wsb)
    assert tl.status_get(st) == 0
    ref = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy_bits, cfg.tile, cfg.W)
    assert int(n_ovf.item()) > 0
    b = dense_branch_bounds(L, dy_bits, ref["ovf_rows"], rows=np.arange(T))
    assert_grad_close(dx.double().cpu().numpy(), ref["dx"], "dx", b["dx"])
    for k, t in zip(("dWgT", "dWuT", "dWd"), dW):
        assert_grad_close(t.double().cpu().numpy(), ref[k], k, b[k])


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_dense_backward_baseline(cfg):
    """The library's dense backward (one bf16 rounding of dz, du, h) against
    the exact gradients: within 2^-7 of the summed term magnitudes (2^-8 for
    the rounding, the rest for fp32 sums)."""
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 5)
    dev = upload(L)
    T, d, f = cfg.T, cfg.d, cfg.f
    dy = tl.to_device_bf16(dy_bits)
    g = {k: torch.full((T if k == "dx" else f, d), float("nan"), dtype=torch.float32, device="cuda")
         for k in GRADS}
    ws = torch.empty(tl.dense_backward_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.dense_ffn_backward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, g["dx"], g["dWgT"], g["dWuT"], g["dWd"],
                          ws, st)
    assert tl.status_get(st) == 0
    ref = O.gated_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy_bits)
    b = dense_branch_bounds(L, dy_bits, np.arange(T), rows=np.arange(T), k=2.0**-7)
    for k in GRADS:
        got = g[k].double().cpu().numpy()
        assert np.isfinite(got).all(), k
        err = np.abs(got - ref[k])
        bound = b[k] + 1e-6 * float(np.sqrt(np.mean(ref[k] ** 2)))
        assert np.all(err <= bound), (k, float((err / bound).max()))


@pytest.mark.parametrize("cfg", SMALL + MID, ids=IDS + MID_IDS)
def test_tensor_core_weight_gradients(cfg):
    """The tensor-core form of the weight gradients (dz, du, h of the rows that
    fit as bf16 value plus remainder, GEMMs over the tokens) against the
    oracle: within the contract and within 2^-15 of the summed term magnitudes
    on top of the tight check."""
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 6)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ovf_rows = torch.empty((T,), dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    dy = tl.to_device_bf16(dy_bits)
    dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
    dW = [torch.full((f, d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward_dx(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf, dx, wsb, st)
    tl.ffn_hybrid_backward_dw(dev["x"], dy, tw, n_ovf, dW[0], dW[1], dW[2], wsb, tensor_cores=True)
    assert tl.status_get(st) == 0
    ref = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy_bits, cfg.tile, cfg.W)
    b = dense_branch_bounds(L, dy_bits, np.arange(T))
    for k, t in zip(("dWgT", "dWuT", "dWd"), dW):
        got = t.double().cpu().numpy()
        assert np.isfinite(got).all(), k
        rms = float(np.sqrt(np.mean(ref[k] ** 2)))
        err = np.abs(got - ref[k])
        assert err.max() <= CONTRACT * rms, (k, float(err.max()), rms)
        assert np.all(err <= b[k] + TIGHT * rms), k


def _forward_for_backward(L, cfg):
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ovf_rows = torch.empty((T,), dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    return dev, tw, ovf_rows, n_ovf, st


@pytest.mark.parametrize("cfg", SMALL + MID, ids=IDS + MID_IDS)
def test_tensor_core_dx(cfg):
    """The tensor-core form of dx (dz, du of the rows that fit as bf16 value
    plus remainder, one GEMM against [Wg; Wu]) against the oracle: within the
    contract and within 2^-15 of the summed term magnitudes on top of the
    tight check; the weight gradients that follow it are unchanged."""
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 7)
    dev, tw, ovf_rows, n_ovf, st = _forward_for_backward(L, cfg)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    dy = tl.to_device_bf16(dy_bits)
    dx = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    dW = [torch.full((f, d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward_dx(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf, dx, wsb, st,
                              tensor_cores=True)
    tl.ffn_hybrid_backward_dw(dev["x"], dy, tw, n_ovf, dW[0], dW[1], dW[2], wsb)
    assert tl.status_get(st) == 0
    ref = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy_bits, cfg.tile, cfg.W)
    n = int(n_ovf.item())
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), ref["ovf_rows"])
    b = dense_branch_bounds(L, dy_bits, np.arange(T), rows=np.arange(T))
    assert_grad_close(dx.double().cpu().numpy(), ref["dx"], "dx", b["dx"])
    ovf = ref["ovf_rows"]
    bw = dense_branch_bounds(L, dy_bits, ovf) if ovf.size else {}
    for k, t in zip(("dWgT", "dWuT", "dWd"), dW):
        assert_grad_close(t.double().cpu().numpy(), ref[k], k, bw.get(k))


def test_full_size_tensor_core_dx():
    """The tensor-core form of dx at the 0.5B size: sampled rows, overflow rows among them."""
    cfg = synth.CONFIGS["0.5b"]
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 8)
    dev, tw, ovf_rows, n_ovf, st = _forward_for_backward(L, cfg)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    dy = tl.to_device_bf16(dy_bits)
    dx = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward_dx(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf, dx, wsb, st,
                              tensor_cores=True)
    assert tl.status_get(st) == 0
    got = dx.double().cpu().numpy()
    assert np.isfinite(got).all()
    ovf = ovf_rows[:int(n_ovf.item())].cpu().numpy()
    rng = np.random.default_rng(9)
    rows = np.union1d(np.sort(rng.choice(T, size=128, replace=False)), ovf[:32])
    ref = O.hybrid_ffn_backward(L["x"][rows], L["WgT"], L["WuT"], L["Wd"], dy_bits[rows], cfg.tile, cfg.W)
    b = dense_branch_bounds(L, dy_bits, rows, rows=rows)
    assert_grad_close(got[rows], ref["dx"], "dx", b["dx"])


@pytest.mark.parametrize("cfg", [SMALL[0], MID[0]], ids=["full_products", "slot_epilogues"])
def test_a_stored_index_outside_its_tile_is_reported_and_adds_nothing(cfg):
    """One stored slot of a row that fits is moved to a column of another tile
    (still inside [0, f)): the backward raises TWELL_ERR_INDEX, every gradient
    stays finite, and the rows and units that slot does not touch keep the
    oracle's values."""
    L = synth.make_layer(cfg, seed=0)
    dy_bits = make_dy(cfg.T, cfg.d, 11)
    dev, tw, ovf_rows, n_ovf, st = _forward_for_backward(L, cfg)
    assert tl.status_get(st) == 0
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    counts = tw.counts.cpu().numpy()
    row_ovf = tw.row_ovf.cpu().numpy()
    cand = [(t, c) for t in range(T) if not row_ovf[t] for c in range(f // 128) if counts[t, c] > 0]
    t, c = cand[len(cand) // 2]
    idx = tw.idx.view(T, f // 128, W)
    j_old = int(idx[t, c, 0].item())
    idx[t, c, 0] = (j_old + 128) % f  # the same unit of the next tile
    dy = tl.to_device_bf16(dy_bits)
    dx = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    dW = [torch.full((f, d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows, n_ovf,
                           dx, dW[0], dW[1], dW[2], wsb, st)
    assert tl.status_get(st) == tl.TWELL_ERR_INDEX
    got = {"dx": dx.double().cpu().numpy(), **{k: v.double().cpu().numpy() for k, v in zip(GRADS[1:], dW)}}
    for k in GRADS:
        assert np.isfinite(got[k]).all(), k
    ref = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy_bits, cfg.tile, cfg.W)
    keep_rows = np.setdiff1d(np.arange(T), [t])
    keep_units = np.setdiff1d(np.arange(f), [j_old, (j_old + 128) % f])
    ovf = ref["ovf_rows"]
    b = dense_branch_bounds(L, dy_bits, ovf, rows=keep_rows) if ovf.size else {}
    assert_grad_close(got["dx"][keep_rows], ref["dx"][keep_rows], "dx", b.get("dx"))
    bw = dense_branch_bounds(L, dy_bits, ovf, cols=keep_units) if ovf.size else {}
    for k in GRADS[1:]:
        assert_grad_close(got[k][keep_units], ref[k][keep_units], k, bw.get(k))
