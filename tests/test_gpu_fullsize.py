"""Parity at the full layer sizes, in the launch configuration bench.py times
(the whole hybrid forward). Counts, overflow flags and routing are compared
bit-exactly over every row (the fp64 oracle gate is computed in row chunks);
the stored slots and y are compared on sampled rows, overflow rows included."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import assert_twell_equal, assert_within_stored_value_bound, assert_y_close, upload, y_to_f64

pytestmark = pytest.mark.gpu

CHUNK = 2048


@pytest.mark.parametrize("name", ["0.5b", "1.5b", "2b"])
def test_full_size_hybrid_forward(name):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    counts = tw.counts.cpu().numpy()
    row_ovf = tw.row_ovf.cpu().numpy()
    idx = tw.idx.cpu().numpy()
    vals = tl.bf16_bits(tw.vals)
    yg = y.double().cpu().numpy()
    assert np.isfinite(yg).all()

    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(T, size=256, replace=False))
    all_counts = np.empty_like(counts)
    for r0 in range(0, T, CHUNK):
        rows = np.arange(r0, min(T, r0 + CHUNK))
        ref = O.twell_pack(O.gate_preactivation(L["x"][rows], L["WgT"]), cfg.tile, W)
        all_counts[rows] = ref["counts"]
        assert np.array_equal(counts[rows], ref["counts"]), f"counts differ in rows {r0}.."
        assert np.array_equal(row_ovf[rows], ref["row_ovf"])
        sel = sample[(sample >= rows[0]) & (sample <= rows[-1])]
        if sel.size:
            got = {"counts": counts[sel], "row_ovf": row_ovf[sel], "idx": idx[sel], "vals": vals[sel]}
            want = {k: ref[k][sel - r0] for k in ("counts", "row_ovf", "idx", "vals")}
            assert_twell_equal(got, want, W)
    ovf_ref = O.route_rows(all_counts, W)
    n = int(n_ovf.item())
    assert n == len(ovf_ref)
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), ovf_ref)
    if name == "2b":
        heavy = np.nonzero(L["p_t"] >= cfg.heavy_lo)[0]
        assert set(heavy.tolist()) <= set(ovf_ref.tolist())

    # y: the oracle's result of the method on sampled rows (stored bf16 gate
    # values for rows that fit, the exact dense layer for overflow rows)
    keep = sample[row_ovf[sample] == 0]
    ovf = ovf_ref[:64]
    ref = O.twell_pack(O.gate_preactivation(L["x"][keep], L["WgT"]), cfg.tile, W)
    y_keep = O.sparse_ffn_from_twell(ref, L["x"][keep], L["WuT"], L["Wd"])
    rows = np.concatenate([keep, ovf])
    y_ref = np.concatenate([y_keep, O.gated_ffn(L["x"][ovf], L["WgT"], L["WuT"], L["Wd"])])
    assert_y_close(yg[rows], y_ref)
    assert_within_stored_value_bound(yg[keep], L, keep)


@pytest.mark.parametrize("name", ["0.5b", "1.5b", "2b"])
def test_full_size_tensor_core_up_hybrid_forward(name):
    """The tensor-core-up hybrid forward at the full layer sizes, as bench.py
    times it: routing over every row, y on sampled rows that fit and on
    overflow rows."""
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward_tc_up(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    row_ovf = tw.row_ovf.cpu().numpy()
    n = int(n_ovf.item())
    ovf = ovf_rows[:n].cpu().numpy()
    assert np.array_equal(ovf, np.nonzero(row_ovf)[0])
    rng = np.random.default_rng(3)
    sample = np.sort(rng.choice(T, size=256, replace=False))
    keep = sample[row_ovf[sample] == 0]
    x = O.bf16_bits_to_f64(L["x"][keep])
    want = O.twell_pack_hidden(x @ O.bf16_bits_to_f64(L["WgT"]).T, x @ O.bf16_bits_to_f64(L["WuT"]).T,
                               cfg.tile, W)
    assert np.array_equal(want["row_ovf"], np.zeros(len(keep), np.uint8))
    y_keep = O.sparse_down_from_twell(want, L["Wd"])
    rows = np.concatenate([keep, ovf[:64]])
    y_ref = np.concatenate([y_keep, O.gated_ffn(L["x"][ovf[:64]], L["WgT"], L["WuT"], L["Wd"])])
    assert_y_close(yg[rows], y_ref)


UNION_CASES = [
    # output tiles >= the SM count (the size the union form is built for)
    synth.LayerConfig("union_mid", T=2400, d=2048, f=1024, tile=128, W=16, density=0.05, sigma=0.5,
                      dead_frac=0.03),
    # ragged T, d = 9 x 256, heavy tokens that overflow
    synth.LayerConfig("union_heavy", T=2219, d=2304, f=2304, tile=128, W=24, density=0.012, sigma=0.5,
                      heavy_frac=0.08, heavy_lo=0.25, heavy_hi=0.40),
]


def _union_against_per_token(dev, tw, T, d, f, keep):
    """The union down projection and the per-token kernel on the same pack:
    the same exact products summed in another order, so the rows that fit
    agree to fp32 summation error."""
    st = tl.new_status()
    yu = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    wsu = torch.empty(tl.sparse_down_union_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    tl.sparse_down_union(dev["Wd"], tw, yu, True, wsu, st)
    assert tl.status_get(st) == 0
    y2 = torch.zeros((T, d), dtype=torch.float32, device="cuda")
    tl.sparse_down(dev["Wd"], tw, y2, True, st)
    assert tl.status_get(st) == 0
    a, b = y_to_f64(yu)[keep], y_to_f64(y2)[keep]
    assert np.isfinite(a).all()
    rms = float(np.sqrt(np.mean(b**2)))
    assert float(np.abs(a - b).max()) <= 1e-5 * rms
    return a


@pytest.mark.parametrize("cfg", UNION_CASES, ids=[c.name for c in UNION_CASES])
def test_union_down_projection_every_row(cfg):
    """The tensor-core-up hybrid forward on every row against the oracle's
    result of the method, then the down projection over the tiles' unions of
    stored units on its pack: within the stored-value bound of the oracle and
    within fp32 summation error of the per-token kernel."""
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward_tc_up(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_ffn_up_dense(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, W)
    n = int(n_ovf.item())
    assert n == len(out["ovf_rows"])
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), out["ovf_rows"])
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    keep = np.setdiff1d(np.arange(T), out["ovf_rows"])
    yu = _union_against_per_token(dev, tw, T, d, f, keep)
    assert_within_stored_value_bound(yu, L, keep, stored="h")
    assert_y_close(yu, out["y"][keep])


def test_union_relu_hybrid_forward():
    """The non-gated hybrid forward, then the union down projection on its
    pack (which holds ReLU(x W1) itself)."""
    cfg = UNION_CASES[1]
    L = synth.make_layer(cfg, seed=1)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W)
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.relu_ffn_hybrid_forward(dev["x"], dev["WgT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_relu_ffn(L["x"], L["WgT"], L["Wd"], cfg.tile, W)
    n = int(n_ovf.item())
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), out["ovf_rows"])
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    keep = np.setdiff1d(np.arange(T), out["ovf_rows"])
    yu = _union_against_per_token(dev, tw, T, d, f, keep)
    assert_y_close(yu, out["y"][keep])
