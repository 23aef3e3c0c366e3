"""GPU parity of the hybrid forwards' dense branch where it takes the routed
rows' hidden activations from the pack GEMM (the overflowing tiles, exact,
written at the row's compact slot by the epilogue) and from the pack (the
tiles that fit, bf16 h) instead of a second GEMM over those rows: the
tensor-core-up form of the gated layer (h = ReLU(z) u from its gate+up GEMM)
and the non-gated layer's large-batch forward (h = ReLU(z) from its pack GEMM).

For every routed row: y within the bound of one bf16 rounding of the stored
units' h against the exact dense layer (|dy| <= 2^-8 sum_j |h_j W[j, :]| over
the units of the tiles that fit, plus the fp32 sums' share), and close to the
dense-rows entry point, which recomputes h exactly. The rows that fit are the
down projection of the pack, as before. Shapes: heavy tokens at several
batch sizes (one and several M tiles, a ragged last tile, d = 9 x 256; for
the non-gated layer batches past the small-batch gate path, and f an odd
number of tiles, so that the last 256-column block holds one tile)."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import assert_y_close, upload, y_to_f64

pytestmark = pytest.mark.gpu

LC = synth.LayerConfig
CASES = [
    LC("branch_one_tile", T=100, d=256, f=1024, tile=128, W=16, density=0.02, heavy_frac=0.1, heavy_lo=0.25,
       heavy_hi=0.40),
    LC("branch_ragged", T=1000, d=256, f=2304, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.08,
       heavy_lo=0.25, heavy_hi=0.40),
    LC("branch_2b_width", T=700, d=2304, f=2304, tile=128, W=24, density=0.012, heavy_frac=0.15, heavy_lo=0.17,
       heavy_hi=0.30),
]
RELU_CASES = [
    LC("relu_branch", T=2048, d=256, f=2304, tile=128, W=24, density=0.012, heavy_frac=0.08, heavy_lo=0.25,
       heavy_hi=0.40),
    LC("relu_branch_odd_tiles", T=1500, d=320, f=3840, tile=128, W=16, density=0.01, sigma=0.5, heavy_frac=0.06,
       heavy_lo=0.2, heavy_hi=0.35),
    LC("relu_branch_2b_width", T=1100, d=2304, f=4608, tile=128, W=24, density=0.012, heavy_frac=0.15,
       heavy_lo=0.17, heavy_hi=0.30),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_tc_up_dense_branch_reuses_the_gemm_hidden_activations(cfg):
    L = synth.make_layer(cfg, seed=3)
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
    rows = out["ovf_rows"]
    assert n == len(rows) and n > 0
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), rows)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])

    # the routed rows against the exact dense layer: the units of the tiles
    # that fit carry one bf16 rounding of h, the overflowing tiles none
    x = O.bf16_bits_to_f64(L["x"][rows])
    z = x @ O.bf16_bits_to_f64(L["WgT"]).T
    h = np.maximum(z, 0.0) * (x @ O.bf16_bits_to_f64(L["WuT"]).T)
    wd = O.bf16_bits_to_f64(L["Wd"])
    counts = np.stack([(z[:, c * 128:(c + 1) * 128] > 0).sum(axis=1) for c in range(f // 128)], axis=1)
    fits = np.repeat(counts <= W, 128, axis=1)  # units whose tile fits
    bound = 2.0**-8 * (np.abs(h * fits) @ np.abs(wd)) + 2.0**-16 * (np.abs(h) @ np.abs(wd)) + 1e-6
    err = np.abs(yg[rows] - h @ wd)
    assert np.all(err <= bound), float((err / bound).max())

    # and close to the entry point that recomputes the routed rows' h exactly
    y2 = torch.zeros((T, d), dtype=torch.float32, device="cuda")
    tl.dense_rows_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], ovf_rows, n_ovf, y2, ws, st)
    assert tl.status_get(st) == 0
    assert_y_close(yg[rows], y_to_f64(y2)[rows])


def _routed_bound_check(yg, rows, h, wd, W):
    """y of the routed rows against the exact dense layer: the units of the
    tiles that fit carry one bf16 rounding of h, the overflowing tiles none."""
    counts = np.stack([(h[:, c * 128:(c + 1) * 128] > 0).sum(axis=1) for c in range(h.shape[1] // 128)], axis=1)
    fits = np.repeat(counts <= W, 128, axis=1)
    bound = 2.0**-8 * (np.abs(h * fits) @ np.abs(wd)) + 2.0**-16 * (np.abs(h) @ np.abs(wd)) + 1e-6
    err = np.abs(yg[rows] - h @ wd)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("cfg", RELU_CASES, ids=[c.name for c in RELU_CASES])
def test_relu_dense_branch_reuses_the_pack_gemm_hidden_activations(cfg):
    L = synth.make_layer(cfg, seed=5)
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
    rows = out["ovf_rows"]
    assert n == len(rows) and n > 0
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), rows)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])

    h = np.maximum(O.gate_preactivation(L["x"][rows], L["WgT"]), 0.0)
    _routed_bound_check(yg, rows, h, O.bf16_bits_to_f64(L["Wd"]), W)

    y2 = torch.zeros((T, d), dtype=torch.float32, device="cuda")
    tl.relu_dense_rows_forward(dev["x"], dev["WgT"], dev["Wd"], ovf_rows, n_ovf, y2, ws, st)
    assert tl.status_get(st) == 0
    assert_y_close(yg[rows], y_to_f64(y2)[rows])
