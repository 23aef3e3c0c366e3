"""GPU parity of the path for batches of at most 8 tokens (CUDA-core GEMVs:
the gate GEMV with the TwELL pack made by four-block clusters, routing with
the flags derived from the counts, the sparse step, and the dense branch as
GEMVs with fp32 hidden activations), and of the dense baselines' GEMV path.
Shapes: 1, 2, 3, 5 and 8 tokens (kernels compiled for 1, 2, 4 and 8); d of
256 to 2304 (the 2B layer's, 9 x 256); heavy tokens that overflow and take the
dense branch; and one d that is not a multiple of 256, which takes the split-K
GEMM path instead. All
three forms of the hybrid forward against the oracle's result of the method:
pack and routing bit-exact, y within the 2e-2 * rms contract; the dense
baselines within the bound of one bf16 rounding of h."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import (assert_dense_bf16_hidden_bound, assert_twell_equal, assert_y_close, twell_to_host,
                               upload, y_to_f64)

pytestmark = pytest.mark.gpu

LC = synth.LayerConfig
CASES = [
    LC("gemv_one", T=1, d=256, f=256, tile=128, W=16, density=0.1),
    LC("gemv_one_heavy", T=1, d=256, f=2304, tile=128, W=24, density=0.012, heavy_frac=1.0, heavy_lo=0.25,
       heavy_hi=0.40),
    LC("gemv_two", T=2, d=512, f=640, tile=128, W=16, density=0.04, sigma=0.5),
    LC("gemv_three", T=3, d=768, f=384, tile=128, W=8, density=0.03),
    LC("gemv_five_mixed", T=5, d=256, f=2304, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.4,
       heavy_lo=0.25, heavy_hi=0.40),
    LC("gemv_eight_2b", T=8, d=2304, f=9216, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.25,
       heavy_lo=0.25, heavy_hi=0.40),
    # d not a multiple of 256: the same batch sizes take the split-K GEMM path
    LC("small_d320", T=3, d=320, f=384, tile=128, W=8, density=0.05, heavy_frac=0.34, heavy_lo=0.25,
       heavy_hi=0.40),
]
IDS = [c.name for c in CASES]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


def _buffers(cfg):
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -7, dtype=torch.int32, device="cuda")
    n_ovf = torch.full((1,), -3, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    return tw, y, ovf_rows, n_ovf, ws


def _routing(ovf_rows, n_ovf, want_rows):
    n = int(n_ovf.item())
    assert n == len(want_rows)
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), want_rows)


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_small_batch_hybrid_gate_form(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    tw, y, ovf_rows, n_ovf, ws = _buffers(cfg)
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)
    _routing(ovf_rows, n_ovf, out["ovf_rows"])
    assert_twell_equal(twell_to_host(tw), out["twell"], cfg.W)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    if len(out["ovf_rows"]):
        # the dense branch keeps h in fp32: far inside the contract
        r = out["ovf_rows"]
        assert_y_close(yg[r], O.gated_ffn(L["x"][r], L["WgT"], L["WuT"], L["Wd"]), "dense-branch rows")


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_small_batch_hybrid_tensor_core_up_form(cfg):
    L = synth.make_layer(cfg, seed=1)
    dev = upload(L)
    tw, y, ovf_rows, n_ovf, ws = _buffers(cfg)
    st = tl.new_status()
    tl.ffn_hybrid_forward_tc_up(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_ffn_up_dense(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)
    _routing(ovf_rows, n_ovf, out["ovf_rows"])
    got, want = twell_to_host(tw), out["twell"]
    assert np.array_equal(got["counts"], want["counts"])
    assert np.array_equal(got["row_ovf"], want["row_ovf"])
    live = np.arange(cfg.W)[None, None, :] < np.minimum(want["counts"].astype(np.int64), cfg.W)[:, :, None]
    assert np.array_equal(got["idx"][live], want["idx"][live])
    # h = bf16(ReLU(z) u) from fp32 sums: within one bf16 step of the oracle's
    gv = O.bf16_bits_to_f64(got["vals"][live])
    wv = O.bf16_bits_to_f64(want["vals"][live])
    assert np.all(np.abs(gv - wv) <= 2.0**-7 * np.abs(wv) + 1e-30)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_small_batch_relu_hybrid_forward(cfg):
    L = synth.make_layer(cfg, seed=2)
    dev = upload(L)
    tw, y, ovf_rows, n_ovf, ws = _buffers(cfg)
    st = tl.new_status()
    tl.relu_ffn_hybrid_forward(dev["x"], dev["WgT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_relu_ffn(L["x"], L["WgT"], L["Wd"], cfg.tile, cfg.W)
    _routing(ovf_rows, n_ovf, out["ovf_rows"])
    assert_twell_equal(twell_to_host(tw), out["twell"], cfg.W)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_small_batch_dense_baselines(cfg):
    L = synth.make_layer(cfg, seed=3)
    dev = upload(L)
    ws = torch.empty(tl.dense_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    tl.dense_ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], y, ws, st)
    assert tl.status_get(st) == 0
    yg = y_to_f64(y)
    assert_y_close(yg, O.gated_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"]))
    assert_dense_bf16_hidden_bound(yg, L)
    y2 = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    tl.relu_dense_ffn_forward(dev["x"], dev["WgT"], dev["Wd"], y2, ws, st)
    assert tl.status_get(st) == 0
    assert_y_close(y_to_f64(y2), O.relu_ffn(L["x"], L["WgT"], L["Wd"]))


def test_small_batch_two_calls_give_the_same_pack_and_routing():
    """The pack is made by clusters exchanging counts: run it twice on
    different inputs into the same buffers; nothing of the first call may
    survive into the second."""
    cfg = CASES[3]
    tw, y, ovf_rows, n_ovf, ws = _buffers(cfg)
    for seed in (4, 5):
        L = synth.make_layer(cfg, seed=seed)
        dev = upload(L)
        st = tl.new_status()
        tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
        assert tl.status_get(st) == 0
        out = O.hybrid_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)
        _routing(ovf_rows, n_ovf, out["ovf_rows"])
        assert_twell_equal(twell_to_host(tw), out["twell"], cfg.W)
        assert_y_close(y_to_f64(y), out["y"])
