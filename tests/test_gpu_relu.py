"""GPU parity of the non-gated layer y = ReLU(x W1) W2 (hybrid forward and the
dense baseline) against the CPU oracle. The synthetic layers' gate weights
serve as W1 and their down weights as W2, so the sparsity structure is that of
the gated configurations. TwELL and routing are bit-exact; y must satisfy
max|y - y_ref| <= 2e-2 * rms(y_ref) against the oracle's hybrid result and stay
within one bf16 rounding per term of the exact dense layer."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import assert_twell_equal, assert_y_close, twell_to_host, upload, y_to_f64
from tests.test_gpu_parity import IDS, SMALL

pytestmark = pytest.mark.gpu

CHUNK = 2048


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


@pytest.fixture(scope="module")
def layers():
    return {c.name: synth.make_layer(c, seed=0) for c in SMALL}


def relu_bound_check(y_gpu: np.ndarray, L: dict, rows) -> None:
    """|y - ReLU(x W1) W2| <= 2^-7 * ReLU(x W1) |W2| (+ fp32 slack): the sparse
    rows use the bf16-rounded ReLU outputs, one rounding of 2^-8 per term."""
    g = np.maximum(O.gate_preactivation(L["x"][rows], L["WgT"]), 0)
    w2 = O.bf16_bits_to_f64(L["Wd"])
    err = np.abs(y_gpu - g @ w2)
    bound = g @ np.abs(w2) * 2.0**-7 + 1e-6
    assert np.all(err <= bound), float((err / bound).max())


def run_relu_hybrid(dev, cfg):
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -7, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.relu_ffn_hybrid_forward(dev["x"], dev["WgT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    n = int(n_ovf.item())
    return tw, y, ovf_rows[:n].cpu().numpy()


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_relu_hybrid_forward(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw, y, ovf = run_relu_hybrid(dev, cfg)
    out = O.hybrid_relu_ffn(L["x"], L["WgT"], L["Wd"], cfg.tile, cfg.W)
    assert np.array_equal(ovf, out["ovf_rows"])
    assert_twell_equal(twell_to_host(tw), out["twell"], cfg.W)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    relu_bound_check(yg, L, np.arange(cfg.T))
    if ovf.size:
        assert_y_close(yg[ovf], O.relu_ffn(L["x"][ovf], L["WgT"], L["Wd"]), "dense-branch rows")


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_relu_dense_ffn(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tl.dense_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.relu_dense_ffn_forward(dev["x"], dev["WgT"], dev["Wd"], y, ws, st)
    assert tl.status_get(st) == 0
    relu_bound_check(y_to_f64(y), L, np.arange(cfg.T))


def test_relu_all_negative_gives_zero(layers):
    cfg = SMALL[1]
    L = dict(layers[cfg.name])
    neg = O.bf16_bits_to_f64(L["WgT"]).copy()
    neg[:, -1] = -64.0
    L["WgT"] = O.f64_to_bf16_bits(neg)
    tw, y, ovf = run_relu_hybrid(upload(L), cfg)
    assert ovf.size == 0
    assert int(tw.counts.to(torch.int64).sum()) == 0
    assert not torch.any(y)


@pytest.mark.parametrize("name", ["0.5b"])
def test_relu_full_size_hybrid_forward(name):
    """Full layer size, as bench.py times it: counts, flags and routing over
    every row; y on sampled rows and on overflow rows."""
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    tw, y, ovf = run_relu_hybrid(upload(L), cfg)
    counts = tw.counts.cpu().numpy()
    all_counts = np.empty_like(counts)
    for r0 in range(0, cfg.T, CHUNK):
        rows = np.arange(r0, min(cfg.T, r0 + CHUNK))
        all_counts[rows] = O.twell_pack(O.gate_preactivation(L["x"][rows], L["WgT"]), cfg.tile, cfg.W)["counts"]
    assert np.array_equal(counts, all_counts)
    assert np.array_equal(ovf, O.route_rows(all_counts, cfg.W))
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    rng = np.random.default_rng(2)
    sample = np.sort(rng.choice(cfg.T, size=256, replace=False))
    rows = np.union1d(sample, ovf[:64])
    ref = O.hybrid_relu_ffn(L["x"][rows], L["WgT"], L["Wd"], cfg.tile, cfg.W)
    assert_y_close(yg[rows], ref["y"])
    relu_bound_check(yg[rows], L, rows)
