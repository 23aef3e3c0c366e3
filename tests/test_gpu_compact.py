"""GPU parity of dead-unit compaction: the activity bitmap, the column map and
the gathered weights are bit-exact against the oracle; the compacted layer's
hybrid forward matches the oracle on the compacted weights and stays within
one bf16 rounding per term of the original layer on the profile batch."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import assert_y_close, upload, y_to_f64
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

LC = synth.LayerConfig
DEAD = [
    LC("dead30", T=300, d=256, f=1024, tile=128, W=32, density=0.05, sigma=0.5, dead_frac=0.3),
    LC("dead_heavy", T=512, d=128, f=2304, tile=128, W=24, density=0.012, sigma=0.5, dead_frac=0.2,
       heavy_frac=0.08, heavy_lo=0.25, heavy_hi=0.40),
]
CASES = SMALL + DEAD
IDS = [c.name for c in CASES]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


def bits_to_bool(bits: torch.Tensor, f: int) -> np.ndarray:
    w = bits.cpu().numpy().view(np.uint32)
    return ((w[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).astype(bool).reshape(-1)[:f]


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_column_activity_and_compaction(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    st = tl.new_status()
    c = tl.compact_layer(dev["x"], {"WgT": dev["WgT"], "WuT": dev["WuT"], "Wd": dev["Wd"]}, st)
    assert tl.status_get(st) == 0
    act = O.column_activity(O.gate_preactivation(L["x"], L["WgT"]))
    assert np.array_equal(bits_to_bool(c["active_bits"], cfg.f), act)
    want = O.compact_layer(L["WgT"], L["WuT"], L["Wd"], act, cfg.tile)
    assert c["f_live"] == want["f_live"] and c["f_c"] == want["f_c"]
    assert np.array_equal(c["col_map"].cpu().numpy(), want["col_map"])
    for k in ("WgT", "WuT", "Wd"):
        assert np.array_equal(tl.bf16_bits(c[k]), want[k]), k


def test_column_activity_accumulates_over_batches():
    cfg = DEAD[0]
    L = synth.make_layer(cfg, seed=1)
    dev = upload(L)
    st = tl.new_status()
    bits = torch.full((cfg.f // 32,), -1, dtype=torch.int32, device="cuda")
    h = cfg.T // 2
    tl.column_activity(dev["x"][:h].contiguous(), dev["WgT"], bits, False, st)
    tl.column_activity(dev["x"][h:].contiguous(), dev["WgT"], bits, True, st)
    assert tl.status_get(st) == 0
    act = O.column_activity(O.gate_preactivation(L["x"], L["WgT"]))
    assert np.array_equal(bits_to_bool(bits, cfg.f), act)
    empty = torch.full((cfg.f // 32,), -1, dtype=torch.int32, device="cuda")
    tl.column_activity(dev["x"][:0], dev["WgT"], empty, False, st)
    assert not torch.any(empty)


@pytest.mark.parametrize("cfg", DEAD, ids=[c.name for c in DEAD])
def test_compacted_layer_hybrid_forward(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    st = tl.new_status()
    c = tl.compact_layer(dev["x"], {"WgT": dev["WgT"], "WuT": dev["WuT"], "Wd": dev["Wd"]}, st)
    f_c = c["f_c"]
    assert f_c < cfg.f
    tw = tl.Twell(cfg.T, f_c, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.empty((cfg.T,), dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, f_c), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_forward(dev["x"], c["WgT"], c["WuT"], c["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    ref_c = {k: tl.bf16_bits(c[k]) for k in ("WgT", "WuT", "Wd")}
    out = O.hybrid_ffn(L["x"], ref_c["WgT"], ref_c["WuT"], ref_c["Wd"], cfg.tile, cfg.W)
    n = int(n_ovf.item())
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), out["ovf_rows"])
    yg = y_to_f64(y)
    assert_y_close(yg, out["y"])
    # against the original layer: the dropped units were never active on this batch
    x = O.bf16_bits_to_f64(L["x"])
    h = np.maximum(x @ O.bf16_bits_to_f64(L["WgT"]).T, 0) * (x @ O.bf16_bits_to_f64(L["WuT"]).T)
    wd = O.bf16_bits_to_f64(L["Wd"])
    err = np.abs(yg - h @ wd)
    assert np.all(err <= np.abs(h) @ np.abs(wd) * 2.0**-7 + 1e-6)


def test_full_size_compaction_1p5b():
    cfg = synth.CONFIGS["1.5b"]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    st = tl.new_status()
    c = tl.compact_layer(dev["x"], {"WgT": dev["WgT"], "WuT": dev["WuT"], "Wd": dev["Wd"]}, st)
    assert tl.status_get(st) == 0
    act = np.zeros(cfg.f, dtype=bool)
    for r0 in range(0, cfg.T, 2048):
        act |= O.column_activity(O.gate_preactivation(L["x"][r0:r0 + 2048], L["WgT"]))
    assert np.array_equal(bits_to_bool(c["active_bits"], cfg.f), act)
    want = O.compact_layer(L["WgT"], L["WuT"], L["Wd"], act, cfg.tile)
    assert c["f_live"] == want["f_live"] < cfg.f
    assert np.array_equal(c["col_map"].cpu().numpy(), want["col_map"])
    for k in ("WgT", "WuT", "Wd"):
        assert np.array_equal(tl.bf16_bits(c[k]), want[k]), k
