"""GPU parity of the down projection over tile unions on the tensor cores
(twell_sparse_down_union) on the oracle's own pack of hidden values: y of the
rows that fit against the oracle's down projection of the same stored values,
within the contract and within fp32 summation error of the exact sum (a
dropped, doubled or misplaced slot fails it); overflow rows written as zeros
when skipped; the overflow status without skipping; an index outside its tile
reported and left out; an empty pack; a canary margin around y."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import assert_y_close, upload, y_to_f64
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

IDS = [c.name for c in SMALL]
SUM_BOUND = 2.0**-12  # fp32 sums of at most a few thousand exact bf16 x bf16 products


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


def oracle_hidden_pack(L, cfg):
    x = O.bf16_bits_to_f64(L["x"])
    return O.twell_pack_hidden(x @ O.bf16_bits_to_f64(L["WgT"]).T, x @ O.bf16_bits_to_f64(L["WuT"]).T,
                               cfg.tile, cfg.W)


def device_twell(want, cfg):
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    tw.counts.copy_(torch.from_numpy(want["counts"]))
    tw.idx.copy_(torch.from_numpy(want["idx"]))
    tw.vals.copy_(torch.from_numpy(want["vals"].view(np.int16)).view(torch.bfloat16))
    tw.row_ovf.copy_(torch.from_numpy(want["row_ovf"]))
    return tw


def union_ws(cfg):
    return torch.empty(tl.sparse_down_union_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")


def assert_sum_exact(yg, want, L, rows):
    h = O.bf16_bits_to_f64(O.twell_unpack(want["counts"][rows], want["idx"][rows], want["vals"][rows],
                                          O.bf16_bits_to_f64(L["Wd"]).shape[0]))
    wd = O.bf16_bits_to_f64(L["Wd"])
    ref = h @ wd
    bound = SUM_BOUND * (np.abs(h) @ np.abs(wd)) + 1e-30
    err = np.abs(yg - ref)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_union_down_on_oracle_packed_input(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    tw = device_twell(want, cfg)
    y = torch.full((cfg.T, cfg.d), 3.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_union(dev["Wd"], tw, y, True, union_ws(cfg), st)
    assert tl.status_get(st) == 0
    yg = y_to_f64(y)
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    ovf = np.nonzero(want["row_ovf"] == 1)[0]
    assert_y_close(yg[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
    assert_sum_exact(yg[keep], want, L, keep)
    assert np.all(yg[ovf] == 0.0), "a skipped overflow row was not zeroed"


def test_union_down_without_skipping_raises_overflow():
    cfg = next(c for c in SMALL if c.name == "heavy")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    assert want["row_ovf"].any()
    tw = device_twell(want, cfg)
    y = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_union(dev["Wd"], tw, y, False, union_ws(cfg), st)
    assert tl.status_get(st) == tl.TWELL_ERR_OVERFLOW
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    assert_y_close(y_to_f64(y)[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))


@pytest.mark.parametrize("bad", [200, -5, 10_000])
def test_union_down_index_outside_its_tile_is_reported_and_left_out(bad):
    cfg = next(c for c in SMALL if c.name == "mid")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    t = int(np.nonzero((want["row_ovf"] == 0) & (want["counts"][:, 0] > 0))[0][0])
    broken = {k: np.copy(v) for k, v in want.items()}
    broken["idx"][t, 0, 0] = bad  # tile 0 holds columns 0..127: 200 lies in tile 1, the others outside [0, f)
    tw = device_twell(broken, cfg)
    y = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_union(dev["Wd"], tw, y, True, union_ws(cfg), st)
    assert tl.status_get(st) == tl.TWELL_ERR_INDEX
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    keep = np.setdiff1d(np.nonzero(want["row_ovf"] == 0)[0], [t])
    assert_y_close(yg[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
    fixed = {k: np.copy(v) for k, v in want.items()}
    fixed["vals"][t, 0, 0] = 0
    assert_y_close(yg[[t]], O.sparse_down_from_twell(fixed, L["Wd"], rows=[t]))


def test_union_down_empty_pack_gives_zero_and_zero_tokens_is_a_noop():
    cfg = next(c for c in SMALL if c.name == "mid")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    tw.counts.zero_()
    tw.row_ovf.zero_()
    y = torch.full((cfg.T, cfg.d), 7.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_union(dev["Wd"], tw, y, True, union_ws(cfg), st)
    assert tl.status_get(st) == 0
    assert not torch.any(y)
    tw0 = tl.Twell(0, cfg.f, cfg.W)
    y0 = torch.empty((0, cfg.d), dtype=torch.float32, device="cuda")
    tl.sparse_down_union(dev["Wd"], tw0, y0, True, torch.empty(16, dtype=torch.uint8, device="cuda"), st)
    assert tl.status_get(st) == 0


def test_union_down_stays_inside_its_outputs():
    """y and the workspace inside larger allocations with sentinel margins:
    nothing outside them changes."""
    cfg = next(c for c in SMALL if c.name == "heavy")
    L = synth.make_layer(cfg, seed=2)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    tw = device_twell(want, cfg)
    pad = 64
    ybig = torch.full((cfg.T * cfg.d + 2 * pad,), -9.0, dtype=torch.float32, device="cuda")
    y = ybig[pad:pad + cfg.T * cfg.d].view(cfg.T, cfg.d)
    need = tl.sparse_down_union_workspace_bytes(cfg.T, cfg.d, cfg.f)
    wbig = torch.full((need + 2 * 256,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = wbig[256:256 + need]
    st = tl.new_status()
    tl.sparse_down_union(dev["Wd"], tw, y, True, ws, st)
    assert tl.status_get(st) == 0
    assert torch.all(ybig[:pad] == -9.0) and torch.all(ybig[-pad:] == -9.0)
    assert torch.all(wbig[:256] == 0xA5) and torch.all(wbig[-256:] == 0xA5)
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    assert_y_close(y_to_f64(y)[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
