"""GPU parity of the down projection staged through shared memory
(twell_sparse_down_staged, the alternative form of the tensor-core-up
variant's down projection): y against the oracle's down projection of the same
stored values, within the contract tolerance and within fp32 summation error
of the exact sum; rows skipped for overflow left untouched; the overflow and
index statuses; agreement with the per-token kernel at a multi-wave size and
at the full layer sizes. Also the tensor-core-up hybrid forward at the full
layer sizes."""

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
CASES = [c for c in SMALL if c.d >= 128]
IDS = [c.name for c in CASES]
# more units (token groups x 128-column slices) than a B200 has SMs, small enough for the oracle
MULTIWAVE = LC("multiwave", T=2400, d=2048, f=1024, tile=128, W=16, density=0.05, sigma=0.5, dead_frac=0.03)
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


def staged_ws(cfg):
    return torch.empty(tl.sparse_down_staged_workspace_bytes(cfg.T, cfg.d, cfg.f, cfg.W), dtype=torch.uint8,
                       device="cuda")


def assert_sum_exact(yg, want, L, rows):
    """|y - sum of the stored terms| within fp32 summation error of the terms'
    magnitudes: a dropped, doubled or misplaced slot fails this."""
    h = O.bf16_bits_to_f64(O.twell_unpack(want["counts"][rows], want["idx"][rows], want["vals"][rows],
                                          O.bf16_bits_to_f64(L["Wd"]).shape[0]))
    wd = O.bf16_bits_to_f64(L["Wd"])
    ref = h @ wd
    bound = SUM_BOUND * (np.abs(h) @ np.abs(wd)) + 1e-30
    err = np.abs(yg - ref)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_staged_down_on_oracle_packed_input(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    tw = device_twell(want, cfg)
    y = torch.full((cfg.T, cfg.d), 3.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_staged(dev["Wd"], tw, y, True, staged_ws(cfg), st)
    assert tl.status_get(st) == 0
    yg = y_to_f64(y)
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    ovf = np.nonzero(want["row_ovf"] == 1)[0]
    assert_y_close(yg[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
    assert_sum_exact(yg[keep], want, L, keep)
    assert np.all(yg[ovf] == 3.0), "a skipped overflow row was written"


@pytest.mark.parametrize("cfg", CASES, ids=IDS)
def test_staged_down_agrees_with_the_per_token_kernel(cfg):
    L = synth.make_layer(cfg, seed=1)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    tw = device_twell(want, cfg)
    st = tl.new_status()
    y1 = torch.full((cfg.T, cfg.d), 5.0, dtype=torch.float32, device="cuda")
    y2 = torch.full((cfg.T, cfg.d), 5.0, dtype=torch.float32, device="cuda")
    tl.sparse_down(dev["Wd"], tw, y1, True, st)
    tl.sparse_down_staged(dev["Wd"], tw, y2, True, staged_ws(cfg), st)
    assert tl.status_get(st) == 0
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    a, b = y_to_f64(y1), y_to_f64(y2)
    assert np.array_equal(a[want["row_ovf"] == 1], b[want["row_ovf"] == 1])
    assert_sum_exact(b[keep], want, L, keep)
    assert_sum_exact(a[keep], want, L, keep)


def test_staged_down_without_skipping_raises_overflow():
    cfg = next(c for c in CASES if c.name == "heavy")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    assert want["row_ovf"].any()
    tw = device_twell(want, cfg)
    y = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_staged(dev["Wd"], tw, y, False, staged_ws(cfg), st)
    assert tl.status_get(st) == tl.TWELL_ERR_OVERFLOW
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    assert_y_close(y_to_f64(y)[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))


@pytest.mark.parametrize("bad", [200, -5, 10_000])
def test_staged_down_index_outside_its_tile_is_reported_not_read(bad):
    cfg = next(c for c in CASES if c.name == "mid")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    t = int(np.nonzero((want["row_ovf"] == 0) & (want["counts"][:, 0] > 0))[0][0])
    broken = {k: np.copy(v) for k, v in want.items()}
    broken["idx"][t, 0, 0] = bad  # tile 0 holds columns 0..127: 200 lies in tile 1, the others outside [0, f)
    tw = device_twell(broken, cfg)
    y = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_staged(dev["Wd"], tw, y, True, staged_ws(cfg), st)
    assert tl.status_get(st) == tl.TWELL_ERR_INDEX
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    keep = np.setdiff1d(np.nonzero(want["row_ovf"] == 0)[0], [t])
    assert_y_close(yg[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
    # the bad slot adds nothing: row t is the sum of its other slots
    fixed = {k: np.copy(v) for k, v in want.items()}
    fixed["vals"][t, 0, 0] = 0
    assert_y_close(yg[[t]], O.sparse_down_from_twell(fixed, L["Wd"], rows=[t]))


def test_staged_down_empty_pack_gives_zero_and_zero_tokens_is_a_noop():
    cfg = next(c for c in CASES if c.name == "mid")
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    tw.counts.zero_()
    tw.row_ovf.zero_()
    y = torch.full((cfg.T, cfg.d), 7.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down_staged(dev["Wd"], tw, y, True, staged_ws(cfg), st)
    assert tl.status_get(st) == 0
    assert not torch.any(y)
    tw0 = tl.Twell(0, cfg.f, cfg.W)
    y0 = torch.empty((0, cfg.d), dtype=torch.float32, device="cuda")
    tl.sparse_down_staged(dev["Wd"], tw0, y0, True, torch.empty(16, dtype=torch.uint8, device="cuda"), st)
    assert tl.status_get(st) == 0


def _hybrid_buffers(cfg):
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    return tw, y, ovf_rows, n_ovf, ws


def test_staged_down_over_several_waves_matches_the_oracle():
    cfg = MULTIWAVE
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    want = oracle_hidden_pack(L, cfg)
    tw = device_twell(want, cfg)
    st = tl.new_status()
    y = torch.full((cfg.T, cfg.d), 3.0, dtype=torch.float32, device="cuda")
    tl.sparse_down_staged(dev["Wd"], tw, y, True, staged_ws(cfg), st)
    assert tl.status_get(st) == 0
    yg = y_to_f64(y)
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    assert_y_close(yg[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))
    assert_sum_exact(yg[keep], want, L, keep)
    assert np.all(yg[want["row_ovf"] == 1] == 3.0)


@pytest.mark.parametrize("name", ["0.5b", "2b"])
def test_full_size_staged_down_agrees_with_the_per_token_kernel(name):
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    st = tl.new_status()
    tl.gate_up_pack(dev["x"], dev["WgT"], dev["WuT"], tw, st)
    y1 = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    y2 = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    tl.sparse_down(dev["Wd"], tw, y1, True, st)
    tl.sparse_down_staged(dev["Wd"], tw, y2, True, staged_ws(cfg), st)
    assert tl.status_get(st) == 0
    # both sum a token's slots in ascending column order in fp32; allow for reordering
    rms = float(y1.pow(2).mean().sqrt())
    assert float((y1 - y2).abs().max()) <= 1e-5 * rms


@pytest.mark.parametrize("name", ["0.5b", "2b"])
def test_full_size_tensor_core_up_hybrid_forward(name):
    """The tensor-core-up hybrid forward at the full layer sizes, as bench.py
    times it: y on sampled rows that fit and on overflow rows."""
    cfg = synth.CONFIGS[name]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    tw, y, ovf_rows, n_ovf, ws = _hybrid_buffers(cfg)
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
    sample = np.sort(rng.choice(cfg.T, size=256, replace=False))
    keep = sample[row_ovf[sample] == 0]
    x = O.bf16_bits_to_f64(L["x"][keep])
    want = O.twell_pack_hidden(x @ O.bf16_bits_to_f64(L["WgT"]).T, x @ O.bf16_bits_to_f64(L["WuT"]).T,
                               cfg.tile, cfg.W)
    assert np.array_equal(want["row_ovf"], np.zeros(len(keep), np.uint8))
    y_keep = O.sparse_down_from_twell(want, L["Wd"])
    rows = np.concatenate([keep, ovf[:64]])
    y_ref = np.concatenate([y_keep, O.gated_ffn(L["x"][ovf[:64]], L["WgT"], L["WuT"], L["Wd"])])
    assert_y_close(yg[rows], y_ref)
