"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on the
same seeded inputs. TwELL counts, slots, overflow flags and routing must be
bit-exact; y must satisfy max|y - y_ref| <= 2e-2 * rms(y_ref)."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O
from tests.gpu_helpers import (assert_dense_bf16_hidden_bound, assert_twell_equal, assert_within_stored_value_bound,
                               assert_y_close, oracle_pack_rows, run_pack, twell_to_host, upload, y_to_f64)

pytestmark = pytest.mark.gpu

LC = synth.LayerConfig
SMALL = [
    synth.CONFIGS["tiny"],
    # ragged T (2 full row blocks + 44), 4 column blocks, 3% dead columns
    LC("mid", T=300, d=256, f=1024, tile=128, W=16, density=0.05, sigma=0.5, dead_frac=0.03),
    # odd number of column tiles (last 256-column block half outside f), d = 3 K-blocks
    LC("odd", T=130, d=192, f=640, tile=128, W=8, density=0.03),
    # minimum d, full-width W
    LC("wide", T=200, d=64, f=384, tile=128, W=128, density=0.3),
    # heavy tokens that overflow and take the dense branch
    LC("heavy", T=1024, d=256, f=2304, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.08,
       heavy_lo=0.25, heavy_hi=0.40),
    LC("one_row", T=1, d=128, f=256, tile=128, W=16, density=0.1),
]
IDS = [c.name for c in SMALL]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


@pytest.fixture(scope="module")
def layers():
    return {c.name: synth.make_layer(c, seed=0) for c in SMALL}


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_gate_pack_bit_exact(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw, st = run_pack(dev, cfg.W)
    assert st == 0
    want = oracle_pack_rows(L, np.arange(cfg.T), cfg.tile, cfg.W)
    assert_twell_equal(twell_to_host(tw), want, cfg.W)


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_unpack_matches_oracle(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw, _ = run_pack(dev, cfg.W)
    g = torch.empty((cfg.T, cfg.f), dtype=torch.bfloat16, device="cuda")
    st = tl.new_status()
    tl.unpack(tw, g, st)
    assert tl.status_get(st) == 0
    want = oracle_pack_rows(L, np.arange(cfg.T), cfg.tile, cfg.W)
    g_ref = O.twell_unpack(want["counts"], want["idx"], want["vals"], cfg.f)
    assert np.array_equal(tl.bf16_bits(g), g_ref)


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_ffn_forward_non_hybrid(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, st)
    status = tl.status_get(st)
    want = oracle_pack_rows(L, np.arange(cfg.T), cfg.tile, cfg.W)
    n_ovf = int(want["row_ovf"].sum())
    assert status == (tl.TWELL_ERR_OVERFLOW if n_ovf else 0)
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    y_ref = O.sparse_ffn_from_twell(want, L["x"], L["WuT"], L["Wd"], rows=keep)
    assert_y_close(y_to_f64(y)[keep], y_ref)
    assert_within_stored_value_bound(y_to_f64(y)[keep], L, keep)


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_hybrid_forward(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -7, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)
    n = int(n_ovf.item())
    assert n == len(out["ovf_rows"])
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), out["ovf_rows"])
    assert_twell_equal(twell_to_host(tw), out["twell"], cfg.W)
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    keep = np.setdiff1d(np.arange(cfg.T), out["ovf_rows"])
    assert_within_stored_value_bound(yg[keep], L, keep)
    if n:
        y_dense = O.gated_ffn(L["x"][out["ovf_rows"]], L["WgT"], L["WuT"], L["Wd"])
        assert_y_close(yg[out["ovf_rows"]], y_dense, "dense-branch rows")


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_sparse_step_on_oracle_packed_input(cfg, layers):
    """The fused sparse kernel alone, fed the oracle's TwELL (independent of
    the gate kernel); rows that overflow are skipped and left untouched."""
    L = layers[cfg.name]
    dev = upload(L)
    want = oracle_pack_rows(L, np.arange(cfg.T), cfg.tile, cfg.W)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    tw.counts.copy_(torch.from_numpy(want["counts"]))
    tw.idx.copy_(torch.from_numpy(want["idx"]))
    tw.vals.copy_(torch.from_numpy(want["vals"].view(np.int16)).view(torch.bfloat16))
    tw.row_ovf.copy_(torch.from_numpy(want["row_ovf"]))
    sentinel = torch.full((cfg.T, cfg.d), 3.0, dtype=torch.float32, device="cuda")
    y = sentinel.clone()
    st = tl.new_status()
    tl.sparse_ffn(dev["x"], dev["WuT"], dev["Wd"], tw, y, True, st)
    assert tl.status_get(st) == 0
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    skip = np.nonzero(want["row_ovf"] != 0)[0]
    y_ref = O.sparse_ffn_from_twell(want, L["x"], L["WuT"], L["Wd"], rows=keep)
    assert_y_close(y_to_f64(y)[keep], y_ref)
    assert torch.equal(y[torch.from_numpy(skip).cuda()], sentinel[torch.from_numpy(skip).cuda()])


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_dense_ffn(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tl.dense_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.dense_ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], y, ws, st)
    assert tl.status_get(st) == 0
    assert_dense_bf16_hidden_bound(y_to_f64(y), L)


def test_dense_ffn_unquantised_inputs():
    """Plain N(0,1) bf16 inputs (no grid): the tensor-core GEMMs stay within
    the bound of one bf16 rounding of h against fp64."""
    rng = np.random.default_rng(0)
    T, d, f = 384, 512, 1280
    mk = lambda *s, sc=1.0: synth.f32_to_bf16_bits((rng.standard_normal(s) * sc).astype(np.float32))
    L = {"x": mk(T, d), "WgT": mk(f, d, sc=d**-0.5), "WuT": mk(f, d, sc=d**-0.5), "Wd": mk(f, d, sc=f**-0.5)}
    dev = upload(L)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tl.dense_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.dense_ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], y, ws, st)
    assert tl.status_get(st) == 0
    assert_dense_bf16_hidden_bound(y_to_f64(y), L)


def test_all_negative_gate_gives_empty_pack_and_zero_output(layers):
    cfg = SMALL[1]
    L = dict(layers[cfg.name])
    wg = O.bf16_bits_to_f64(L["WgT"]).copy()
    wg[:, -1] = -64.0
    L["WgT"] = synth.f32_to_bf16_bits(wg.astype(np.float32))
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), 5.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, st)
    assert tl.status_get(st) == 0
    assert int(tw.counts.abs().sum()) == 0 and int(tw.row_ovf.sum()) == 0
    assert int((y != 0).sum()) == 0


def test_all_positive_gate_full_width_equals_dense(layers):
    cfg = LC("allpos", T=256, d=128, f=256, tile=128, W=128, density=0.05)
    L = synth.make_layer(cfg, seed=4)
    wg = O.bf16_bits_to_f64(L["WgT"]).copy()
    wg[:, -1] = 64.0
    L["WgT"] = synth.f32_to_bf16_bits(wg.astype(np.float32))
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, st)
    assert tl.status_get(st) == 0
    assert int(tw.counts.min()) == 128
    assert_y_close(y_to_f64(y), O.gated_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"]))


def test_zero_tokens_is_a_noop():
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda")
    tw = tl.Twell(0, 256, 16)
    y = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.ffn_forward(x, w, w, w, tw, y, st)
    assert tl.status_get(st) == 0


def test_overflow_status_is_sticky_and_resettable(layers):
    cfg = SMALL[0]  # seed 0 of the small layer has one row over W = 16
    L = layers[cfg.name]
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.ffn_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, st)
    assert tl.status_get(st) == tl.TWELL_ERR_OVERFLOW
    tl.gate_pack(dev["x"], dev["WgT"], tw, st)
    assert tl.status_get(st) == tl.TWELL_ERR_OVERFLOW  # sticky
    tl.status_reset(st)
    tl.gate_pack(dev["x"], dev["WgT"], tw, st)
    assert tl.status_get(st) == 0


def test_out_of_range_index_is_reported_not_read(layers):
    cfg = SMALL[1]
    L = layers[cfg.name]
    dev = upload(L)
    tw, _ = run_pack(dev, cfg.W)
    torch.cuda.synchronize()
    row = int(torch.nonzero(tw.counts[:, 0] > 0)[0, 0])
    tw.idx[row, 0, 0] = 32000  # beyond f
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_ffn(dev["x"], dev["WuT"], dev["Wd"], tw, y, True, st)
    assert tl.status_get(st) == tl.TWELL_ERR_INDEX


# ---------------------------------------------------------------------------
# Tensor-core-up variant: the gate GEMM also forms u, TwELL holds h = z * u


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_gate_up_pack_pattern_bit_exact_and_hidden_values(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    st = tl.new_status()
    tl.gate_up_pack(dev["x"], dev["WgT"], dev["WuT"], tw, st)
    assert tl.status_get(st) == 0
    x = O.bf16_bits_to_f64(L["x"])
    z = x @ O.bf16_bits_to_f64(L["WgT"]).T
    u = x @ O.bf16_bits_to_f64(L["WuT"]).T
    want = O.twell_pack_hidden(z, u, cfg.tile, cfg.W)
    got = twell_to_host(tw)
    assert np.array_equal(got["counts"], want["counts"])
    assert np.array_equal(got["row_ovf"], want["row_ovf"])
    n = np.minimum(want["counts"].astype(np.int64), cfg.W)
    live = np.arange(cfg.W)[None, None, :] < n[:, :, None]
    assert np.array_equal(got["idx"][live], want["idx"][live])
    # u comes from fp32 tensor-core sums, so bf16(z * u) may differ by one ulp
    hv, wv = O.bf16_bits_to_f64(got["vals"][live]), O.bf16_bits_to_f64(want["vals"][live])
    assert np.all(np.abs(hv - wv) <= 2.0**-7 * np.abs(wv) + 1e-30)


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_hybrid_forward_tensor_core_up(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -7, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward_tc_up(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, ovf_rows, n_ovf, ws, st)
    assert tl.status_get(st) == 0
    out = O.hybrid_ffn_up_dense(L["x"], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)
    n = int(n_ovf.item())
    assert n == len(out["ovf_rows"])
    assert np.array_equal(ovf_rows[:n].cpu().numpy(), out["ovf_rows"])
    yg = y_to_f64(y)
    assert np.isfinite(yg).all()
    assert_y_close(yg, out["y"])
    keep = np.setdiff1d(np.arange(cfg.T), out["ovf_rows"])
    assert_within_stored_value_bound(yg[keep], L, keep, stored="h")


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_sparse_down_on_oracle_packed_input(cfg, layers):
    L = layers[cfg.name]
    dev = upload(L)
    x = O.bf16_bits_to_f64(L["x"])
    want = O.twell_pack_hidden(x @ O.bf16_bits_to_f64(L["WgT"]).T, x @ O.bf16_bits_to_f64(L["WuT"]).T,
                               cfg.tile, cfg.W)
    tw = tl.Twell(cfg.T, cfg.f, cfg.W)
    tw.counts.copy_(torch.from_numpy(want["counts"]))
    tw.idx.copy_(torch.from_numpy(want["idx"]))
    tw.vals.copy_(torch.from_numpy(want["vals"].view(np.int16)).view(torch.bfloat16))
    tw.row_ovf.copy_(torch.from_numpy(want["row_ovf"]))
    y = torch.full((cfg.T, cfg.d), 3.0, dtype=torch.float32, device="cuda")
    st = tl.new_status()
    tl.sparse_down(dev["Wd"], tw, y, True, st)
    assert tl.status_get(st) == 0
    keep = np.nonzero(want["row_ovf"] == 0)[0]
    assert_y_close(y_to_f64(y)[keep], O.sparse_down_from_twell(want, L["Wd"], rows=keep))


def test_gate_pack_unquantised_inputs():
    """Plain N(0,1) bf16 inputs (no exact grid): the tensor cores' fp32 sums
    may differ from fp64 in the last bits, so the pack is compared where the
    sign of z is decided: tiles whose every |z| exceeds 2^-10 * sum|x w| match
    exactly in counts and indices (values within one bf16 step); elsewhere the
    count may move by at most the number of undecided entries. The excluded
    count is reported."""
    rng = np.random.default_rng(7)
    T, d, f, W = 256, 512, 1024, 128
    mk = lambda *s, sc=1.0: synth.f32_to_bf16_bits((rng.standard_normal(s) * sc).astype(np.float32))
    L = {"x": mk(T, d), "WgT": mk(f, d, sc=d**-0.5)}
    dev = upload(dict(L, WuT=L["WgT"], Wd=L["WgT"]))
    tw = tl.Twell(T, f, W)
    st = tl.new_status()
    tl.gate_pack(dev["x"], dev["WgT"], tw, st)
    assert tl.status_get(st) == 0
    got = twell_to_host(tw)
    x, w = O.bf16_bits_to_f64(L["x"]), O.bf16_bits_to_f64(L["WgT"])
    z = x @ w.T
    margin = 2.0**-10 * (np.abs(x) @ np.abs(w).T)
    undecided = np.abs(z) <= margin
    ref = O.twell_pack(z, 128, W)
    nT = f // 128
    und_tiles = undecided.reshape(T, nT, 128).sum(axis=2)
    clean = und_tiles == 0
    print(f"undecided entries: {int(undecided.sum())} of {T * f}; tiles excluded: {int((~clean).sum())}")
    assert np.array_equal(got["counts"][clean], ref["counts"][clean])
    assert np.all(np.abs(got["counts"].astype(int) - ref["counts"].astype(int)) <= und_tiles)
    for t, c in zip(*np.nonzero(clean)):
        n = int(ref["counts"][t, c])
        assert np.array_equal(got["idx"][t, c, :n], ref["idx"][t, c, :n])
        gv, rv = O.bf16_bits_to_f64(got["vals"][t, c, :n]), O.bf16_bits_to_f64(ref["vals"][t, c, :n])
        assert np.all(np.abs(gv - rv) <= 2.0**-7 * np.abs(rv))
