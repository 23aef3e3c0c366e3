"""Pins for the CPU oracle, checked against things other than the oracle itself:
closed forms, exact rational arithmetic, torch's bf16 conversions (library
routines), a hand-written fixture, brute-force loops and invariants.

CPU only (no GPU marker)."""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from oracle import twell_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_bf16_bits(values_f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) by torch, as raw bits."""
    t = torch.from_numpy(np.ascontiguousarray(values_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_of_exact(values) -> np.ndarray:
    """bf16 bits of values that are exactly representable in bf16."""
    v = np.asarray(values, dtype=np.float32)
    b = torch_bf16_bits(v)
    assert np.array_equal(O.bf16_bits_to_f64(b), v.astype(np.float64))
    return b


# ---------------------------------------------------------------------------
# bf16 conversions


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 16, size=20000, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_bits_to_f64(bits), ref)


def test_bf16_round_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(2)
    raw = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    raw = raw[(raw & 0x7F800000) != 0x7F800000]  # finite
    raw = raw[(raw & 0x7F800000) < 0x7F000000]  # keep clear of overflow to inf
    ties = (rng.integers(0, 1 << 16, size=5000, dtype=np.uint32) << 16) | 0x8000
    ties = ties[(ties & 0x7F800000) < 0x7F000000].astype(np.uint32)
    vals = np.concatenate([raw, ties]).view(np.float32)
    assert np.array_equal(O.f64_to_bf16_bits(vals.astype(np.float64)), torch_bf16_bits(vals))


def _all_finite_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)  # +0 .. largest finite
    return bits, O.bf16_bits_to_f64(bits)


def test_bf16_round_bruteforce_nearest_even():
    """Direct fp64 -> bf16 rounding equals the nearest entry of the full table
    of bf16 values, ties to the even bit pattern (no double rounding)."""
    tb, tv = _all_finite_bf16()
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, size=4000),
        np.ldexp(rng.random(500), -rng.integers(120, 134, size=500)),  # bf16 subnormals
        [1 + 2.0**-8, 1 + 3 * 2.0**-8, 1 + 2.0**-8 + 2.0**-30, 0.0, -0.0, 2.0**-133, 3 * 2.0**-134],
    ])
    got = O.f64_to_bf16_bits(x)
    for xi, gi in zip(x, got):
        a = abs(xi)
        k = int(np.searchsorted(tv, a))
        cands = [c for c in (k - 1, k) if 0 <= c < len(tv)]
        best = min(cands, key=lambda c: (abs(tv[c] - a), int(tb[c]) & 1))
        want = int(tb[best]) | (0x8000 if math.copysign(1.0, xi) < 0 else 0)
        assert int(gi) == want, (xi, hex(int(gi)), hex(want))
    # the case where rounding through fp32 first would differ
    assert int(O.f64_to_bf16_bits(np.array([1 + 2.0**-8 + 2.0**-30]))[0]) == 0x3F81


# ---------------------------------------------------------------------------
# TwELL pack against a hand-derived fixture


def load_golden_pack(path):
    z = None
    counts, slots, ovf = {}, {}, {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "shape":
            T, f, tile, W = map(int, tok[1:])
            z = np.full((T, f), -1.0)
        elif tok[0] == "z":
            z[int(tok[1]), int(tok[2])] = float(tok[3])
        elif tok[0] == "counts":
            counts[(int(tok[1]), int(tok[2]))] = int(tok[3])
        elif tok[0] == "slot":
            slots[(int(tok[1]), int(tok[2]), int(tok[3]))] = (int(tok[4]), int(tok[5], 16))
        elif tok[0] == "ovf":
            ovf[int(tok[1])] = int(tok[2])
    return z, tile, W, counts, slots, ovf


def test_pack_matches_hand_fixture():
    z, tile, W, counts, slots, ovf = load_golden_pack(os.path.join(GOLDEN, "twell_pack_small.txt"))
    tw = O.twell_pack(z, tile, W)
    for (t, c), n in counts.items():
        assert tw["counts"][t, c] == n
    for (t, c, s), (j, v) in slots.items():
        assert tw["idx"][t, c, s] == j and tw["vals"][t, c, s] == v
    # every slot past the stored ones is padding
    T, nT, _ = tw["idx"].shape
    for t in range(T):
        for c in range(nT):
            for s in range(min(counts[(t, c)], W), W):
                assert tw["idx"][t, c, s] == -1 and tw["vals"][t, c, s] == 0
    assert [int(v) for v in tw["row_ovf"]] == [ovf[t] for t in range(T)]
    assert O.route_rows(tw["counts"], W).tolist() == [t for t in range(T) if ovf[t]]


# ---------------------------------------------------------------------------
# TwELL pack by brute force


def pack_by_loops(z, tile, W):
    T, f = z.shape
    nT = f // tile
    counts = np.zeros((T, nT), dtype=np.int64)
    idx = np.full((T, nT, W), -1, dtype=np.int64)
    vals = np.zeros((T, nT, W), dtype=np.int64)
    for t in range(T):
        for c in range(nT):
            n = 0
            for k in range(tile):
                j = c * tile + k
                if z[t, j] > 0:
                    if n < W:
                        idx[t, c, n] = j
                        vals[t, c, n] = int(torch_bf16_bits(np.array([z[t, j]], np.float32))[0])
                    n += 1
            counts[t, c] = n
    return counts, idx, vals


@pytest.mark.parametrize("W", [1, 2, 16, 128])
@pytest.mark.parametrize("seed", range(4))
def test_pack_bruteforce(W, seed):
    rng = np.random.default_rng(100 + seed)
    T, f, tile = int(rng.integers(1, 9)), 256, 128
    density = rng.choice([0.02, 0.1, 0.5, 0.95])
    z = rng.standard_normal((T, f)).astype(np.float32)
    z = np.where(rng.random((T, f)) < density, np.abs(z), -np.abs(z))
    z[rng.random((T, f)) < 0.05] = 0.0  # exact zeros are inactive
    z = z.astype(np.float64)  # fp32-exact values, so torch's rounding applies
    tw = O.twell_pack(z, tile, W)
    counts, idx, vals = pack_by_loops(z, tile, W)
    assert np.array_equal(tw["counts"], counts)
    assert np.array_equal(tw["idx"], idx)
    assert np.array_equal(tw["vals"].astype(np.int64), vals)
    assert np.array_equal(tw["row_ovf"], (counts > W).any(axis=1).astype(np.uint8))


def test_pack_unpack_roundtrip_full_width():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((16, 512)).astype(np.float32).astype(np.float64)
    tw = O.twell_pack(z, 128, 128)
    g = O.twell_unpack(tw["counts"], tw["idx"], tw["vals"], 512)
    want = torch_bf16_bits(np.maximum(z, 0).astype(np.float32))
    assert np.array_equal(g, want)
    assert tw["row_ovf"].sum() == 0


MID = synth.LayerConfig("mid", T=512, d=256, f=1024, tile=128, W=16, density=0.05,
                        sigma=0.5, dead_frac=0.03)
HEAVY = synth.LayerConfig("heavy", T=1024, d=256, f=2304, tile=128, W=24, density=0.012,
                          sigma=0.5, heavy_frac=0.08, heavy_lo=0.25, heavy_hi=0.40)


@pytest.mark.parametrize("cfg", [synth.CONFIGS["tiny"], MID], ids=lambda c: c.name)
def test_pack_invariants_on_synthetic_layers(cfg):
    L = synth.make_layer(cfg, seed=0)
    z = O.gate_preactivation(L["x"], L["WgT"])
    tw = O.twell_pack(z, cfg.tile, cfg.W)
    assert tw["counts"].astype(np.int64).sum() == int((z > 0).sum())
    n = np.minimum(tw["counts"], cfg.W)
    for t in range(cfg.T):
        for c in range(cfg.nT):
            js = tw["idx"][t, c, : n[t, c]].astype(np.int64)
            assert np.all(np.diff(js) > 0)
            assert np.all((js >= c * cfg.tile) & (js < (c + 1) * cfg.tile))
            assert np.all(z[t, js] > 0)
            assert np.array_equal(tw["vals"][t, c, : n[t, c]], O.f64_to_bf16_bits(z[t, js]))
    assert np.array_equal(tw["row_ovf"], (tw["counts"] > cfg.W).any(axis=1).astype(np.uint8))


def test_route_is_the_overflow_predicate():
    rng = np.random.default_rng(7)
    counts = rng.integers(0, 40, size=(300, 9)).astype(np.int16)
    for W in (8, 16, 24, 32, 39):
        want = [t for t in range(counts.shape[0]) if any(int(c) > W for c in counts[t])]
        assert O.route_rows(counts, W).tolist() == want


# ---------------------------------------------------------------------------
# The dense layer: closed forms and exact arithmetic


def test_dense_permutation_closed_form():
    """With permutation matrices the layer is an index shuffle:
    z_j = x[pa(j)], u_j = x[pb(j)], y[pc(j)] = ReLU(z_j) * u_j. A transposed
    operand would apply the inverse permutation and fail."""
    rng = np.random.default_rng(8)
    n, T = 32, 5
    pa, pb, pc = rng.permutation(n), rng.permutation(n), rng.permutation(n)
    assert not np.array_equal(pa, np.argsort(pa))
    eye = np.eye(n)
    WgT, WuT, Wd = eye[pa], eye[pb], eye[pc]  # WgT[j, pa(j)] = 1, Wd[j, pc(j)] = 1
    xv = (rng.integers(-40, 40, size=(T, n)) / 8.0)
    x = bits_of_exact(xv)
    y = O.gated_ffn(x, bits_of_exact(WgT), bits_of_exact(WuT), bits_of_exact(Wd))
    want = np.zeros((T, n))
    for j in range(n):
        want[:, pc[j]] = np.maximum(xv[:, pa[j]], 0) * xv[:, pb[j]]
    assert np.array_equal(y, want)


def test_dense_exact_rational_bruteforce():
    rng = np.random.default_rng(9)
    T, d, f = 3, 6, 10
    x = torch_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    WgT = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    WuT = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    Wd = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    F = lambda b: [[Fraction(float(v)) for v in row] for row in O.bf16_bits_to_f64(b)]
    xf, gf, uf, df = F(x), F(WgT), F(WuT), F(Wd)
    y = O.gated_ffn(x, WgT, WuT, Wd)
    for t in range(T):
        for k in range(d):
            acc = Fraction(0)
            for j in range(f):
                zj = sum(xf[t][i] * gf[j][i] for i in range(d))
                uj = sum(xf[t][i] * uf[j][i] for i in range(d))
                acc += max(zj, Fraction(0)) * uj * df[j][k]
            assert abs(y[t, k] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_dense_special_cases():
    L = synth.make_layer(synth.CONFIGS["tiny"], seed=3)
    x, WgT, WuT, Wd = L["x"], L["WgT"], L["WuT"], L["Wd"]
    y = O.gated_ffn(x, WgT, WuT, Wd)
    # scaling x by 2 scales both z and u: y quadruples (exact powers of two)
    x2 = bits_of_exact(2 * O.bf16_bits_to_f64(x))
    assert np.array_equal(O.gated_ffn(x2, WgT, WuT, Wd), 4 * y)
    # scaling Wd by 2 doubles y
    assert np.array_equal(O.gated_ffn(x, WgT, WuT, bits_of_exact(2 * O.bf16_bits_to_f64(Wd))), 2 * y)
    # an all-negative gate gives y == 0 and an empty pack
    neg = O.bf16_bits_to_f64(WgT).copy()
    neg[:, -1] = -64.0
    negb = bits_of_exact(neg)
    assert not np.any(O.gated_ffn(x, negb, WuT, Wd))
    tw = O.twell_pack(O.gate_preactivation(x, negb), 128, 16)
    assert tw["counts"].sum() == 0 and tw["row_ovf"].sum() == 0
    # one active column j*: y = relu(z_j*) * u_j* * Wd[j*, :]
    one = neg.copy()
    js = 77
    one[js, -1] = 64.0
    oneb = bits_of_exact(one)
    xf = O.bf16_bits_to_f64(x)
    zj = xf @ O.bf16_bits_to_f64(oneb)[js]
    uj = xf @ O.bf16_bits_to_f64(WuT)[js]
    want = (zj * uj)[:, None] * O.bf16_bits_to_f64(Wd)[js][None, :]
    assert np.all(zj > 0)
    np.testing.assert_allclose(O.gated_ffn(x, oneb, WuT, Wd), want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# sparse == dense


def test_sparse_equals_dense_when_gate_is_bf16_exact():
    """Small-integer inputs keep z exactly representable in bf16, so the
    stored values are exact and the sparse sum equals the dense layer."""
    rng = np.random.default_rng(11)
    T, d, f = 24, 8, 256
    x = bits_of_exact(rng.integers(-3, 4, size=(T, d)).astype(np.float64))
    WgT = bits_of_exact(rng.integers(-3, 4, size=(f, d)).astype(np.float64))
    WuT = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    Wd = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    z = O.gate_preactivation(x, WgT)
    tw = O.twell_pack(z, 128, 128)
    assert np.array_equal(O.bf16_bits_to_f64(O.f64_to_bf16_bits(z)), z)
    ys = O.sparse_ffn_from_twell(tw, x, WuT, Wd)
    yd = O.gated_ffn(x, WgT, WuT, Wd)
    np.testing.assert_allclose(ys, yd, rtol=1e-12, atol=1e-12 * np.abs(yd).max())


def test_sparse_within_bf16_bound_of_dense():
    """With the stored bf16 gate, each term h_j Wd[j,k] moves by at most
    2^-8 relative (one nearest rounding to 8 significant bits), which bounds
    |y_sparse - y_dense|."""
    cfg = synth.CONFIGS["tiny"]
    L = synth.make_layer(cfg, seed=0)
    z = O.gate_preactivation(L["x"], L["WgT"])
    tw = O.twell_pack(z, cfg.tile, cfg.W)
    keep = np.nonzero(tw["row_ovf"] == 0)[0]
    ys = O.sparse_ffn_from_twell(tw, L["x"], L["WuT"], L["Wd"], rows=keep)
    yd = O.gated_ffn(L["x"][keep], L["WgT"], L["WuT"], L["Wd"])
    xf = O.bf16_bits_to_f64(L["x"][keep])
    g = np.maximum(z[keep], 0)
    u = xf @ O.bf16_bits_to_f64(L["WuT"]).T
    bound = (np.abs(g * u) @ np.abs(O.bf16_bits_to_f64(L["Wd"]))) * 2.0**-8 + 1e-12
    assert np.all(np.abs(ys - yd) <= bound)
    assert np.abs(ys - yd).max() > 0  # the rounding is visible


def test_hybrid_routes_heavy_tokens_and_combines_branches():
    L = synth.make_layer(HEAVY, seed=0)
    out = O.hybrid_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"], HEAVY.tile, HEAVY.W)
    ovf = out["ovf_rows"]
    assert np.all(np.diff(ovf) > 0)
    heavy = np.nonzero(L["p_t"] >= HEAVY.heavy_lo)[0]
    assert set(heavy.tolist()) <= set(ovf.tolist())  # Binomial tail: a miss is ~1e-12
    assert len(ovf) < len(heavy) + 0.05 * HEAVY.T
    yd = O.gated_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"])
    assert np.array_equal(out["y"][ovf], yd[ovf])
    rms = np.sqrt(np.mean(yd**2))
    assert np.abs(out["y"] - yd).max() <= 1e-2 * rms


# ---------------------------------------------------------------------------
# The generator keeps the gate exact in fp32 under any summation order


@pytest.mark.parametrize("cfg", [synth.CONFIGS["tiny"], MID, HEAVY], ids=lambda c: c.name)
def test_generator_gate_is_order_free_in_fp32(cfg):
    L = synth.make_layer(cfg, seed=0)
    xf = O.bf16_bits_to_f64(L["x"])
    wf = O.bf16_bits_to_f64(L["WgT"])
    d = cfg.d
    e = int(math.floor(math.log2(math.sqrt(d)))) + 5
    assert np.array_equal(np.rint(xf[:, : d - 2] * 8), xf[:, : d - 2] * 8)
    assert np.array_equal(np.rint(wf[:, : d - 2] * 2.0**e), wf[:, : d - 2] * 2.0**e)
    assert np.array_equal(np.rint(xf[:, d - 2:] * 32), xf[:, d - 2:] * 32)
    assert np.array_equal(np.rint(wf[:, d - 2:] * 32), wf[:, d - 2:] * 32)
    assert e + 3 <= 13
    # Cauchy-Schwarz bound on every partial sum of |x_k w_k|
    bound = (np.linalg.norm(xf[:, : d - 2], axis=1).max() * np.linalg.norm(wf[:, : d - 2], axis=1).max()
             + np.abs(xf[:, d - 2]).max() + np.abs(wf[:, d - 1]).max())
    assert bound < 2.0**11
    z64 = O.gate_preactivation(L["x"], L["WgT"])
    z32 = (torch.from_numpy(xf.astype(np.float32)) @ torch.from_numpy(wf.astype(np.float32)).T).numpy()
    assert np.array_equal(z32.astype(np.float64), z64)


def test_generator_density_and_determinism():
    cfg = synth.CONFIGS["tiny"]
    a = synth.make_layer(cfg, seed=0)
    b = synth.make_layer(cfg, seed=0)
    c = synth.make_layer(cfg, seed=1)
    for k in ("x", "WgT", "WuT", "Wd"):
        assert np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])
    z = O.gate_preactivation(a["x"], a["WgT"])
    assert abs((z > 0).mean() - 0.05) < 0.006
    L = synth.make_layer(MID, seed=0)
    z = O.gate_preactivation(L["x"], L["WgT"])
    assert not np.any(z[:, L["dead"]] > 0)
    assert abs((z > 0).mean() - MID.density) < 0.01


# ---------------------------------------------------------------------------
# Tensor-core-up variant: same pattern, hidden values, down projection alone


def test_hidden_pack_keeps_the_gate_pattern_and_stores_h():
    L = synth.make_layer(MID, seed=2)
    x = O.bf16_bits_to_f64(L["x"])
    z = x @ O.bf16_bits_to_f64(L["WgT"]).T
    u = x @ O.bf16_bits_to_f64(L["WuT"]).T
    tg = O.twell_pack(z, MID.tile, MID.W)
    th = O.twell_pack_hidden(z, u, MID.tile, MID.W)
    assert np.array_equal(tg["counts"], th["counts"]) and np.array_equal(tg["idx"], th["idx"])
    assert np.array_equal(tg["row_ovf"], th["row_ovf"])
    t, c = np.nonzero(tg["counts"] > 0)
    t, c = t[:200], c[:200]
    j = tg["idx"][t, c, 0].astype(np.int64)
    want = torch_bf16_bits((z[t, j] * u[t, j]).astype(np.float32))  # z > 0 at stored slots
    assert np.array_equal(th["vals"][t, c, 0], want)


def test_down_only_equals_dense_when_hidden_is_bf16_exact():
    rng = np.random.default_rng(12)
    T, d, f = 16, 4, 256  # |z|, |u| <= 4, so h = z * u is an integer <= 16: exact in bf16
    x = bits_of_exact(rng.integers(-1, 2, size=(T, d)).astype(np.float64))
    WgT = bits_of_exact(rng.integers(-1, 2, size=(f, d)).astype(np.float64))
    WuT = bits_of_exact(rng.integers(-1, 2, size=(f, d)).astype(np.float64))
    Wd = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    xf = O.bf16_bits_to_f64(x)
    z, u = xf @ O.bf16_bits_to_f64(WgT).T, xf @ O.bf16_bits_to_f64(WuT).T
    th = O.twell_pack_hidden(z, u, 128, 128)
    yd = O.gated_ffn(x, WgT, WuT, Wd)
    np.testing.assert_allclose(O.sparse_down_from_twell(th, Wd), yd, rtol=1e-12, atol=1e-12 * np.abs(yd).max())


def test_up_dense_hybrid_within_one_rounding_of_dense():
    L = synth.make_layer(HEAVY, seed=0)
    out = O.hybrid_ffn_up_dense(L["x"], L["WgT"], L["WuT"], L["Wd"], HEAVY.tile, HEAVY.W)
    ref = O.hybrid_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"], HEAVY.tile, HEAVY.W)
    assert np.array_equal(out["ovf_rows"], ref["ovf_rows"])
    x = O.bf16_bits_to_f64(L["x"])
    h = np.maximum(x @ O.bf16_bits_to_f64(L["WgT"]).T, 0) * (x @ O.bf16_bits_to_f64(L["WuT"]).T)
    wd = O.bf16_bits_to_f64(L["Wd"])
    bound = np.abs(h) @ np.abs(wd) * 2.0**-8 + 1e-12
    assert np.all(np.abs(out["y"] - h @ wd) <= bound)


# ---------------------------------------------------------------------------
# Non-gated variant y = ReLU(x W1) W2


def test_relu_ffn_exact_rational_bruteforce():
    rng = np.random.default_rng(21)
    T, d, f = 3, 6, 10
    x = torch_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    W1T = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    W2 = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    F = lambda b: [[Fraction(float(v)) for v in row] for row in O.bf16_bits_to_f64(b)]
    xf, af, bf = F(x), F(W1T), F(W2)
    y = O.relu_ffn(x, W1T, W2)
    for t in range(T):
        for k in range(d):
            acc = Fraction(0)
            for j in range(f):
                zj = sum(xf[t][i] * af[j][i] for i in range(d))
                acc += max(zj, Fraction(0)) * bf[j][k]
            assert abs(y[t, k] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_relu_ffn_permutation_closed_form():
    """Permutation weights: y[pc(j)] = ReLU(x[pa(j)]); a transposed operand
    applies the inverse permutation and fails."""
    rng = np.random.default_rng(22)
    n, T = 32, 4
    pa, pc = rng.permutation(n), rng.permutation(n)
    eye = np.eye(n)
    xv = rng.integers(-40, 40, size=(T, n)) / 8.0
    y = O.relu_ffn(bits_of_exact(xv), bits_of_exact(eye[pa]), bits_of_exact(eye[pc]))
    want = np.zeros((T, n))
    for j in range(n):
        want[:, pc[j]] = np.maximum(xv[:, pa[j]], 0)
    assert np.array_equal(y, want)


def test_relu_ffn_is_the_gated_layer_with_unit_up_projection():
    """The synthetic x carries a constant 1 in its last feature, so an up
    projection that selects it gives u == 1 and the gated layer reduces to the
    non-gated one, exactly."""
    cfg = synth.CONFIGS["tiny"]
    L = synth.make_layer(cfg, seed=4)
    assert np.all(O.bf16_bits_to_f64(L["x"])[:, -1] == 1.0)
    sel = np.zeros((cfg.f, cfg.d))
    sel[:, -1] = 1.0
    assert np.array_equal(O.relu_ffn(L["x"], L["WgT"], L["Wd"]),
                          O.gated_ffn(L["x"], L["WgT"], bits_of_exact(sel), L["Wd"]))


def test_relu_hybrid_exact_when_hidden_is_bf16_exact_and_routes_like_the_gate():
    rng = np.random.default_rng(23)
    T, d, f, W = 40, 8, 384, 8
    # z = (small-integer dot product over 7 features) + x[:, 7] * w1[:, 7]: the
    # last feature is a bias of -4 (sparse rows) or +4 (five dense rows that
    # overflow); every z is a small integer, exact in bf16
    xv = rng.integers(-1, 2, size=(T, d)).astype(np.float64)
    xv[:, 7] = 1.0
    xv[:5, 7] = -1.0
    x = bits_of_exact(xv)
    w1 = rng.integers(-1, 2, size=(f, d)).astype(np.float64)
    w1[:, 7] = -4.0
    W1T = bits_of_exact(w1)
    W2 = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
    out = O.hybrid_relu_ffn(x, W1T, W2, 128, W)
    z = O.gate_preactivation(x, W1T)
    assert np.array_equal(O.bf16_bits_to_f64(O.f64_to_bf16_bits(z)), z)
    assert np.array_equal(out["ovf_rows"], O.route_rows(O.twell_pack(z, 128, W)["counts"], W))
    assert set(range(5)) <= set(out["ovf_rows"].tolist()) and len(out["ovf_rows"]) < T // 2
    keep = np.setdiff1d(np.arange(T), out["ovf_rows"])
    assert out["twell"]["counts"][keep].sum() > 0  # the sparse branch has work
    yd = O.relu_ffn(x, W1T, W2)
    np.testing.assert_allclose(out["y"], yd, rtol=1e-12, atol=1e-12 * np.abs(yd).max())


def test_relu_hybrid_within_one_rounding_of_dense_and_special_cases():
    L = synth.make_layer(HEAVY, seed=1)
    out = O.hybrid_relu_ffn(L["x"], L["WgT"], L["Wd"], HEAVY.tile, HEAVY.W)
    z = O.gate_preactivation(L["x"], L["WgT"])
    g = np.maximum(z, 0)
    w2 = O.bf16_bits_to_f64(L["Wd"])
    bound = g @ np.abs(w2) * 2.0**-8 + 1e-12
    assert np.all(np.abs(out["y"] - g @ w2) <= bound)
    assert np.array_equal(out["y"][out["ovf_rows"]], (g @ w2)[out["ovf_rows"]])
    # all-negative pre-activation: y == 0; one active column: y = z_j W2[j]
    neg = O.bf16_bits_to_f64(L["WgT"]).copy()
    neg[:, -1] = -64.0
    assert not np.any(O.hybrid_relu_ffn(L["x"], bits_of_exact(neg), L["Wd"], HEAVY.tile, HEAVY.W)["y"])
    js = 130
    neg[js, -1] = 64.0
    zj = O.bf16_bits_to_f64(L["x"]) @ neg[js]
    assert np.all(zj > 0)
    got = O.hybrid_relu_ffn(L["x"], bits_of_exact(neg), L["Wd"], HEAVY.tile, HEAVY.W)["y"]
    want = O.bf16_bits_to_f64(O.f64_to_bf16_bits(zj))[:, None] * w2[js][None, :]
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# Dead-column compaction


def test_column_activity_bruteforce():
    rng = np.random.default_rng(31)
    z = rng.integers(-3, 2, size=(7, 300)).astype(np.float64)
    z[:, 5] = 0.0  # zero is not active
    z[3, 6] = 0.5  # one token suffices
    want = np.array([any(z[t, j] > 0 for t in range(z.shape[0])) for j in range(z.shape[1])])
    got = O.column_activity(z)
    assert np.array_equal(got, want)
    assert not got[5] and got[6]


def test_compaction_keeps_the_layer_on_the_profile_batch():
    """Dropping units that are never active on a batch changes nothing on that
    batch: y (gated and non-gated) is the same up to fp64 rounding, and the
    packs agree as sets of (row, original column, value)."""
    cfg = synth.LayerConfig("dead", T=96, d=128, f=1024, tile=128, W=128, density=0.05, sigma=0.5,
                            dead_frac=0.3)
    L = synth.make_layer(cfg, seed=5)
    z = O.gate_preactivation(L["x"], L["WgT"])
    act = O.column_activity(z)
    c = O.compact_layer(L["WgT"], L["WuT"], L["Wd"], act, cfg.tile)
    assert c["f_live"] == int(act.sum()) < cfg.f * 0.8
    assert c["f_c"] % cfg.tile == 0 and c["f_c"] - c["f_live"] < cfg.tile
    assert np.all(np.diff(c["col_map"][:c["f_live"]]) > 0) and np.all(c["col_map"][c["f_live"]:] == -1)
    assert not np.any(c["WgT"][c["f_live"]:]) and not np.any(c["Wd"][c["f_live"]:])
    y0 = O.gated_ffn(L["x"], L["WgT"], L["WuT"], L["Wd"])
    y1 = O.gated_ffn(L["x"], c["WgT"], c["WuT"], c["Wd"])
    np.testing.assert_allclose(y1, y0, rtol=1e-12, atol=1e-12 * np.abs(y0).max())
    r0 = O.relu_ffn(L["x"], L["WgT"], L["Wd"])
    np.testing.assert_allclose(O.relu_ffn(L["x"], c["WgT"], c["Wd"]), r0, rtol=1e-12, atol=1e-12 * np.abs(r0).max())
    zc = O.gate_preactivation(L["x"], c["WgT"])
    assert not np.any(zc[:, c["f_live"]:] > 0)  # padding never activates
    p0 = O.twell_pack(z, cfg.tile, cfg.tile)
    p1 = O.twell_pack(zc, cfg.tile, cfg.tile)

    def pairs(p, cmap):
        out = set()
        T, nT, W = p["idx"].shape
        for t in range(T):
            for ct in range(nT):
                for s in range(min(int(p["counts"][t, ct]), W)):
                    j = int(p["idx"][t, ct, s])
                    out.add((t, int(cmap[j]) if cmap is not None else j, int(p["vals"][t, ct, s])))
        return out

    assert pairs(p1, c["col_map"]) == pairs(p0, None)


def test_compaction_of_a_layer_with_no_dead_units_is_the_identity():
    rng = np.random.default_rng(32)
    f, d = 256, 64
    m = rng.integers(0, 1 << 16, size=(f, d)).astype(np.uint16)
    c = O.compact_layer(m, m, m, np.ones(f, dtype=bool), 128)
    assert c["f_c"] == f and np.array_equal(c["WgT"], m) and np.array_equal(c["col_map"], np.arange(f))
    e = O.compact_layer(m, None, m, np.zeros(f, dtype=bool), 128)
    assert e["f_live"] == 0 and e["f_c"] == 128 and not np.any(e["WgT"]) and "WuT" not in e


# ---------------------------------------------------------------------------
# Backward pass


def _rand_bf16(rng, shape, scale=1.0):
    return torch_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


def test_backward_matches_finite_differences():
    """Central differences of L = <dy, y> in float64, along random directions,
    at a point whose gate pre-activations are far from the ReLU kink."""
    rng = np.random.default_rng(41)
    T, d, f = 4, 6, 9
    x, WgT, WuT, Wd, dy = (_rand_bf16(rng, s) for s in ((T, d), (f, d), (f, d), (f, d), (T, d)))
    F = O.bf16_bits_to_f64
    xv, gv, uv, wv, dyv = F(x), F(WgT), F(WuT), F(Wd), F(dy)
    assert np.abs(xv @ gv.T).min() > 1e-3

    def loss(xv, gv, uv, wv):
        return float(np.sum(dyv * ((np.maximum(xv @ gv.T, 0) * (xv @ uv.T)) @ wv)))

    grads = O.gated_ffn_backward(x, WgT, WuT, Wd, dy)
    eps = 1e-6
    for name, pos in (("dx", 0), ("dWgT", 1), ("dWuT", 2), ("dWd", 3)):
        for _ in range(3):
            args = [xv, gv, uv, wv]
            v = rng.standard_normal(args[pos].shape)
            plus = list(args)
            minus = list(args)
            plus[pos] = args[pos] + eps * v
            minus[pos] = args[pos] - eps * v
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            an = float(np.sum(grads[name] * v))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_exact_rational_bruteforce():
    rng = np.random.default_rng(42)
    T, d, f = 2, 3, 4
    x, WgT, WuT, Wd, dy = (_rand_bf16(rng, s) for s in ((T, d), (f, d), (f, d), (f, d), (T, d)))
    F = lambda b: [[Fraction(float(v)) for v in row] for row in O.bf16_bits_to_f64(b)]
    X, G, U, D, DY = F(x), F(WgT), F(WuT), F(Wd), F(dy)
    got = O.gated_ffn_backward(x, WgT, WuT, Wd, dy)
    dx = [[Fraction(0)] * d for _ in range(T)]
    dG = [[Fraction(0)] * d for _ in range(f)]
    dU = [[Fraction(0)] * d for _ in range(f)]
    dD = [[Fraction(0)] * d for _ in range(f)]
    for t in range(T):
        for j in range(f):
            z = sum(X[t][k] * G[j][k] for k in range(d))
            u = sum(X[t][k] * U[j][k] for k in range(d))
            if z <= 0:
                continue
            dh = sum(DY[t][k] * D[j][k] for k in range(d))
            for k in range(d):
                dx[t][k] += dh * u * G[j][k] + dh * z * U[j][k]
                dG[j][k] += dh * u * X[t][k]
                dU[j][k] += dh * z * X[t][k]
                dD[j][k] += z * u * DY[t][k]
    for name, ref in (("dx", dx), ("dWgT", dG), ("dWuT", dU), ("dWd", dD)):
        r = np.array([[float(v) for v in row] for row in ref])
        np.testing.assert_allclose(got[name], r, rtol=1e-12, atol=1e-12 * max(1.0, np.abs(r).max()))


def test_backward_special_cases():
    L = synth.make_layer(synth.CONFIGS["tiny"], seed=6)
    rng = np.random.default_rng(43)
    dy = _rand_bf16(rng, (64, 128))
    zero = O.gated_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], np.zeros_like(dy))
    assert all(not np.any(zero[k]) for k in ("dx", "dWgT", "dWuT", "dWd"))
    neg = O.bf16_bits_to_f64(L["WgT"]).copy()
    neg[:, -1] = -64.0
    dead = O.gated_ffn_backward(L["x"], bits_of_exact(neg), L["WuT"], L["Wd"], dy)
    assert all(not np.any(dead[k]) for k in ("dx", "dWgT", "dWuT", "dWd"))
    # one active unit j: dWd[j] = sum_t z_j u_j dy_t, other rows zero
    js = 9
    neg[js, -1] = 64.0
    one = O.gated_ffn_backward(L["x"], bits_of_exact(neg), L["WuT"], L["Wd"], dy)
    xf = O.bf16_bits_to_f64(L["x"])
    zj = xf @ neg[js]
    uj = xf @ O.bf16_bits_to_f64(L["WuT"])[js]
    assert np.all(zj > 0)
    np.testing.assert_allclose(one["dWd"][js], (zj * uj) @ O.bf16_bits_to_f64(dy), rtol=1e-12, atol=1e-12)
    assert not np.any(np.delete(one["dWd"], js, axis=0))


def test_hybrid_backward_exact_when_gate_is_bf16_exact():
    rng = np.random.default_rng(44)
    T, d, f, W = 40, 8, 384, 8
    xv = rng.integers(-1, 2, size=(T, d)).astype(np.float64)
    xv[:, 7] = 1.0
    xv[:5, 7] = -1.0  # five dense rows that overflow
    w1 = rng.integers(-1, 2, size=(f, d)).astype(np.float64)
    w1[:, 7] = -4.0
    x, WgT = bits_of_exact(xv), bits_of_exact(w1)
    WuT, Wd, dy = _rand_bf16(rng, (f, d)), _rand_bf16(rng, (f, d)), _rand_bf16(rng, (T, d))
    out = O.hybrid_ffn_backward(x, WgT, WuT, Wd, dy, 128, W)
    assert set(range(5)) <= set(out["ovf_rows"].tolist()) and len(out["ovf_rows"]) < T // 2
    ref = O.gated_ffn_backward(x, WgT, WuT, Wd, dy)
    for k in ("dx", "dWgT", "dWuT", "dWd"):
        np.testing.assert_allclose(out[k], ref[k], rtol=1e-12, atol=1e-12 * np.abs(ref[k]).max())


def test_hybrid_backward_within_one_rounding_of_dense():
    """Sparse rows use the stored bf16 gate g: h = g u and du = dh g move by at
    most 2^-8 relative per term; dz = dh u does not involve g."""
    L = synth.make_layer(HEAVY, seed=2)
    rng = np.random.default_rng(45)
    dy = _rand_bf16(rng, (HEAVY.T, HEAVY.d))
    out = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy, HEAVY.tile, HEAVY.W)
    ref = O.gated_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy)
    F = O.bf16_bits_to_f64
    x, WgT, WuT, Wd, dyv = F(L["x"]), F(L["WgT"]), F(L["WuT"]), F(L["Wd"]), F(dy)
    z = x @ WgT.T
    g = np.maximum(z, 0)
    u = x @ WuT.T
    dh = dyv @ Wd.T
    du = np.abs(dh * g)
    tiny = 1e-12
    assert np.all(np.abs(out["dx"] - ref["dx"]) <= 2.0**-8 * (du @ np.abs(WuT)) + tiny)
    assert np.all(np.abs(out["dWuT"] - ref["dWuT"]) <= 2.0**-8 * (du.T @ np.abs(x)) + tiny)
    assert np.all(np.abs(out["dWd"] - ref["dWd"]) <= 2.0**-8 * (np.abs(g * u).T @ np.abs(dyv)) + tiny)
    np.testing.assert_allclose(out["dWgT"], ref["dWgT"], rtol=1e-10, atol=1e-10 * np.abs(ref["dWgT"]).max())
    assert np.array_equal(out["dx"][out["ovf_rows"]], ref["dx"][out["ovf_rows"]])
    assert np.abs(out["dWd"] - ref["dWd"]).max() > 0  # the rounding is visible


def test_backward_weight_rows_agree_with_the_full_hybrid_backward():
    L = synth.make_layer(HEAVY, seed=3)
    rng = np.random.default_rng(46)
    dy = _rand_bf16(rng, (HEAVY.T, HEAVY.d))
    full = O.hybrid_ffn_backward(L["x"], L["WgT"], L["WuT"], L["Wd"], dy, HEAVY.tile, HEAVY.W)
    assert len(full["ovf_rows"]) > 0
    cols = np.sort(rng.choice(HEAVY.f, size=40, replace=False))
    part = O.hybrid_backward_weight_rows(L["x"], L["WgT"], L["WuT"], L["Wd"], dy, full["ovf_rows"], cols)
    for k in ("dWgT", "dWuT", "dWd"):
        np.testing.assert_allclose(part[k], full[k][cols], rtol=1e-11, atol=1e-11 * np.abs(full[k]).max())


def test_tiny_layers_bruteforce_over_1000_seeds():
    """Tiny layers (T <= 8, d <= 16, f = 256) for seeds 0..999: the gate from
    small-integer x and Wg (exact), the pack against plain loops (bf16 values
    from torch's rounding, computed once per case), the routing predicate, and
    for the rows that fit the sparse step against the dense layer."""
    tile = 128
    for seed in range(1000):
        rng = np.random.default_rng(seed)
        T, d, f = int(rng.integers(1, 9)), int(rng.integers(1, 17)), 256
        W = (1, 2, 8, 16, 128)[seed % 5]
        x = rng.integers(-3, 4, size=(T, d)).astype(np.float64)
        wg = rng.integers(-3, 4, size=(f, d)).astype(np.float64)
        shift = rng.integers(-6, 3)  # moves the density from nearly empty to nearly full
        wg[:, 0] += shift
        z = x @ wg.T
        tw = O.twell_pack(z, tile, W)
        zb = torch_bf16_bits(z.astype(np.float32)).astype(np.int64)
        for t in range(T):
            for c in range(f // tile):
                n = 0
                for k in range(tile):
                    j = c * tile + k
                    if z[t, j] > 0:
                        if n < W:
                            assert tw["idx"][t, c, n] == j and int(tw["vals"][t, c, n]) == zb[t, j], (seed, t, j)
                        n += 1
                assert tw["counts"][t, c] == n, (seed, t, c)
        assert np.array_equal(tw["row_ovf"], (tw["counts"] > W).any(axis=1).astype(np.uint8))
        keep = np.nonzero(tw["row_ovf"] == 0)[0]
        if keep.size and seed % 10 == 0:  # the sparse step on a tenth of the cases
            xb, wgb = bits_of_exact(x), bits_of_exact(wg)
            wu = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
            wd = torch_bf16_bits(rng.standard_normal((f, d)).astype(np.float32))
            ys = O.sparse_ffn_from_twell(tw, xb, wu, wd, rows=keep)
            yd = O.gated_ffn(xb[keep], wgb, wu, wd)
            np.testing.assert_allclose(ys, yd, rtol=1e-12, atol=1e-12 * max(1.0, np.abs(yd).max()))
