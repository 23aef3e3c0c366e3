"""Shared helpers of the GPU parity tests: upload synthetic layers, run the
library through its C ABI, and compare with the oracle."""

from __future__ import annotations

import numpy as np
import torch

from activation_sparse_gated_gemm_b200 import twell as tl
from oracle import twell_oracle as O

Y_RTOL = 2e-2  # max|y - y_ref| <= 2e-2 * rms(y_ref), y_ref = the oracle's result of the method


def upload(L: dict, device="cuda") -> dict:
    return {k: tl.to_device_bf16(L[k], device) for k in ("x", "WgT", "WuT", "Wd")}


def run_pack(dev: dict, W: int):
    T, d = dev["x"].shape
    f = dev["WgT"].shape[0]
    tw = tl.Twell(T, f, W)
    st = tl.new_status()
    tl.gate_pack(dev["x"], dev["WgT"], tw, st)
    return tw, tl.status_get(st)


def twell_to_host(tw: tl.Twell) -> dict:
    return {
        "counts": tw.counts.cpu().numpy(),
        "idx": tw.idx.cpu().numpy(),
        "vals": tl.bf16_bits(tw.vals),
        "row_ovf": tw.row_ovf.cpu().numpy(),
    }


def assert_twell_equal(got: dict, want: dict, W: int, rows=None) -> None:
    """Bit-exact comparison of what TwELL defines: counts, overflow flags and
    the first min(count, W) slots of every (row, tile). Padding is not part
    of the format on the device and is not compared."""
    if rows is None:
        rows = np.arange(want["counts"].shape[0])
    gc, wc = got["counts"][rows], want["counts"]
    assert np.array_equal(gc, wc), f"counts differ at {np.argwhere(gc != wc)[:5].tolist()}"
    assert np.array_equal(got["row_ovf"][rows], want["row_ovf"])
    n = np.minimum(wc.astype(np.int64), W)
    live = np.arange(W)[None, None, :] < n[:, :, None]
    gi, wi = got["idx"][rows], want["idx"]
    gv, wv = got["vals"][rows], want["vals"]
    bad = live & ((gi != wi) | (gv != wv))
    assert not bad.any(), f"slots differ at {np.argwhere(bad)[:5].tolist()}"


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "y") -> float:
    rms = float(np.sqrt(np.mean(y_ref**2)))
    err = float(np.abs(y_gpu - y_ref).max())
    assert err <= Y_RTOL * rms, f"{what}: max|err| {err:.3e} > {Y_RTOL} * rms {rms:.3e}"
    return err / rms


def y_to_f64(y: torch.Tensor) -> np.ndarray:
    return y.detach().double().cpu().numpy()


def oracle_pack_rows(L: dict, rows, tile: int, W: int) -> dict:
    z = O.gate_preactivation(L["x"][rows], L["WgT"])
    return O.twell_pack(z, tile, W)


def assert_dense_bf16_hidden_bound(y_gpu: np.ndarray, L: dict) -> None:
    """A dense layer that stores h once as bf16 has |y - y_exact| <= 2^-8 *
    sum_j |h_j Wd[j, k]| (one nearest rounding of each h_j to 8 significant
    bits); 2^-7 leaves room for the fp32 sums."""
    x = O.bf16_bits_to_f64(L["x"])
    h = np.maximum(x @ O.bf16_bits_to_f64(L["WgT"]).T, 0) * (x @ O.bf16_bits_to_f64(L["WuT"]).T)
    wd = O.bf16_bits_to_f64(L["Wd"])
    y = h @ wd
    bound = np.abs(h) @ np.abs(wd) * 2.0**-7 + 1e-6
    assert np.all(np.abs(y_gpu - y) <= bound), float((np.abs(y_gpu - y) / bound).max())


def assert_within_stored_value_bound(y_gpu: np.ndarray, L: dict, rows, stored: str = "g") -> None:
    """Against the exact dense layer: the method stores one bf16 value per
    active unit (g, or h for the tensor-core up variant), so each term
    h_j Wd[j, k] moves by at most 2^-8 relative; 2^-7 leaves room for the fp32
    sums. Checked on non-overflow rows."""
    x = O.bf16_bits_to_f64(L["x"][rows])
    h = np.maximum(x @ O.bf16_bits_to_f64(L["WgT"]).T, 0) * (x @ O.bf16_bits_to_f64(L["WuT"]).T)
    wd = O.bf16_bits_to_f64(L["Wd"])
    bound = np.abs(h) @ np.abs(wd) * 2.0**-7 + 1e-6
    err = np.abs(y_gpu - h @ wd)
    assert np.all(err <= bound), float((err / bound).max())
