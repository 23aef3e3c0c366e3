"""Canary guards: every output buffer of the main entry points sits inside a
larger allocation whose margins hold a sentinel bit pattern; after each call
the margins must be unchanged (no kernel writes outside its outputs)."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from tests.gpu_helpers import upload
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

PAD = 64  # elements of margin on each side (keeps 16-byte alignment for every dtype used)
CASES = [c for c in SMALL if c.name in ("mid", "odd", "heavy", "one_row")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()


class Guarded:
    """A tensor of `shape` carved from the middle of a larger one whose margins
    are filled with a sentinel byte pattern."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        self.full = torch.empty(n + 2 * PAD, dtype=dtype, device="cuda")
        raw = self.full.view(torch.uint8)
        raw.fill_(0xA5)
        self.t = self.full[PAD:PAD + n].view(*shape)
        self.before = raw.clone()

    def check(self, name):
        raw = self.full.view(torch.uint8)
        es = self.full.element_size()
        head, tail = PAD * es, raw.numel() - PAD * es
        assert torch.equal(raw[:head], self.before[:head]), f"{name}: write below the buffer"
        assert torch.equal(raw[tail:], self.before[tail:]), f"{name}: write past the buffer"


def guarded_twell(T, f, W):
    nT = f // 128
    g = {"counts": Guarded((T, nT), torch.int16), "idx": Guarded((T, nT, W), torch.int16),
         "vals": Guarded((T, nT, W), torch.bfloat16), "row_ovf": Guarded((T,), torch.uint8)}
    tw = tl.Twell(1, f, W)  # replaced below by the guarded views
    tw.T = T
    for k, v in g.items():
        setattr(tw, k, v.t)
    tw.desc = tl.twell_t(tw.counts.data_ptr(), tw.idx.data_ptr(), tw.vals.data_ptr(), tw.row_ovf.data_ptr(),
                         T, f, 128, W)
    return tw, g


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_forward_backward_and_unpack_stay_inside_their_outputs(cfg):
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw, gtw = guarded_twell(T, f, W)
    y = Guarded((T, d), torch.float32)
    ovf_rows = Guarded((T,), torch.int32)
    n_ovf = Guarded((1,), torch.int32)
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    for fwd in (tl.ffn_hybrid_forward, tl.ffn_hybrid_forward_tc_up):
        fwd(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y.t, ovf_rows.t, n_ovf.t, ws, st)
        assert tl.status_get(st) == 0
        for k, v in list(gtw.items()) + [("y", y), ("ovf_rows", ovf_rows), ("n_ovf", n_ovf)]:
            v.check(f"{fwd.__name__}: {k}")
    tl.relu_ffn_hybrid_forward(dev["x"], dev["WgT"], dev["Wd"], tw, y.t, ovf_rows.t, n_ovf.t, ws, st)
    assert tl.status_get(st) == 0
    y.check("relu forward: y")
    # backward from the gate form's pack
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y.t, ovf_rows.t, n_ovf.t, ws, st)
    dy = tl.to_device_bf16(synth.make_dy(T, d, 0))
    g = {k: Guarded((T if k == "dx" else f, d), torch.float32) for k in ("dx", "dWgT", "dWuT", "dWd")}
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device="cuda")
    tl.ffn_hybrid_backward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], dy, tw, ovf_rows.t, n_ovf.t, g["dx"].t,
                           g["dWgT"].t, g["dWuT"].t, g["dWd"].t, wsb, st)
    assert tl.status_get(st) == 0
    for k, v in g.items():
        v.check(f"backward: {k}")
    dense = Guarded((T, f), torch.bfloat16)
    tl.unpack(tw, dense.t, st)
    assert tl.status_get(st) == 0
    dense.check("unpack")


def test_compaction_stays_inside_its_outputs():
    cfg = SMALL[1]
    L = synth.make_layer(cfg, seed=0)
    dev = upload(L)
    f, d = cfg.f, cfg.d
    st = tl.new_status()
    bits = Guarded((f // 32,), torch.int32)
    col_map = Guarded((f,), torch.int32)
    f_live = Guarded((1,), torch.int32)
    tl.column_activity(dev["x"], dev["WgT"], bits.t, False, st)
    tl.compact_columns(bits.t, f, col_map.t, f_live.t)
    out = Guarded((f - 128, d), torch.bfloat16)
    tl.gather_rows(dev["WgT"], col_map.t, f_live.t, out.t, st)
    assert tl.status_get(st) == 0
    for k, v in (("bits", bits), ("col_map", col_map), ("f_live", f_live), ("rows", out)):
        v.check(k)
