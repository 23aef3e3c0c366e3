"""The hybrid forward that needs no workspace from its caller.

Some users of this library cannot allocate device memory for a workspace: a
framework that hands out every byte of device memory from its own pool, a
serving loop that must never reach the allocator, or a plugin whose host gives
it only its inputs and outputs. twell_ffn_hybrid_forward_noalloc serves them
from a scratch array compiled into the library. These tests call it through
the C ABI twice in a row and check each result against the ordinary entry
point that takes a workspace -- at a batch that takes the large-batch path and
at two small batches, where the scratch also holds the split-K gate
accumulator -- and check that sizes beyond the built-in scratch are refused
before anything is launched.

The pack and the routing must be bit-identical to the workspace entry point's.
y is compared within 1e-5 of its rms (2000 times tighter than the method's
tolerance): both calls run the same kernels on the same inputs, but where the
GPU cannot be filled otherwise they add split partial sums into y with
atomics, whose order (and so the last bits of an fp32 sum) varies from run to
run. A scratch slip -- stale or foreign hidden activations, a missing zeroing
-- moves y by a sizeable fraction of its rms and fails this.

This file is named to be collected last."""

import numpy as np
import pytest
import torch

from activation_sparse_gated_gemm_b200 import synth
from activation_sparse_gated_gemm_b200 import twell as tl
from tests.gpu_helpers import assert_twell_equal, twell_to_host, upload

pytestmark = pytest.mark.gpu

LC = synth.LayerConfig
CASES = [
    LC("noalloc", T=700, d=256, f=2304, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.08, heavy_lo=0.25,
       heavy_hi=0.40),
    LC("noalloc_small", T=64, d=256, f=2304, tile=128, W=24, density=0.012, sigma=0.5, heavy_frac=0.08,
       heavy_lo=0.25, heavy_hi=0.40),
    LC("noalloc_one", T=1, d=256, f=2304, tile=128, W=24, density=0.012, heavy_frac=1.0, heavy_lo=0.25,
       heavy_hi=0.40),
]
Y_TIGHT = 1e-5


def _hybrid_outputs(cfg):
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ovf_rows = torch.full((cfg.T,), -1, dtype=torch.int32, device="cuda")
    n_ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    return y, ovf_rows, n_ovf


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(cfg):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    tl.load()
    assert tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f) <= tl.NOALLOC_SCRATCH_BYTES
    dev = upload(synth.make_layer(cfg, seed=0))

    tw_ref = tl.Twell(cfg.T, cfg.f, cfg.W)
    y_ref, rows_ref, n_ref = _hybrid_outputs(cfg)
    ws = torch.empty(tl.hybrid_workspace_bytes(cfg.T, cfg.d, cfg.f), dtype=torch.uint8, device="cuda")
    st = tl.new_status()
    tl.ffn_hybrid_forward(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw_ref, y_ref, rows_ref, n_ref, ws, st)
    assert tl.status_get(st) == 0
    n = int(n_ref.item())
    assert n > 0  # the heavy rows exercise the scratch-using dense branch
    want = twell_to_host(tw_ref)
    rms = float(y_ref.pow(2).mean().sqrt())

    for call in range(2):
        tw = tl.Twell(cfg.T, cfg.f, cfg.W)
        y, rows, n_ovf = _hybrid_outputs(cfg)
        st = tl.new_status()
        tl.ffn_hybrid_forward_noalloc(dev["x"], dev["WgT"], dev["WuT"], dev["Wd"], tw, y, rows, n_ovf, st)
        assert tl.status_get(st) == 0, f"call {call}"
        assert int(n_ovf.item()) == n
        assert torch.equal(rows[:n], rows_ref[:n])
        assert_twell_equal(twell_to_host(tw), want, cfg.W)
        assert torch.isfinite(y).all()
        err = float((y - y_ref).abs().max())
        assert err <= Y_TIGHT * rms, f"call {call}: max|y - y_ref| {err:.3e} > {Y_TIGHT} * rms {rms:.3e}"


def test_noalloc_refuses_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    T, d, f, W = 4096, 1536, 4096, 32
    assert tl.hybrid_workspace_bytes(T, d, f) > tl.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((f, d), dtype=torch.bfloat16, device="cuda")
    tw = tl.Twell(T, f, W)
    y, rows, n_ovf = _hybrid_outputs(LC("big", T=T, d=d, f=f, tile=128, W=W, density=0.05))
    st = tl.new_status()
    with pytest.raises(tl.TwellError) as err:
        tl.ffn_hybrid_forward_noalloc(x, w, w, w, tw, y, rows, n_ovf, st)
    assert err.value.status == tl.TWELL_ERR_WORKSPACE
    assert torch.isnan(y).all()  # nothing ran
    assert np.all(rows.cpu().numpy() == -1)
