"""Every pipeline wait in the library is bounded. This checks the mechanism on
the GPU without faulting it: a warp waits, through the library's own wait
helper, on an mbarrier phase that nothing completes, with a 20 ms limit. The
kernel must give up, report TWELL_ERR_TIMEOUT through the status word and
return, leaving the context usable."""

import ctypes
import os
import subprocess

import pytest
import torch

from activation_sparse_gated_gemm_b200 import build as tb
from activation_sparse_gated_gemm_b200 import twell as tl

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("probe") / "bounded_wait_probe.so")
    cmd = [tb._nvcc(), *tb.ARCH_FLAGS, "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           f"-I{tb.CSRC}", "-o", out, os.path.join(HERE, "cuda", "bounded_wait_probe.cu")]
    subprocess.run(cmd, check=True, capture_output=True)
    lib = ctypes.CDLL(out)
    lib.launch_bounded_wait_probe.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p]
    lib.launch_bounded_wait_probe.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("limit_ms", [20, 50])
def test_unsatisfied_wait_times_out_and_reports(probe, limit_ms):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    rc = probe.launch_bounded_wait_probe(ctypes.c_void_p(status.data_ptr()), limit_ms * 1_000_000,
                                         ctypes.c_void_p(waited.data_ptr()))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == tl.TWELL_ERR_TIMEOUT
    w = int(waited.item())
    assert limit_ms * 1_000_000 <= w < limit_ms * 1_000_000 + 500_000_000
    # the context still runs work afterwards
    assert float((torch.ones(4, device="cuda") * 3).sum().item()) == 12.0
