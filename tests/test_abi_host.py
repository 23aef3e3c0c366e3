"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, and rejects bad arguments synchronously
before touching the device. No call here launches anything."""

import ctypes
import os
import re

import pytest

from activation_sparse_gated_gemm_b200 import build as tb
from activation_sparse_gated_gemm_b200 import twell as tl

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "twell.h")

FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails its checks first
MIS = 0x10008   # misaligned


@pytest.fixture(scope="module")
def lib():
    tb.build()
    return tl.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(twell_[a-z_]+)\s*\(", text)))


def test_header_and_library_agree(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(tl.EXPORTED)
    assert lib.twell_version().decode().startswith("twell-b200")


def tw_desc(T=64, f=512, W=16, tile=128, ptr=FAKE):
    return tl.twell_t(ptr, ptr, ptr, ptr, T, f, tile, W)


def call_pack(lib, T=64, d=128, f=512, tw=None, x=FAKE, w=FAKE, st=FAKE):
    tw = tw or tw_desc(T, f)
    return lib.twell_gate_pack(x, w, T, d, f, ctypes.byref(tw), st, None)


def test_shape_errors(lib):
    assert call_pack(lib, T=-1, tw=tw_desc(T=-1)) == tl.TWELL_ERR_SHAPE
    assert call_pack(lib, d=100) == tl.TWELL_ERR_SHAPE        # d % 64
    assert call_pack(lib, d=8192) == tl.TWELL_ERR_SHAPE       # d > 4096
    assert call_pack(lib, f=500, tw=tw_desc(f=500)) == tl.TWELL_ERR_SHAPE
    assert call_pack(lib, f=32768, tw=tw_desc(f=32768)) == tl.TWELL_ERR_SHAPE
    assert call_pack(lib, tw=tw_desc(T=65)) == tl.TWELL_ERR_SHAPE    # descriptor mismatch
    assert call_pack(lib, tw=tw_desc(W=12)) == tl.TWELL_ERR_SHAPE    # W % 8
    assert call_pack(lib, tw=tw_desc(W=136)) == tl.TWELL_ERR_SHAPE   # W > 128
    assert call_pack(lib, tw=tw_desc(tile=64)) == tl.TWELL_ERR_SHAPE


def test_null_and_alignment_errors(lib):
    assert call_pack(lib, x=None) == tl.TWELL_ERR_NULL
    assert call_pack(lib, st=None) == tl.TWELL_ERR_NULL
    assert lib.twell_gate_pack(FAKE, FAKE, 64, 128, 512, None, FAKE, None) == tl.TWELL_ERR_NULL
    assert call_pack(lib, x=MIS) == tl.TWELL_ERR_ALIGN
    assert call_pack(lib, tw=tw_desc(ptr=MIS)) == tl.TWELL_ERR_ALIGN
    assert call_pack(lib, tw=tw_desc(ptr=0)) == tl.TWELL_ERR_NULL


def test_zero_tokens_returns_without_launching(lib):
    tw = tw_desc(T=0)
    assert lib.twell_gate_pack(None, None, 0, 128, 512, ctypes.byref(tw), None, None) == tl.TWELL_OK
    assert lib.twell_ffn_forward(None, None, None, None, 0, 128, 512, ctypes.byref(tw), None, None,
                                 None) == tl.TWELL_OK


def test_workspace_queries_and_errors(lib):
    T, d, f = 1000, 1536, 4096
    hyb = lib.twell_hybrid_workspace_bytes(T, d, f)
    den = lib.twell_dense_workspace_bytes(T, d, f)
    assert hyb >= T * (d + f) * 2 and hyb % 256 == 0
    assert den >= T * f * 2 and den % 256 == 0
    assert lib.twell_hybrid_workspace_bytes(0, d, f) == 0
    tw = tw_desc(T, f, 32)
    r = lib.twell_ffn_hybrid_forward(FAKE, FAKE, FAKE, FAKE, T, d, f, ctypes.byref(tw), FAKE, FAKE, FAKE,
                                     FAKE, hyb - 1, FAKE, None)
    assert r == tl.TWELL_ERR_WORKSPACE
    r = lib.twell_dense_ffn_forward(FAKE, FAKE, FAKE, FAKE, T, d, f, FAKE, None, den, FAKE, None)
    assert r == tl.TWELL_ERR_WORKSPACE
    r = lib.twell_dense_rows_forward(FAKE, FAKE, FAKE, FAKE, T, d, f, FAKE, FAKE, FAKE, MIS, hyb, FAKE, None)
    assert r == tl.TWELL_ERR_ALIGN


def test_status_strings(lib):
    for code in (0, 1, 2, 3, 4, 5, 6, 16, 17, 18):
        s = tl.status_str(code)
        assert s and s != "unknown status"
    assert tl.status_str(99) == "unknown status"


def test_compaction_argument_errors(lib):
    # shapes are checked before anything else
    assert lib.twell_column_activity(FAKE, FAKE, 64, 100, 512, FAKE, 0, FAKE, None) == tl.TWELL_ERR_SHAPE
    assert lib.twell_compact_columns(FAKE, 500, FAKE, FAKE, None) == tl.TWELL_ERR_SHAPE
    assert lib.twell_compact_columns(FAKE, 32768, FAKE, FAKE, None) == tl.TWELL_ERR_SHAPE
    assert lib.twell_gather_rows(FAKE, 512, 128, FAKE, FAKE, 513, FAKE, FAKE, None) == tl.TWELL_ERR_SHAPE
    assert lib.twell_gather_rows(FAKE, 512, 128, FAKE, FAKE, 0, FAKE, FAKE, None) == tl.TWELL_ERR_SHAPE
    assert lib.twell_gather_rows(FAKE, 512, 96, FAKE, FAKE, 128, FAKE, FAKE, None) == tl.TWELL_ERR_SHAPE
    # then pointers
    assert lib.twell_column_activity(FAKE, FAKE, 64, 128, 512, None, 0, FAKE, None) == tl.TWELL_ERR_NULL
    assert lib.twell_compact_columns(FAKE, 512, None, FAKE, None) == tl.TWELL_ERR_NULL
    assert lib.twell_gather_rows(FAKE, 512, 128, MIS, FAKE, 128, FAKE, FAKE, None) == tl.TWELL_ERR_ALIGN


def test_backward_argument_errors(lib):
    tw = tw_desc()
    bw = lib.twell_ffn_hybrid_backward
    args = dict(x=FAKE, g=FAKE, u=FAKE, d=FAKE, dy=FAKE, T=64, dm=128, f=512, ovf=FAKE, n=FAKE, dx=FAKE,
                a=FAKE, b=FAKE, c=FAKE, ws=FAKE, wsb=1 << 30, st=FAKE)

    def call(**kw):
        a = dict(args, **kw)
        return bw(a["x"], a["g"], a["u"], a["d"], a["dy"], a["T"], a["dm"], a["f"], ctypes.byref(tw), a["ovf"], a["n"],
                  a["dx"], a["a"], a["b"], a["c"], a["ws"], a["wsb"], a["st"], None)

    assert call(dm=100) == tl.TWELL_ERR_SHAPE
    assert call(f=500) == tl.TWELL_ERR_SHAPE
    assert call(dy=None) == tl.TWELL_ERR_NULL
    assert call(a=None) == tl.TWELL_ERR_NULL
    assert call(dx=MIS) == tl.TWELL_ERR_ALIGN
    assert call(ws=None) == tl.TWELL_ERR_WORKSPACE
    assert call(wsb=16) == tl.TWELL_ERR_WORKSPACE
    need = lib.twell_backward_workspace_bytes(64, 128, 512, 16)
    assert need > 0 and lib.twell_backward_workspace_bytes(0, 128, 512, 16) == 0
    assert lib.twell_dense_backward_workspace_bytes(64, 128, 512) > 0
    assert lib.twell_dense_ffn_backward(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 128, 512, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                        FAKE, None) == tl.TWELL_ERR_WORKSPACE
    assert lib.twell_relu_ffn_hybrid_forward(FAKE, FAKE, None, 64, 128, 512, ctypes.byref(tw), FAKE, FAKE, FAKE, FAKE,
                                             1 << 30, FAKE, None) == tl.TWELL_ERR_NULL


def test_union_down_argument_errors_and_workspace(lib):
    T, d, f, W = 1000, 2304, 9216, 24
    need = lib.twell_sparse_down_union_workspace_bytes(T, d, f)
    num_m = (T + 127) // 128
    # the tiles' hidden-value blocks, their union lists and K block counts
    assert need >= num_m * 128 * f * 2 + num_m * f * 4 + num_m * 4 and need % 256 == 0
    assert need <= num_m * 128 * f * 2 + num_m * f * 4 + num_m * 4 + 3 * 256
    assert lib.twell_sparse_down_union_workspace_bytes(0, d, f) == 0
    tw = tw_desc(T, f, W)
    un = lib.twell_sparse_down_union

    def call(d_=d, y=FAKE, ws=FAKE, wsb=need, desc=tw):
        return un(FAKE, T, d_, f, ctypes.byref(desc), 1, y, ws, wsb, FAKE, None)

    assert call(d_=100) == tl.TWELL_ERR_SHAPE
    assert call(desc=tw_desc(T + 1, f, W)) == tl.TWELL_ERR_SHAPE
    assert call(y=None) == tl.TWELL_ERR_NULL
    assert call(ws=None) == tl.TWELL_ERR_WORKSPACE
    assert call(wsb=need - 1) == tl.TWELL_ERR_WORKSPACE
    assert call(ws=MIS) == tl.TWELL_ERR_ALIGN
    z = tw_desc(0, f, W)
    assert un(None, 0, d, f, ctypes.byref(z), 1, None, None, 0, None, None) == tl.TWELL_OK
    # the form query answers 0 for invalid shapes and when no device is current
    assert lib.twell_hybrid_down_is_union(T, 100, f, 1 << 40) == 0
    assert lib.twell_hybrid_down_is_union(0, d, f, 1 << 40) == 0
