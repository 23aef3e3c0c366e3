"""ctypes binding of libtwell.so (include/twell.h). Argument marshalling only:
torch supplies device memory and the stream, every step runs in the library's
CUDA kernels. Loading fails loudly when the library is missing; there is no
fallback path.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtwell.so")

TWELL_OK = 0
TWELL_ERR_NULL = 1
TWELL_ERR_SHAPE = 2
TWELL_ERR_ALIGN = 3
TWELL_ERR_WORKSPACE = 4
TWELL_ERR_CUDA = 5
TWELL_ERR_DEVICE = 6
TWELL_ERR_OVERFLOW = 16
TWELL_ERR_INDEX = 17
TWELL_ERR_TIMEOUT = 18

EXPORTED = (
    "twell_gate_pack", "twell_sparse_ffn", "twell_ffn_forward", "twell_route",
    "twell_hybrid_workspace_bytes", "twell_dense_rows_forward", "twell_ffn_hybrid_forward", "twell_dense_workspace_bytes",
    "twell_dense_ffn_forward", "twell_unpack", "twell_status_reset", "twell_status_get",
    "twell_status_str", "twell_version", "twell_ffn_hybrid_forward_noalloc",
    "twell_gate_up_pack", "twell_sparse_down", "twell_ffn_hybrid_forward_tc_up",
    "twell_relu_ffn_hybrid_forward", "twell_relu_dense_rows_forward", "twell_relu_dense_ffn_forward",
    "twell_column_activity", "twell_compact_columns", "twell_gather_rows",
    "twell_backward_workspace_bytes", "twell_ffn_hybrid_backward", "twell_ffn_hybrid_backward_dx",
    "twell_ffn_hybrid_backward_dw", "twell_dense_backward_workspace_bytes", "twell_dense_ffn_backward",
    "twell_ffn_hybrid_backward_dw_tc", "twell_ffn_hybrid_backward_dx_tc", "twell_sparse_down_union",
    "twell_sparse_down_union_workspace_bytes", "twell_hybrid_down_is_union",
)
NOALLOC_SCRATCH_BYTES = 32 << 20


class TwellError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class twell_t(ctypes.Structure):
    _fields_ = [
        ("counts", ctypes.c_void_p),
        ("idx", ctypes.c_void_p),
        ("vals", ctypes.c_void_p),
        ("row_ovf", ctypes.c_void_p),
        ("T", ctypes.c_int32),
        ("f", ctypes.c_int32),
        ("tile", ctypes.c_int32),
        ("W", ctypes.c_int32),
    ]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m activation_sparse_gated_gemm_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    tw = ctypes.POINTER(twell_t)
    sig = {
        "twell_gate_pack": ([vp, vp, i32, i32, i32, tw, vp, vp], i32),
        "twell_sparse_ffn": ([vp, vp, vp, i32, i32, i32, tw, i32, vp, vp, vp], i32),
        "twell_ffn_forward": ([vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp], i32),
        "twell_route": ([tw, vp, vp, vp], i32),
        "twell_gate_up_pack": ([vp, vp, vp, i32, i32, i32, tw, vp, vp], i32),
        "twell_sparse_down": ([vp, i32, i32, i32, tw, i32, vp, vp, vp], i32),
        "twell_sparse_down_union": ([vp, i32, i32, i32, tw, i32, vp, vp, sz, vp, vp], i32),
        "twell_sparse_down_union_workspace_bytes": ([i32, i32, i32], sz),
        "twell_hybrid_down_is_union": ([i32, i32, i32, sz], i32),
        "twell_ffn_hybrid_forward_tc_up": ([vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_hybrid_workspace_bytes": ([i32, i32, i32], sz),
        "twell_dense_rows_forward": ([vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_ffn_hybrid_forward": ([vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_dense_workspace_bytes": ([i32, i32, i32], sz),
        "twell_dense_ffn_forward": ([vp, vp, vp, vp, i32, i32, i32, vp, vp, sz, vp, vp], i32),
        "twell_relu_ffn_hybrid_forward": ([vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_relu_dense_rows_forward": ([vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_relu_dense_ffn_forward": ([vp, vp, vp, i32, i32, i32, vp, vp, sz, vp, vp], i32),
        "twell_backward_workspace_bytes": ([i32, i32, i32, i32], sz),
        "twell_ffn_hybrid_backward": ([vp, vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp],
                                      i32),
        "twell_ffn_hybrid_backward_dx": ([vp, vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_ffn_hybrid_backward_dx_tc": ([vp, vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, sz, vp, vp],
                                            i32),
        "twell_ffn_hybrid_backward_dw": ([vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, vp, sz, vp], i32),
        "twell_ffn_hybrid_backward_dw_tc": ([vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, vp, sz, vp], i32),
        "twell_dense_backward_workspace_bytes": ([i32, i32, i32], sz),
        "twell_dense_ffn_backward": ([vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp], i32),
        "twell_column_activity": ([vp, vp, i32, i32, i32, vp, i32, vp, vp], i32),
        "twell_compact_columns": ([vp, i32, vp, vp, vp], i32),
        "twell_gather_rows": ([vp, i32, i32, vp, vp, i32, vp, vp, vp], i32),
        "twell_unpack": ([tw, vp, vp, vp], i32),
        "twell_ffn_hybrid_forward_noalloc": ([vp, vp, vp, vp, i32, i32, i32, tw, vp, vp, vp, vp, vp], i32),
        "twell_status_reset": ([vp, vp], i32),
        "twell_status_get": ([vp, vp, ctypes.POINTER(ctypes.c_int32)], i32),
        "twell_status_str": ([i32], ctypes.c_char_p),
        "twell_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_str(status: int) -> str:
    return load().twell_status_str(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != TWELL_OK:
        raise TwellError(fn, status, status_str(status))


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(name: str, t: torch.Tensor, shape: tuple, dtype) -> None:
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of shape {shape}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _bf16(name: str, t: torch.Tensor, shape: tuple) -> None:
    if name == "y":
        _dev(name, t, shape, torch.float32)
    else:
        _dev(name, t, shape, torch.bfloat16)


class Twell:
    """Device buffers of one TwELL-packed gate activation (see twell.h)."""

    def __init__(self, T: int, f: int, W: int, device="cuda", tile: int = 128):
        nT = f // tile
        self.T, self.f, self.W, self.tile, self.nT = T, f, W, tile, nT
        self.counts = torch.empty((T, nT), dtype=torch.int16, device=device)
        self.idx = torch.empty((T, nT, W), dtype=torch.int16, device=device)
        self.vals = torch.empty((T, nT, W), dtype=torch.bfloat16, device=device)
        self.row_ovf = torch.empty((T,), dtype=torch.uint8, device=device)
        self.desc = twell_t(self.counts.data_ptr(), self.idx.data_ptr(), self.vals.data_ptr(),
                            self.row_ovf.data_ptr(), T, f, tile, W)

    def ref(self):
        return ctypes.byref(self.desc)


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def status_reset(dev_status: torch.Tensor, stream=None) -> None:
    _check("twell_status_reset", load().twell_status_reset(_ptr(dev_status), _stream(stream)))


def status_get(dev_status: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("twell_status_get", load().twell_status_get(_ptr(dev_status), _stream(stream), ctypes.byref(out)))
    return int(out.value)


def gate_pack(x, WgT, tw: Twell, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    _bf16("x", x, (T, d))
    _bf16("WgT", WgT, (f, d))
    _check("twell_gate_pack", load().twell_gate_pack(_ptr(x), _ptr(WgT), T, d, f, tw.ref(),
                                                     _ptr(dev_status), _stream(stream)))


def sparse_ffn(x, WuT, Wd, tw: Twell, y, skip_overflow_rows: bool, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WuT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)), ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_sparse_ffn", load().twell_sparse_ffn(_ptr(x), _ptr(WuT), _ptr(Wd), T, d, f, tw.ref(),
                                                       int(bool(skip_overflow_rows)), _ptr(y),
                                                       _ptr(dev_status), _stream(stream)))


def ffn_forward(x, WgT, WuT, Wd, tw: Twell, y, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_ffn_forward", load().twell_ffn_forward(_ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f,
                                                         tw.ref(), _ptr(y), _ptr(dev_status),
                                                         _stream(stream)))


def gate_up_pack(x, WgT, WuT, tw: Twell, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d))):
        _bf16(n, t, s)
    _check("twell_gate_up_pack", load().twell_gate_up_pack(_ptr(x), _ptr(WgT), _ptr(WuT), T, d, f, tw.ref(),
                                                           _ptr(dev_status), _stream(stream)))


def sparse_down(Wd, tw: Twell, y, skip_overflow_rows: bool, dev_status, stream=None) -> None:
    f, d = Wd.shape
    T = tw.T
    _bf16("Wd", Wd, (f, d))
    _bf16("y", y, (T, d))
    _check("twell_sparse_down", load().twell_sparse_down(_ptr(Wd), T, d, f, tw.ref(), int(bool(skip_overflow_rows)),
                                                         _ptr(y), _ptr(dev_status), _stream(stream)))


def sparse_down_union(Wd, tw: Twell, y, skip_overflow_rows: bool, workspace, dev_status, stream=None) -> None:
    """The down projection per 128-row tile over the tile's union of stored
    units, on the tensor cores; workspace of sparse_down_union_workspace_bytes(T, d, f)."""
    f, d = Wd.shape
    T = tw.T
    _bf16("Wd", Wd, (f, d))
    _bf16("y", y, (T, d))
    _check("twell_sparse_down_union", load().twell_sparse_down_union(
        _ptr(Wd), T, d, f, tw.ref(), int(bool(skip_overflow_rows)), _ptr(y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def sparse_down_union_workspace_bytes(T: int, d: int, f: int) -> int:
    return int(load().twell_sparse_down_union_workspace_bytes(T, d, f))


def hybrid_down_is_union(T: int, d: int, f: int, workspace_bytes: int) -> bool:
    """Whether the hybrid forwards whose pack holds hidden activations run the
    down projection over tile unions at this shape with this much workspace."""
    return bool(load().twell_hybrid_down_is_union(T, d, f, workspace_bytes))


def ffn_hybrid_forward_tc_up(x, WgT, WuT, Wd, tw: Twell, y, ovf_rows, n_ovf, workspace, dev_status,
                             stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_ffn_hybrid_forward_tc_up", load().twell_ffn_hybrid_forward_tc_up(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f, tw.ref(), _ptr(y), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def route(tw: Twell, ovf_rows, n_ovf, stream=None) -> None:
    _check("twell_route", load().twell_route(tw.ref(), _ptr(ovf_rows), _ptr(n_ovf), _stream(stream)))


def hybrid_workspace_bytes(T: int, d: int, f: int) -> int:
    return int(load().twell_hybrid_workspace_bytes(T, d, f))


def dense_workspace_bytes(T: int, d: int, f: int) -> int:
    return int(load().twell_dense_workspace_bytes(T, d, f))


def ffn_hybrid_forward(x, WgT, WuT, Wd, tw: Twell, y, ovf_rows, n_ovf, workspace, dev_status,
                       stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_ffn_hybrid_forward", load().twell_ffn_hybrid_forward(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f, tw.ref(), _ptr(y), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def ffn_hybrid_forward_noalloc(x, WgT, WuT, Wd, tw: Twell, y, ovf_rows, n_ovf, dev_status,
                               stream=None) -> None:
    """Hybrid forward on the library's built-in device scratch, for callers
    that cannot allocate a workspace (see twell_ffn_hybrid_forward_noalloc)."""
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_ffn_hybrid_forward_noalloc", load().twell_ffn_hybrid_forward_noalloc(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f, tw.ref(), _ptr(y), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(dev_status), _stream(stream)))


def dense_rows_forward(x, WgT, WuT, Wd, rows, n_rows, y, workspace, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_dense_rows_forward", load().twell_dense_rows_forward(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f, _ptr(rows), _ptr(n_rows), _ptr(y),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def dense_ffn_forward(x, WgT, WuT, Wd, y, workspace, dev_status, stream=None) -> None:
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_dense_ffn_forward", load().twell_dense_ffn_forward(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), T, d, f, _ptr(y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def relu_ffn_hybrid_forward(x, W1T, W2, tw: Twell, y, ovf_rows, n_ovf, workspace, dev_status,
                            stream=None) -> None:
    """Non-gated layer y = ReLU(x W1) W2, hybrid forward (W1T = W1 transposed, [f, d])."""
    T, d = x.shape
    f = W1T.shape[0]
    for n, t, s in (("x", x, (T, d)), ("W1T", W1T, (f, d)), ("W2", W2, (f, d)), ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_relu_ffn_hybrid_forward", load().twell_relu_ffn_hybrid_forward(
        _ptr(x), _ptr(W1T), _ptr(W2), T, d, f, tw.ref(), _ptr(y), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def relu_dense_rows_forward(x, W1T, W2, rows, n_rows, y, workspace, dev_status, stream=None) -> None:
    T, d = x.shape
    f = W1T.shape[0]
    for n, t, s in (("x", x, (T, d)), ("W1T", W1T, (f, d)), ("W2", W2, (f, d)), ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_relu_dense_rows_forward", load().twell_relu_dense_rows_forward(
        _ptr(x), _ptr(W1T), _ptr(W2), T, d, f, _ptr(rows), _ptr(n_rows), _ptr(y),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def relu_dense_ffn_forward(x, W1T, W2, y, workspace, dev_status, stream=None) -> None:
    T, d = x.shape
    f = W1T.shape[0]
    for n, t, s in (("x", x, (T, d)), ("W1T", W1T, (f, d)), ("W2", W2, (f, d)), ("y", y, (T, d))):
        _bf16(n, t, s)
    _check("twell_relu_dense_ffn_forward", load().twell_relu_dense_ffn_forward(
        _ptr(x), _ptr(W1T), _ptr(W2), T, d, f, _ptr(y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def backward_workspace_bytes(T: int, d: int, f: int, W: int) -> int:
    return int(load().twell_backward_workspace_bytes(T, d, f, W))


def ffn_hybrid_backward(x, WgT, WuT, Wd, dy, tw: Twell, ovf_rows, n_ovf, dx, dWgT, dWuT, dWd, workspace,
                        dev_status, stream=None) -> None:
    """Gradients of the hybrid forward (gate form) for upstream gradient dy:
    dx [T, d] and dWgT, dWuT, dWd [f, d], all fp32 (see twell_ffn_hybrid_backward)."""
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("dy", dy, (T, d))):
        _bf16(n, t, s)
    for n, t, s in (("dx", dx, (T, d)), ("dWgT", dWgT, (f, d)), ("dWuT", dWuT, (f, d)), ("dWd", dWd, (f, d))):
        _dev(n, t, s, torch.float32)
    _check("twell_ffn_hybrid_backward", load().twell_ffn_hybrid_backward(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), _ptr(dy), T, d, f, tw.ref(), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(dx), _ptr(dWgT), _ptr(dWuT), _ptr(dWd), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_status), _stream(stream)))


def ffn_hybrid_backward_dx(x, WgT, WuT, Wd, dy, tw: Twell, ovf_rows, n_ovf, dx, workspace, dev_status,
                           stream=None, tensor_cores: bool = False) -> None:
    """dx and the per-slot records: the rows that fit by per-token axpys on the
    CUDA cores, or (tensor_cores) by one GEMM over their scattered dz, du."""
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("dy", dy, (T, d))):
        _bf16(n, t, s)
    _dev("dx", dx, (T, d), torch.float32)
    name = "twell_ffn_hybrid_backward_dx_tc" if tensor_cores else "twell_ffn_hybrid_backward_dx"
    _check(name, getattr(load(), name)(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), _ptr(dy), T, d, f, tw.ref(), _ptr(ovf_rows), _ptr(n_ovf),
        _ptr(dx), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def ffn_hybrid_backward_dw(x, dy, tw: Twell, n_ovf, dWgT, dWuT, dWd, workspace, stream=None,
                           tensor_cores: bool = False) -> None:
    """Weight gradients after ffn_hybrid_backward_dx: per-unit sums on the CUDA
    cores, or (tensor_cores) the dense-scatter form on the tensor cores."""
    T, d = x.shape
    f = tw.f
    _bf16("x", x, (T, d))
    _bf16("dy", dy, (T, d))
    for n, t in (("dWgT", dWgT), ("dWuT", dWuT), ("dWd", dWd)):
        _dev(n, t, (f, d), torch.float32)
    name = "twell_ffn_hybrid_backward_dw_tc" if tensor_cores else "twell_ffn_hybrid_backward_dw"
    _check(name, getattr(load(), name)(
        _ptr(x), _ptr(dy), T, d, f, tw.ref(), _ptr(n_ovf), _ptr(dWgT), _ptr(dWuT), _ptr(dWd), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def dense_backward_workspace_bytes(T: int, d: int, f: int) -> int:
    return int(load().twell_dense_backward_workspace_bytes(T, d, f))


def dense_ffn_backward(x, WgT, WuT, Wd, dy, dx, dWgT, dWuT, dWd, workspace, dev_status, stream=None) -> None:
    """The library's dense backward (tensor cores, bf16 dz/du/h): the baseline of the hybrid backward."""
    T, d = x.shape
    f = WgT.shape[0]
    for n, t, s in (("x", x, (T, d)), ("WgT", WgT, (f, d)), ("WuT", WuT, (f, d)), ("Wd", Wd, (f, d)),
                    ("dy", dy, (T, d))):
        _bf16(n, t, s)
    for n, t, s in (("dx", dx, (T, d)), ("dWgT", dWgT, (f, d)), ("dWuT", dWuT, (f, d)), ("dWd", dWd, (f, d))):
        _dev(n, t, s, torch.float32)
    _check("twell_dense_ffn_backward", load().twell_dense_ffn_backward(
        _ptr(x), _ptr(WgT), _ptr(WuT), _ptr(Wd), _ptr(dy), T, d, f, _ptr(dx), _ptr(dWgT), _ptr(dWuT), _ptr(dWd),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def column_activity(x, WgT, active_bits, accumulate: bool, dev_status, stream=None) -> None:
    """Bit j of active_bits ([f // 32] int32 tensor) := some row of x has x . Wg[:, j] > 0
    (OR-ed into the existing bits when accumulate)."""
    T, d = x.shape
    f = WgT.shape[0]
    _bf16("x", x, (T, d))
    _bf16("WgT", WgT, (f, d))
    _dev("active_bits", active_bits, (f // 32,), torch.int32)
    _check("twell_column_activity", load().twell_column_activity(
        _ptr(x), _ptr(WgT), T, d, f, _ptr(active_bits), int(bool(accumulate)), _ptr(dev_status), _stream(stream)))


def compact_columns(active_bits, f: int, col_map, f_live, stream=None) -> None:
    _dev("active_bits", active_bits, (f // 32,), torch.int32)
    _dev("col_map", col_map, (f,), torch.int32)
    _dev("f_live", f_live, (1,), torch.int32)
    _check("twell_compact_columns", load().twell_compact_columns(
        _ptr(active_bits), f, _ptr(col_map), _ptr(f_live), _stream(stream)))


def gather_rows(W, col_map, f_live, W_out, dev_status, stream=None) -> None:
    f, d = W.shape
    f_out = W_out.shape[0]
    _bf16("W", W, (f, d))
    _bf16("W_out", W_out, (f_out, d))
    _dev("col_map", col_map, (f,), torch.int32)
    _check("twell_gather_rows", load().twell_gather_rows(
        _ptr(W), f, d, _ptr(col_map), _ptr(f_live), f_out, _ptr(W_out), _ptr(dev_status), _stream(stream)))


def compact_layer(x_profile, weights, dev_status, tile: int = 128, stream=None) -> dict:
    """Drop the hidden units that no row of x_profile activates: returns the
    gathered weights (same keys as `weights`, e.g. WgT/WuT/Wd, each [f_c, d]),
    col_map (original unit of each kept row, -1 for padding), f_live and f_c
    (f_live rounded up to a whole tile). The gate weight is weights["WgT"].
    Reads f_live back to the host once (a one-time model transformation)."""
    WgT = weights["WgT"]
    f = WgT.shape[0]
    dev = WgT.device
    bits = torch.empty((f // 32,), dtype=torch.int32, device=dev)
    col_map = torch.empty((f,), dtype=torch.int32, device=dev)
    f_live = torch.zeros((1,), dtype=torch.int32, device=dev)
    column_activity(x_profile, WgT, bits, False, dev_status, stream)
    compact_columns(bits, f, col_map, f_live, stream)
    n = int(f_live.item())
    f_c = max(tile, -(-n // tile) * tile)
    out = {"col_map": col_map[:f_c].clone(), "f_live": n, "f_c": f_c, "active_bits": bits}
    for k, W in weights.items():
        Wc = torch.empty((f_c, W.shape[1]), dtype=W.dtype, device=dev)
        gather_rows(W, col_map, f_live, Wc, dev_status, stream)
        out[k] = Wc
    return out


def unpack(tw: Twell, g_dense, dev_status, stream=None) -> None:
    _bf16("g_dense", g_dense, (tw.T, tw.f))
    _check("twell_unpack", load().twell_unpack(tw.ref(), _ptr(g_dense), _ptr(dev_status), _stream(stream)))


def to_device_bf16(bits, device="cuda") -> torch.Tensor:
    """Upload a uint16 numpy array of bf16 bit patterns as a bfloat16 tensor."""
    import numpy as np

    a = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return a.view(torch.bfloat16).to(device)


def bf16_bits(t: torch.Tensor):
    """bfloat16 tensor -> uint16 numpy array of its bit patterns."""
    import numpy as np

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
