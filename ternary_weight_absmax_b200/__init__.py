"""Python binding of libbitnet_w2a8.so, the B200 W2A8 (ternary x int8) library.

Argument marshalling only: every function here has the name of the C entry
point it calls (declared in ``include/bitnet_w2a8.h``), checks that the
buffers it was handed match the sizes it passes, and raises ``BitnetError``
on a non-OK status.  All computation happens in the CUDA kernels (device
calls) or in the library's host packer (``bitnet_pack_i2s`` /
``bitnet_unpack_i2s``).  PyTorch is used only to hand over device pointers
and the current CUDA stream.

If the shared library has not been built, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import _build_lib

LIB_PATH = _build_lib.LIB

BITNET_OK = 0
BITNET_ERR_NULL = 1
BITNET_ERR_SHAPE = 2
BITNET_ERR_ALIGN = 3
BITNET_ERR_VALUE = 4
BITNET_ERR_CORRUPT = 5
BITNET_ERR_BUFSIZE = 6
BITNET_ERR_CUDA = 7
BITNET_ERR_TIMEOUT = 8
BITNET_ERR_UNSUPPORTED = 9

BITNET_ABSMEAN_PER_TENSOR = 0
BITNET_ABSMEAN_PER_BLOCK = 1
BITNET_LAYOUT_VERSION = 1
BITNET_WEIGHT_UNIFORM_ROWS = 1
QK = 128


class BitnetError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str):
        self.status = status
        self.detail = detail
        super().__init__(f"{what}: {bitnet_status_string(status)} ({detail})")


class bitnet_weight(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("data", ctypes.c_void_p),
                ("bytes", ctypes.c_size_t), ("layout_version", ctypes.c_uint32),
                ("flags", ctypes.c_uint32)]


class bitnet_linear_desc(ctypes.Structure):
    _fields_ = [("w", ctypes.POINTER(bitnet_weight)), ("x_dev", ctypes.c_void_p), ("y_dev", ctypes.c_void_p),
                ("wait_for", ctypes.c_int32)]


BITNET_SEQ_MAX_LINEARS = 256
BITNET_SEQ_MAX_COLS = 16384


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbitnet_w2a8.so is not built ({LIB_PATH}); run __graft_entry__.build() "
                          "or python ternary_weight_absmax_b200/_build_lib.py")
    lib = ctypes.CDLL(LIB_PATH)
    i64, sz, vp, st = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
    W = ctypes.POINTER(bitnet_weight)
    sigs = {
        "bitnet_status_string": ([st], ctypes.c_char_p),
        "bitnet_last_error_detail": ([], ctypes.c_char_p),
        "bitnet_version": ([], ctypes.c_uint32),
        "bitnet_i2s_code_bytes": ([i64, i64], sz),
        "bitnet_i2s_num_scales": ([i64, i64], sz),
        "bitnet_repacked_bytes": ([i64, i64], sz),
        "bitnet_pack_i2s": ([vp, i64, i64, vp, sz], st),
        "bitnet_unpack_i2s": ([vp, i64, i64, vp, sz], st),
        "bitnet_ternarize_workspace_bytes": ([i64, i64], sz),
        "bitnet_ternarize_absmean_device": ([vp, i64, i64, ctypes.c_int, vp, vp, vp, sz, vp], st),
        "bitnet_ternarize_absmean_device_noalloc": ([vp, i64, i64, ctypes.c_int, vp, vp, vp], st),
        "bitnet_repack_device": ([vp, vp, i64, i64, W, vp], st),
        "bitnet_unrepack_device": ([W, vp, vp, vp], st),
        "bitnet_quant_act": ([vp, i64, i64, vp, vp, vp, vp], st),
        "bitnet_w2a8_gemv": ([W, vp, vp, i64, vp, vp], st),
        "bitnet_w2a8_gemm": ([W, vp, vp, i64, vp, vp], st),
        "bitnet_w2a8_gemm_workspace_bytes": ([i64, i64], sz),
        "bitnet_w2a8_gemm_ws": ([W, vp, vp, i64, vp, vp, sz, vp], st),
        "bitnet_w2a8_linear_ws": ([W, vp, i64, vp, vp, vp, vp, sz, vp], st),
        "bitnet_w2a8_linear": ([W, vp, i64, vp, vp, vp, vp], st),
        "bitnet_w2a8_linear_acc": ([W, vp, i64, vp, vp, vp, vp, vp], st),
        "bitnet_w2a8_gemv_acc": ([W, vp, vp, i64, vp, vp, vp], st),
        "bitnet_w2a8_gemv_lut": ([W, vp, vp, vp, vp], st),
        "bitnet_w2a8_gemm_acc": ([W, vp, vp, i64, vp, vp, vp], st),
        "bitnet_w2a8_linear_seq_workspace_bytes": ([ctypes.c_int32], sz),
        "bitnet_w2a8_linear_seq": ([ctypes.POINTER(bitnet_linear_desc), ctypes.c_int32, vp, sz, vp], st),
        "bitnet_get_device_error": ([vp], st),
        "bitnet_set_wait_limit": ([ctypes.c_uint32], st),
    }
    for name, (args, res) in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()

def library() -> ctypes.CDLL:
    return _lib


def bitnet_status_string(status: int) -> str:
    return _lib.bitnet_status_string(status).decode()


def bitnet_last_error_detail() -> str:
    return _lib.bitnet_last_error_detail().decode()


def _check(status: int, what: str):
    if status != BITNET_OK:
        raise BitnetError(status, what, bitnet_last_error_detail())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dptr(t, dtype_name: str, numel: int, what: str):
    """Device pointer of a CUDA tensor, after checking dtype, device and size."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if str(t.dtype) != f"torch.{dtype_name}":
        raise ValueError(f"{what} must be {dtype_name}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{what} holds {t.numel()} elements, needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


def bitnet_version() -> int:
    return _lib.bitnet_version()


def bitnet_i2s_code_bytes(rows: int, cols: int) -> int:
    return _lib.bitnet_i2s_code_bytes(rows, cols)


def bitnet_i2s_num_scales(rows: int, cols: int) -> int:
    return _lib.bitnet_i2s_num_scales(rows, cols)


def bitnet_repacked_bytes(rows: int, cols: int) -> int:
    return _lib.bitnet_repacked_bytes(rows, cols)


# ------------------------------------------------------------------ host --

def bitnet_pack_i2s(ternary: np.ndarray) -> np.ndarray:
    """int8 {-1,0,1} [rows][cols] (host) -> i2_s codes uint8 [rows][cols/4]."""
    t = np.ascontiguousarray(ternary, dtype=np.int8)
    if t.ndim != 2:
        raise ValueError("ternary must be 2-D")
    rows, cols = t.shape
    out = np.empty((rows, cols // 4), dtype=np.uint8)
    _check(_lib.bitnet_pack_i2s(t.ctypes.data, rows, cols, out.ctypes.data, out.nbytes),
           "bitnet_pack_i2s")
    return out


def bitnet_unpack_i2s(codes: np.ndarray, cols: int) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    rows = c.shape[0]
    out = np.empty((rows, cols), dtype=np.int8)
    _check(_lib.bitnet_unpack_i2s(c.ctypes.data, rows, cols, out.ctypes.data, out.nbytes),
           "bitnet_unpack_i2s")
    return out


# ---------------------------------------------------------------- device --

def bitnet_ternarize_workspace_bytes(rows: int, cols: int) -> int:
    return _lib.bitnet_ternarize_workspace_bytes(rows, cols)


def bitnet_ternarize_absmean_device(w, rows: int, cols: int, mode: int, codes_out, scales_out, workspace,
                                    stream=None):
    """fp32 w [rows*cols] -> i2_s codes uint8 [rows*cols/4] and fp32 block scales (CUDA tensors)."""
    _check(_lib.bitnet_ternarize_absmean_device(
        _dptr(w, "float32", rows * cols, "w"), rows, cols, mode,
        _dptr(codes_out, "uint8", rows * cols // 4, "codes"),
        _dptr(scales_out, "float32", rows * cols // QK, "scales"),
        _dptr(workspace, "uint8", bitnet_ternarize_workspace_bytes(rows, cols), "workspace"),
        workspace.numel(), _stream(stream)), "bitnet_ternarize_absmean_device")


class Weight:
    """A repacked device weight: the C struct plus the buffer that backs it."""

    def __init__(self, struct: bitnet_weight, buffer):
        self.struct = struct
        self.buffer = buffer

    @property
    def rows(self) -> int:
        return self.struct.rows

    @property
    def cols(self) -> int:
        return self.struct.cols

    @property
    def uniform(self) -> bool:
        return bool(self.struct.flags & BITNET_WEIGHT_UNIFORM_ROWS)

    def ref(self):
        return ctypes.byref(self.struct)


def bitnet_ternarize_absmean_device_noalloc(w, rows: int, cols: int, mode: int, codes_out, scales_out,
                                            stream=None):
    """As bitnet_ternarize_absmean_device, with the library's static scratch
    instead of a caller workspace (for callers that cannot allocate)."""
    _check(_lib.bitnet_ternarize_absmean_device_noalloc(
        _dptr(w, "float32", rows * cols, "w"), rows, cols, mode,
        _dptr(codes_out, "uint8", rows * cols // 4, "codes"),
        _dptr(scales_out, "float32", rows * cols // QK, "scales"), _stream(stream)),
        "bitnet_ternarize_absmean_device_noalloc")


def bitnet_repack_device(codes_dev, scales_dev, rows: int, cols: int, data_dev, stream=None) -> Weight:
    """codes uint8 [rows*cols/4], scales float32 [rows*cols/128], data uint8
    [bitnet_repacked_bytes] (all CUDA tensors) -> Weight.  Synchronous."""
    w = bitnet_weight()
    w.data = _dptr(data_dev, "uint8", bitnet_repacked_bytes(rows, cols), "data").value
    w.bytes = data_dev.numel()
    _check(_lib.bitnet_repack_device(_dptr(codes_dev, "uint8", rows * cols // 4, "codes"),
                                     _dptr(scales_dev, "float32", rows * cols // QK, "scales"),
                                     rows, cols, ctypes.byref(w), _stream(stream)),
           "bitnet_repack_device")
    return Weight(w, data_dev)


def bitnet_unrepack_device(w: Weight, codes_out, scales_out, stream=None):
    _check(_lib.bitnet_unrepack_device(w.ref(), _dptr(codes_out, "uint8", w.rows * w.cols // 4, "codes"),
                                       _dptr(scales_out, "float32", w.rows * w.cols // QK, "scales"),
                                       _stream(stream)), "bitnet_unrepack_device")


def bitnet_quant_act(x, T: int, K: int, q, s, blocksum=None, stream=None):
    _check(_lib.bitnet_quant_act(_dptr(x, "float32", T * K, "x"), T, K, _dptr(q, "int8", T * K, "q"),
                                 _dptr(s, "float32", T, "s"),
                                 _dptr(blocksum, "int32", T * (K // QK), "blocksum"), _stream(stream)),
           "bitnet_quant_act")


def bitnet_w2a8_gemv(w: Weight, q, s, B: int, y, stream=None):
    _check(_lib.bitnet_w2a8_gemv(w.ref(), _dptr(q, "int8", B * w.cols, "q"), _dptr(s, "float32", B, "s"), B,
                                 _dptr(y, "float32", B * w.rows, "y"), _stream(stream)), "bitnet_w2a8_gemv")


def bitnet_w2a8_gemm(w: Weight, q, s, T: int, y, stream=None):
    _check(_lib.bitnet_w2a8_gemm(w.ref(), _dptr(q, "int8", T * w.cols, "q"), _dptr(s, "float32", T, "s"), T,
                                 _dptr(y, "float32", T * w.rows, "y"), _stream(stream)), "bitnet_w2a8_gemm")


def bitnet_w2a8_gemm_workspace_bytes(rows: int, cols: int) -> int:
    return _lib.bitnet_w2a8_gemm_workspace_bytes(rows, cols)


def bitnet_w2a8_gemm_ws(w: Weight, q, s, T: int, y, workspace, stream=None):
    """bitnet_w2a8_gemm with a workspace (uint8 CUDA tensor of
    bitnet_w2a8_gemm_workspace_bytes(rows, cols) bytes, or None)."""
    n = bitnet_w2a8_gemm_workspace_bytes(w.rows, w.cols)
    ws = _dptr(workspace, "uint8", n, "workspace") if workspace is not None else None
    _check(_lib.bitnet_w2a8_gemm_ws(w.ref(), _dptr(q, "int8", T * w.cols, "q"), _dptr(s, "float32", T, "s"), T,
                                    _dptr(y, "float32", T * w.rows, "y"), ws,
                                    workspace.numel() if workspace is not None else 0, _stream(stream)),
           "bitnet_w2a8_gemm_ws")


def bitnet_w2a8_linear_ws(w: Weight, x, T: int, y, q_out, s_out, workspace=None, stream=None):
    """Linear layer at any T: fp32 x [T*K] -> y [T*rows], q_out / s_out written;
    workspace: uint8 CUDA tensor of bitnet_w2a8_gemm_workspace_bytes(rows, cols) or None."""
    n = bitnet_w2a8_gemm_workspace_bytes(w.rows, w.cols)
    ws = _dptr(workspace, "uint8", n, "workspace") if workspace is not None else None
    _check(_lib.bitnet_w2a8_linear_ws(w.ref(), _dptr(x, "float32", T * w.cols, "x"), T,
                                      _dptr(y, "float32", T * w.rows, "y"), _dptr(q_out, "int8", T * w.cols, "q_out"),
                                      _dptr(s_out, "float32", T, "s_out"), ws,
                                      workspace.numel() if workspace is not None else 0, _stream(stream)),
           "bitnet_w2a8_linear_ws")


def bitnet_w2a8_linear(w: Weight, x, B: int, y, q_out=None, s_out=None, stream=None):
    """Fused act-quant + GEMV: fp32 x [B*K] -> y [B*rows]; optional q_out/s_out."""
    _check(_lib.bitnet_w2a8_linear(w.ref(), _dptr(x, "float32", B * w.cols, "x"), B,
                                   _dptr(y, "float32", B * w.rows, "y"), _dptr(q_out, "int8", B * w.cols, "q_out"),
                                   _dptr(s_out, "float32", B, "s_out"), _stream(stream)), "bitnet_w2a8_linear")


def bitnet_w2a8_linear_acc(w: Weight, x, B: int, y, acc, q_out=None, s_out=None, stream=None):
    _check(_lib.bitnet_w2a8_linear_acc(w.ref(), _dptr(x, "float32", B * w.cols, "x"), B,
                                       _dptr(y, "float32", B * w.rows, "y"),
                                       _dptr(q_out, "int8", B * w.cols, "q_out"),
                                       _dptr(s_out, "float32", B, "s_out"),
                                       _dptr(acc, "int32", B * w.rows * (w.cols // QK), "acc"), _stream(stream)),
           "bitnet_w2a8_linear_acc")


def bitnet_w2a8_gemv_acc(w: Weight, q, s, B: int, y, acc, stream=None):
    _check(_lib.bitnet_w2a8_gemv_acc(w.ref(), _dptr(q, "int8", B * w.cols, "q"), _dptr(s, "float32", B, "s"),
                                     B, _dptr(y, "float32", B * w.rows, "y"),
                                     _dptr(acc, "int32", B * w.rows * (w.cols // QK), "acc"), _stream(stream)),
           "bitnet_w2a8_gemv_acc")


def bitnet_w2a8_gemv_lut(w: Weight, q, s, y, stream=None):
    _check(_lib.bitnet_w2a8_gemv_lut(w.ref(), _dptr(q, "int8", w.cols, "q"), _dptr(s, "float32", 1, "s"),
                                     _dptr(y, "float32", w.rows, "y"), _stream(stream)),
           "bitnet_w2a8_gemv_lut")


def bitnet_w2a8_gemm_acc(w: Weight, q, s, T: int, y, acc, stream=None):
    _check(_lib.bitnet_w2a8_gemm_acc(w.ref(), _dptr(q, "int8", T * w.cols, "q"), _dptr(s, "float32", T, "s"),
                                     T, _dptr(y, "float32", T * w.rows, "y"),
                                     _dptr(acc, "int32", T * w.rows * (w.cols // QK), "acc"), _stream(stream)),
           "bitnet_w2a8_gemm_acc")


def bitnet_w2a8_linear_seq_workspace_bytes(n: int) -> int:
    return _lib.bitnet_w2a8_linear_seq_workspace_bytes(n)


def bitnet_w2a8_linear_seq(entries, workspace=None, stream=None):
    """One kernel for a list of batch-1 decode linears.  entries: sequence of
    (Weight, x, y, wait_for) with x fp32 [cols] and y fp32 [rows] CUDA tensors
    (or views) and wait_for -1 or the index of the entry whose y x reads.
    workspace: uint8 CUDA tensor of bitnet_w2a8_linear_seq_workspace_bytes(n)
    bytes, zero-filled before first use (needed only when an entry waits)."""
    n = len(entries)
    arr = (bitnet_linear_desc * max(n, 1))()
    for i, (w, x, y, wait_for) in enumerate(entries):
        arr[i].w = ctypes.pointer(w.struct)
        arr[i].x_dev = _dptr(x, "float32", w.cols, f"x[{i}]")
        arr[i].y_dev = _dptr(y, "float32", w.rows, f"y[{i}]")
        arr[i].wait_for = int(wait_for)
    ws = _dptr(workspace, "uint8", bitnet_w2a8_linear_seq_workspace_bytes(n), "workspace") if workspace is not None \
        else None
    _check(_lib.bitnet_w2a8_linear_seq(arr, n, ws, workspace.numel() if workspace is not None else 0,
                                       _stream(stream)), "bitnet_w2a8_linear_seq")


def bitnet_get_device_error(stream=None) -> int:
    """Returns the status (does not raise): BITNET_OK or the latched device error."""
    return _lib.bitnet_get_device_error(_stream(stream))


def bitnet_set_wait_limit(max_iterations: int):
    _check(_lib.bitnet_set_wait_limit(max_iterations), "bitnet_set_wait_limit")
