"""CPU oracle for the W2A8 linear layer -- TEST INFRASTRUCTURE.

Plain C (``w2a8_oracle.c``) compiled with gcc and loaded through ctypes.
Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package; the library under
``ternary_weight_absmax_b200`` never does.  It shares no code with the CUDA
path.  Every function cites the page section it follows in the C source.

Parity status: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (closed forms, hand-worked bytes, ties-to-even
cases, brute-force fp64 matmul, the absmean zero-fraction statistic).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w2a8_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

QK = 128
EPS = np.float32(1e-5)

OK, BAD_VALUE, CORRUPT, BAD_SHAPE = 0, 1, 2, 3

_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (strict IEEE: no contraction, no fast math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-frounding-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, p = ctypes.c_int64, ctypes.c_void_p
            lib.orc_pack_i2s.argtypes = [p, i64, i64, p]
            lib.orc_unpack_i2s.argtypes = [p, i64, i64, p]
            lib.orc_absmean_tensor.argtypes = [p, i64, p, p]
            lib.orc_absmean_tensor.restype = None
            lib.orc_absmean_blocks.argtypes = [p, i64, i64, p, p]
            lib.orc_quant_act.argtypes = [p, i64, i64, p, p, p]
            lib.orc_block_acc.argtypes = [p, i64, i64, p, i64, p]
            lib.orc_linear.argtypes = [p, p, i64, i64, p, p, i64, p, p]
            for name in ("orc_pack_i2s", "orc_unpack_i2s", "orc_absmean_blocks",
                         "orc_quant_act", "orc_block_acc", "orc_linear"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


def pack_i2s(t: np.ndarray) -> np.ndarray:
    """int8 ternary [rows][cols] -> i2_s codes uint8 [rows][cols/4]."""
    t = _c(t, np.int8)
    rows, cols = t.shape
    codes = np.empty((rows, cols // 4), dtype=np.uint8)
    _check(_load().orc_pack_i2s(_ptr(t), rows, cols, _ptr(codes)), "pack_i2s")
    return codes


def unpack_i2s(codes: np.ndarray, cols: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    rows = codes.shape[0]
    t = np.empty((rows, cols), dtype=np.int8)
    _check(_load().orc_unpack_i2s(_ptr(codes), rows, cols, _ptr(t)), "unpack_i2s")
    return t


def unpack_status(codes: np.ndarray, cols: int) -> int:
    codes = _c(codes, np.uint8)
    t = np.empty((codes.shape[0], cols), dtype=np.int8)
    return _load().orc_unpack_i2s(_ptr(codes), codes.shape[0], cols, _ptr(t))


def pack_status(t: np.ndarray) -> int:
    t = _c(t, np.int8)
    codes = np.empty((t.shape[0], t.shape[1] // 4), dtype=np.uint8)
    return _load().orc_pack_i2s(_ptr(t), t.shape[0], t.shape[1], _ptr(codes))


def absmean_tensor(w: np.ndarray):
    """Per-tensor absmean ternarisation -> (t int8, gamma float32)."""
    w = _c(w, np.float32)
    t = np.empty(w.shape, dtype=np.int8)
    g = np.zeros(1, dtype=np.float32)
    _load().orc_absmean_tensor(_ptr(w), w.size, _ptr(t), _ptr(g))
    return t, np.float32(g[0])


def absmean_blocks(w: np.ndarray):
    """Per-128-block absmean ternarisation -> (t int8, scales [rows][cols/128])."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    t = np.empty(w.shape, dtype=np.int8)
    sc = np.empty((rows, cols // QK), dtype=np.float32)
    _check(_load().orc_absmean_blocks(_ptr(w), rows, cols, _ptr(t), _ptr(sc)), "absmean_blocks")
    return t, sc


def quant_act(x: np.ndarray, with_blocksum: bool = True):
    """Per-row absmax int8 -> (q int8 [T][K], s float32 [T], blocksum int32 [T][K/128])."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    T, K = x.shape
    q = np.empty((T, K), dtype=np.int8)
    s = np.empty(T, dtype=np.float32)
    bs = np.empty((T, K // QK), dtype=np.int32) if with_blocksum else None
    _check(_load().orc_quant_act(_ptr(x), T, K, _ptr(q), _ptr(s),
                                 _ptr(bs) if bs is not None else None), "quant_act")
    return q, s, bs


def block_acc(codes: np.ndarray, cols: int, q: np.ndarray) -> np.ndarray:
    """int32 block accumulators acc[T][rows][cols/128]."""
    codes = _c(codes, np.uint8)
    q = _c(q, np.int8)
    rows = codes.shape[0]
    T = q.shape[0]
    acc = np.empty((T, rows, cols // QK), dtype=np.int32)
    _check(_load().orc_block_acc(_ptr(codes), rows, cols, _ptr(q), T, _ptr(acc)), "block_acc")
    return acc


def linear(codes: np.ndarray, scales: np.ndarray, cols: int, q: np.ndarray, s: np.ndarray,
           want_f64: bool = False):
    """y[T][rows] (fp32); with want_f64 also the fp64 value before rounding."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    q = _c(q, np.int8)
    s = _c(s, np.float32)
    rows = codes.shape[0]
    T = q.shape[0]
    y = np.empty((T, rows), dtype=np.float32)
    y64 = np.empty((T, rows), dtype=np.float64) if want_f64 else None
    _check(_load().orc_linear(_ptr(codes), _ptr(scales), rows, cols, _ptr(q), _ptr(s), T,
                              _ptr(y), _ptr(y64) if y64 is not None else None), "linear")
    return (y, y64) if want_f64 else y
