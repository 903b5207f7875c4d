"""CPU-only checks of the C ABI: the library loads, exports every entry point the
header declares, validates arguments before touching the GPU, and its host
i2_s packer produces the oracle's bytes exactly."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def b():
    import ternary_weight_absmax_b200 as mod
    return mod


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn), encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names.update(re.findall(r"\b(bitnet_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol(b):
    names = declared_symbols()
    assert "bitnet_w2a8_gemv" in names and "bitnet_w2a8_gemm" in names and "bitnet_quant_act" in names
    lib = ctypes.CDLL(b.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(b):
    for v in range(10):
        assert b.bitnet_status_string(v).startswith("BITNET_")
    assert b.bitnet_status_string(0) == "BITNET_OK"


def test_sizes(b, golden):
    for cols, bpr, spr in golden("row_stride.txt"):
        cols = int(cols)
        assert b.bitnet_i2s_code_bytes(3, cols) == 3 * int(bpr)
        assert b.bitnet_i2s_num_scales(3, cols) == 3 * int(spr)
        assert b.bitnet_repacked_bytes(3, cols) >= 3 * int(bpr)
    assert b.bitnet_i2s_code_bytes(3, 100) == 0
    assert b.bitnet_repacked_bytes(-1, 128) == 0


@pytest.mark.parametrize("rows,cols,seed", [(1, 128, 1), (7, 512, 2), (33, 2560, 3), (5, 6912, 4)])
def test_host_pack_matches_oracle_bytes(b, rows, cols, seed):
    t = syn.ternary_uniform(seed, rows, cols)
    np.testing.assert_array_equal(b.bitnet_pack_i2s(t), oracle.pack_i2s(t))
    np.testing.assert_array_equal(b.bitnet_unpack_i2s(oracle.pack_i2s(t), cols), t)


def test_host_pack_hand_byte(b, golden):
    rows = golden("i2s_hand_byte.txt")
    t = np.zeros((1, 128), dtype=np.int8)
    want = None
    for r in rows[1:]:
        if r[0] == "weight":
            t[0, int(r[1])] = int(r[2])
        else:
            want = np.array([int(v, 16) for v in r[1:]], dtype=np.uint8)
    np.testing.assert_array_equal(b.bitnet_pack_i2s(t)[0], want)


def test_host_pack_errors(b):
    lib = b.library()
    t = np.zeros((2, 128), dtype=np.int8)
    out = np.zeros(64, dtype=np.uint8)
    assert lib.bitnet_pack_i2s(None, 2, 128, out.ctypes.data, 64) == b.BITNET_ERR_NULL
    assert lib.bitnet_pack_i2s(t.ctypes.data, 2, 100, out.ctypes.data, 64) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_pack_i2s(t.ctypes.data, 2, 128, out.ctypes.data, 63) == b.BITNET_ERR_BUFSIZE
    t[1, 9] = 3
    assert lib.bitnet_pack_i2s(t.ctypes.data, 2, 128, out.ctypes.data, 64) == b.BITNET_ERR_VALUE
    assert "not ternary" in b.bitnet_last_error_detail()
    with pytest.raises(b.BitnetError):
        b.bitnet_pack_i2s(t)


def test_host_unpack_rejects_code3(b):
    codes = np.full((1, 32), 0x55, dtype=np.uint8)
    codes[0, 31] = 0xFF
    with pytest.raises(b.BitnetError) as e:
        b.bitnet_unpack_i2s(codes, 128)
    assert e.value.status == b.BITNET_ERR_CORRUPT


def test_device_calls_validate_before_touching_the_gpu(b):
    lib = b.library()
    W = b.bitnet_weight
    w = W()
    # Unrepacked handle, bad batch, NULL pointers: all rejected on the host.
    assert lib.bitnet_w2a8_gemv(None, None, None, 1, None, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), None, None, 1, None, None) == b.BITNET_ERR_NULL
    w.data = 256
    w.rows, w.cols, w.bytes = 16, 128, 1 << 20
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), 16, 16, 1, 16, None) == b.BITNET_ERR_VALUE
    w.layout_version = b.BITNET_LAYOUT_VERSION
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), 16, 16, 0, 16, None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), 16, 16, 65, 16, None) == b.BITNET_ERR_SHAPE
    # a fused linear beyond 16 tokens needs q_out / s_out to stage the quantised activations
    assert lib.bitnet_w2a8_linear(ctypes.byref(w), 16, 17, 16, None, None, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), 17, 16, 1, 16, None) == b.BITNET_ERR_ALIGN
    w.bytes = 10
    assert lib.bitnet_w2a8_gemv(ctypes.byref(w), 16, 16, 1, 16, None) == b.BITNET_ERR_BUFSIZE
    w.bytes = 1 << 20
    w.cols = 100
    assert lib.bitnet_w2a8_gemm(ctypes.byref(w), 16, 16, 4, 16, None) == b.BITNET_ERR_SHAPE
    w.cols = 128
    assert lib.bitnet_w2a8_gemm(ctypes.byref(w), 16, 16, -1, 16, None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_w2a8_gemm(ctypes.byref(w), 16, 16, 0, 16, None) == b.BITNET_OK  # T=0: no-op
    # Table-lookup GEMV: NULL / alignment, then weights without uniform rows or K > 8192.
    assert lib.bitnet_w2a8_gemv_lut(ctypes.byref(w), None, 16, 16, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_w2a8_gemv_lut(ctypes.byref(w), 17, 16, 16, None) == b.BITNET_ERR_ALIGN
    w.flags = 0
    assert lib.bitnet_w2a8_gemv_lut(ctypes.byref(w), 16, 16, 16, None) == b.BITNET_ERR_UNSUPPORTED
    w.flags = b.BITNET_WEIGHT_UNIFORM_ROWS
    w.cols = 8320
    assert lib.bitnet_w2a8_gemv_lut(ctypes.byref(w), 16, 16, 16, None) == b.BITNET_ERR_UNSUPPORTED
    w.cols = 128
    assert lib.bitnet_w2a8_gemm(ctypes.byref(w), 16, 16, 4, 8, None) == b.BITNET_ERR_ALIGN
    assert lib.bitnet_quant_act(16, 1, 100, 16, 16, None, None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_quant_act(16, 0, 128, 16, 16, None, None) == b.BITNET_OK
    assert lib.bitnet_quant_act(None, 1, 128, 16, 16, None, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_quant_act(8, 1, 128, 16, 16, None, None) == b.BITNET_ERR_ALIGN
    w2 = W()
    w2.data = 256
    w2.bytes = 1 << 20
    assert lib.bitnet_repack_device(16, 16, 16, 100, ctypes.byref(w2), None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_repack_device(16, 16, 16, 128, None, None) == b.BITNET_ERR_NULL
    w2.bytes = 100
    assert lib.bitnet_repack_device(16, 16, 16, 128, ctypes.byref(w2), None) == b.BITNET_ERR_BUFSIZE
    w2.bytes = 1 << 20
    w2.data = 128
    assert lib.bitnet_repack_device(16, 16, 16, 128, ctypes.byref(w2), None) == b.BITNET_ERR_ALIGN


def test_workspace_calls_validate_before_touching_the_gpu(b):
    # bitnet_w2a8_gemm_ws / bitnet_w2a8_linear_ws: the int8 weights plus the
    # hand-off area, NULL / shape / alignment / workspace size rejected on the host.
    lib = b.library()
    w = b.bitnet_weight()
    w.data = 256
    w.rows, w.cols, w.bytes = 16, 128, 1 << 20
    w.layout_version = b.BITNET_LAYOUT_VERSION
    w.flags = b.BITNET_WEIGHT_UNIFORM_ROWS
    need = b.bitnet_w2a8_gemm_workspace_bytes(16, 128)
    assert need >= 16 * 128
    assert b.bitnet_w2a8_gemm_workspace_bytes(1000, 640) >= 1008 * 640
    assert b.bitnet_w2a8_gemm_workspace_bytes(16, 100) == 0 and b.bitnet_w2a8_gemm_workspace_bytes(0, 128) == 0
    wr = ctypes.byref(w)
    assert lib.bitnet_w2a8_gemm_ws(None, 16, 16, 4, 16, 256, need, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_w2a8_gemm_ws(wr, 16, 16, -1, 16, 256, need, None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_w2a8_gemm_ws(wr, 16, 16, 0, 16, 256, need, None) == b.BITNET_OK  # T = 0: no-op
    assert lib.bitnet_w2a8_gemm_ws(wr, 16, 16, 4, 16, 256, need - 1, None) == b.BITNET_ERR_BUFSIZE
    assert lib.bitnet_w2a8_gemm_ws(wr, 16, 16, 4, 16, 272, need, None) == b.BITNET_ERR_ALIGN
    assert lib.bitnet_w2a8_linear_ws(wr, 16, 4, 16, None, 16, 256, need, None) == b.BITNET_ERR_NULL
    assert lib.bitnet_w2a8_linear_ws(wr, 16, 0, 16, 16, 16, 256, need, None) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_w2a8_linear_ws(wr, 16, 4, 8, 16, 16, 256, need, None) == b.BITNET_ERR_ALIGN
    assert lib.bitnet_w2a8_linear_ws(wr, 16, 4, 16, 16, 16, 256, need - 1, None) == b.BITNET_ERR_BUFSIZE
    assert lib.bitnet_w2a8_linear_ws(wr, 16, 4, 16, 16, 16, 272, need, None) == b.BITNET_ERR_ALIGN


def test_linear_seq_validates_before_touching_the_gpu(b):
    """bitnet_w2a8_linear_seq rejects, on the host: bad counts, waits on later
    entries, overlapping outputs, reads of another entry's output without a
    wait between them, weights without uniform rows, wide K, and a missing or
    short workspace when an entry waits."""
    lib = b.library()
    W = b.bitnet_weight

    def weight(rows, cols, flags=b.BITNET_WEIGHT_UNIFORM_ROWS):
        w = W()
        w.data, w.rows, w.cols, w.bytes = 256, rows, cols, 1 << 30
        w.layout_version, w.flags = b.BITNET_LAYOUT_VERSION, flags
        return w

    keep = []

    def call(entries, ws=None, wsb=0):
        arr = (b.bitnet_linear_desc * max(len(entries), 1))()
        for i, (w, x, y, d) in enumerate(entries):
            keep.append(w)
            arr[i].w = ctypes.pointer(w)
            arr[i].x_dev, arr[i].y_dev, arr[i].wait_for = x, y, d
        return lib.bitnet_w2a8_linear_seq(arr, len(entries), ws, wsb, None)

    A = 1 << 20  # fake device addresses, never dereferenced on the host
    w1, w2 = weight(64, 256), weight(32, 128)
    assert lib.bitnet_w2a8_linear_seq(None, 1, None, 0, None) == b.BITNET_ERR_NULL
    assert call([]) == b.BITNET_ERR_SHAPE
    assert lib.bitnet_w2a8_linear_seq_workspace_bytes(0) == 0
    assert lib.bitnet_w2a8_linear_seq_workspace_bytes(3) >= 16
    assert call([(w1, A, A + 4096, 0)]) == b.BITNET_ERR_VALUE                      # waits on itself
    assert call([(w1, A, A + 4096, -2)]) == b.BITNET_ERR_VALUE
    assert call([(w1, A, A + 4096, -1), (w2, A + 8192, A + 4096 + 128, -1)]) == b.BITNET_ERR_VALUE  # y overlap
    assert call([(w1, A, A + 4096, -1), (w2, A + 4096, A + 8192, -1)]) == b.BITNET_ERR_VALUE  # x reads y, no wait
    assert call([(w1, A, A, -1)]) == b.BITNET_ERR_VALUE                              # reads its own output
    assert call([(w1, A + 4, A + 4096, -1)]) == b.BITNET_ERR_ALIGN
    assert call([(w1, None, A + 4096, -1)]) == b.BITNET_ERR_NULL
    assert call([(weight(64, 256, flags=0), A, A + 4096, -1)]) == b.BITNET_ERR_UNSUPPORTED
    assert call([(weight(64, 16384 + 128), A, A + (1 << 22), -1)]) == b.BITNET_ERR_UNSUPPORTED
    chain = [(w1, A, A + 4096, -1), (w2, A + 4096, A + 8192, 0)]
    assert call(chain) == b.BITNET_ERR_NULL                                           # waits need a workspace
    assert call(chain, A + 65536, 4) == b.BITNET_ERR_BUFSIZE
    assert call(chain, A + 65538, 1 << 12) == b.BITNET_ERR_ALIGN
