"""The prefill GEMM with a workspace (bitnet_w2a8_gemm_ws): from 256 tokens
on uniform rows the weights are expanded to int8 once per call and both MMA
operands come in by TMA.  It must give the int32 sums exactly (unit scales,
s = 1: y is the sum itself) and the same y, bit for bit, as
bitnet_w2a8_gemm on every shape, including rows that end inside a 256-row
tile and token counts that end inside a 128-token tile; below 256 tokens,
on block-scale weights and without a workspace it is bitnet_w2a8_gemm.
bitnet_w2a8_linear_ws (fp32 x in; from 256 tokens with a workspace one
kernel quantises x and expands the weights) must give the q, s and y of the
quantiser followed by bitnet_w2a8_gemm, bit for bit.
The product is the integer add / subtract / skip of the ternary weights
("BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级功耗遥测", section
"三值权重与 1.58-bit 的由来")."""
import ctypes

import numpy as np
import pytest

import oracle
import synthetic as syn
from helpers import QK, assert_close, cuda, device_weight, gpu_quant, lib, to_np, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert lib().bitnet_get_device_error() == lib().BITNET_OK


def _workspace(rows, K, extra=0):
    n = lib().bitnet_w2a8_gemm_workspace_bytes(rows, K)
    assert n == ((rows + 15) // 16) * 16 * K
    # Filled with a pattern, so stale bytes would show.
    return torch().full((n + extra,), 0x5A, dtype=torch().uint8, device="cuda")


def _both(t, sc, x, guard=64):
    """y of bitnet_w2a8_gemm and of bitnet_w2a8_gemm_ws on the same q, s."""
    b = lib()
    tt = torch()
    rows, K = t.shape
    T = x.shape[0]
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ys = []
    for ws in (None, _workspace(rows, K)):
        buf = tt.full((T * rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
        y = buf[guard:guard + T * rows]
        if ws is None:
            b.bitnet_w2a8_gemm(w, q, s, T, y)
        else:
            b.bitnet_w2a8_gemm_ws(w, q, s, T, y, ws)
        assert b.bitnet_get_device_error() == b.BITNET_OK
        yb = to_np(buf)
        assert np.all(yb[:guard] == 12345.0) and np.all(yb[guard + T * rows:] == 12345.0), "guard overwritten"
        ys.append(to_np(y).reshape(T, rows))
    return q, s, ys[0], ys[1]


@pytest.mark.parametrize("rows,K,T", [(1000, 640, 300), (2560, 2560, 256), (13824, 2560, 2048)])
def test_gemm_ws_int32_sums_exact(rows, K, T):
    tt = torch()
    seed = rows * 3 + K + T
    t = syn.ternary_uniform(seed, rows, K)
    sc = np.ones((rows, K // QK), dtype=np.float32)
    x = syn.integer_rows(seed + 1, T, K)
    rq, rs, _ = oracle.quant_act(x)
    assert np.all(rs == 1.0) and np.array_equal(rq.astype(np.float32), x)
    pick = None
    if rows * T > 10**6:
        pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(seed, np.arange(48)) % np.uint64(rows)]))
        pick = pick.astype(np.int64)
    tp = t if pick is None else t[pick]
    sums = oracle.block_acc(oracle.pack_i2s(tp), K, rq).astype(np.int64).sum(axis=-1)
    assert np.abs(sums).max() < 2**24
    w, _ = device_weight(t, sc)
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_gemm_ws(w, cuda(rq.reshape(-1)), tt.ones(T, device="cuda"), T, y, _workspace(rows, K))
    got = to_np(y).reshape(T, rows)
    got = got if pick is None else got[:, pick]
    assert np.array_equal(got, sums.astype(np.float32)), f"gemm_ws {rows}x{K} T={T}: int32 sums differ"


@pytest.mark.parametrize("rows,K,T", [
    (300, 256, 512), (2576, 2560, 257), (17, 128, 300), (4000, 1280, 640),
    (13824, 2560, 2048), (2560, 6912, 512), (28672, 4096, 1024), (4096, 14336, 1024),
])
def test_gemm_ws_matches_gemm_bitwise(rows, K, T):
    t = syn.ternary_uniform(rows + 7 * K + T, rows, K)
    sc = syn.positive_scales(rows + K, rows, K // QK, per_tensor=True)
    x = syn.activations(rows + T, T, K, outliers=True)
    _, _, y0, y1 = _both(t, sc, x)
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32)), f"{rows}x{K} T={T}"


def test_gemm_ws_matches_oracle():
    rows, K, T = 700, 1024, 384
    t = syn.ternary_uniform(5, rows, K)
    sc = syn.positive_scales(6, rows, K // QK, per_tensor=True)
    x = syn.activations(7, T, K, outliers=True)
    q, s, _, y1 = _both(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(to_np(q).reshape(T, K), rq)
    assert_close(y1, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), "gemm_ws vs oracle")


def test_gemm_ws_small_T_and_block_scales_take_the_other_paths():
    # Below 256 tokens, and on block-scale weights, the workspace is not used:
    # the result is bitnet_w2a8_gemm's, and the workspace keeps its pattern.
    b = lib()
    tt = torch()
    for mode, T in (("tensor", 100), ("block", 512)):
        rows, K = 256, 512
        t = syn.ternary_uniform(T, rows, K)
        sc = syn.positive_scales(T + 1, rows, K // QK, per_tensor=(mode == "tensor"))
        x = syn.activations(T + 2, T, K)
        w, _ = device_weight(t, sc)
        q, s, _ = gpu_quant(x)
        ws = _workspace(rows, K)
        y0 = tt.empty(T * rows, dtype=tt.float32, device="cuda")
        y1 = tt.empty(T * rows, dtype=tt.float32, device="cuda")
        b.bitnet_w2a8_gemm(w, q, s, T, y0)
        b.bitnet_w2a8_gemm_ws(w, q, s, T, y1, ws)
        b.bitnet_w2a8_gemm_ws(w, q, s, T, y1, None)
        assert b.bitnet_get_device_error() == b.BITNET_OK
        assert tt.equal(y0, y1), mode
        assert bool((ws == 0x5A).all()), f"{mode}: workspace written"


def test_gemm_ws_rejects_small_or_misaligned_workspace():
    b = lib()
    tt = torch()
    rows, K, T = 256, 512, 256
    t = syn.ternary_uniform(9, rows, K)
    sc = syn.positive_scales(10, rows, K // QK, per_tensor=True)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(syn.activations(11, T, K))
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    need = b.bitnet_w2a8_gemm_workspace_bytes(rows, K)
    ws = tt.zeros(need + 256, dtype=tt.uint8, device="cuda")
    raw = b.library().bitnet_w2a8_gemm_ws
    args = (w.ref(), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(s.data_ptr()), T,
            ctypes.c_void_p(y.data_ptr()))
    assert raw(*args, ctypes.c_void_p(ws.data_ptr()), need - 1, None) == b.BITNET_ERR_BUFSIZE
    assert raw(*args, ctypes.c_void_p(ws.data_ptr() + 16), need, None) == b.BITNET_ERR_ALIGN
    assert raw(*args, ctypes.c_void_p(ws.data_ptr()), need, None) == b.BITNET_OK
    assert b.bitnet_get_device_error() == b.BITNET_OK
    assert b.bitnet_w2a8_gemm_workspace_bytes(0, K) == 0 and b.bitnet_w2a8_gemm_workspace_bytes(rows, 100) == 0


def test_gemm_ws_wait_timeout_is_reported_and_recoverable():
    b = lib()
    tt = torch()
    rows, K, T = 512, 1024, 512
    t = syn.ternary_uniform(77, rows, K)
    sc = syn.positive_scales(78, rows, K // QK, per_tensor=True)
    x = syn.activations(79, T, K)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ws = _workspace(rows, K)
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_set_wait_limit(1)
    try:
        for _ in range(4):
            b.bitnet_w2a8_gemm_ws(w, q, s, T, y, ws)
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st == b.BITNET_ERR_TIMEOUT
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_w2a8_gemm_ws(w, q, s, T, y, ws)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    rq, rs, _ = oracle.quant_act(x)
    assert_close(to_np(y).reshape(T, rows), oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), "after timeout")


@pytest.mark.parametrize("rows,K,T,mode,with_ws", [
    (256, 512, 64, "tensor", True), (300, 640, 100, "tensor", True), (1000, 1280, 300, "tensor", True),
    (13824, 2560, 2048, "tensor", True), (2560, 6912, 512, "tensor", True), (2576, 2560, 257, "tensor", True),
    (300, 640, 300, "tensor", False), (256, 512, 512, "block", True),
])
def test_linear_ws_matches_quantiser_then_gemm(rows, K, T, mode, with_ws):
    # bitnet_w2a8_linear_ws (from 256 tokens with a workspace: one kernel that
    # quantises x and expands the weights, then the pair GEMM) against the
    # quantiser followed by bitnet_w2a8_gemm (bitnet_w2a8_linear up to 64
    # tokens): q, s and y bit for bit.
    b = lib()
    tt = torch()
    t = syn.ternary_uniform(rows * 5 + T, rows, K)
    sc = syn.positive_scales(rows + 3, rows, K // QK, per_tensor=(mode == "tensor"))
    x = cuda(syn.activations(K + T, T, K, outliers=True).reshape(-1))
    w, _ = device_weight(t, sc)
    q0 = tt.empty(T * K, dtype=tt.int8, device="cuda")
    s0 = tt.empty(T, dtype=tt.float32, device="cuda")
    y0 = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    if T <= 64:
        b.bitnet_w2a8_linear(w, x, T, y0, q0, s0)
    else:
        b.bitnet_quant_act(x, T, K, q0, s0)
        b.bitnet_w2a8_gemm(w, q0, s0, T, y0)
    q1 = tt.full((T * K,), 99, dtype=tt.int8, device="cuda")
    s1 = tt.full((T,), -1.0, dtype=tt.float32, device="cuda")
    y1 = tt.full((T * rows,), float("nan"), dtype=tt.float32, device="cuda")
    b.bitnet_w2a8_linear_ws(w, x, T, y1, q1, s1, _workspace(rows, K) if with_ws else None)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    assert tt.equal(q0, q1) and tt.equal(s0, s1), "q or s differ"
    assert np.array_equal(to_np(y0).view(np.uint32), to_np(y1).view(np.uint32)), f"{rows}x{K} T={T} {mode}"


def test_linear_ws_checks_its_arguments():
    b = lib()
    tt = torch()
    rows, K, T = 256, 512, 300
    t = syn.ternary_uniform(21, rows, K)
    w, _ = device_weight(t, syn.positive_scales(22, rows, K // QK, per_tensor=True))
    x = tt.zeros(T * K, dtype=tt.float32, device="cuda")
    q = tt.empty(T * K, dtype=tt.int8, device="cuda")
    s = tt.empty(T, dtype=tt.float32, device="cuda")
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    need = b.bitnet_w2a8_gemm_workspace_bytes(rows, K)
    ws = tt.zeros(need, dtype=tt.uint8, device="cuda")
    raw = b.library().bitnet_w2a8_linear_ws
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    assert raw(w.ref(), p(x), T, p(y), None, p(s), p(ws), need, None) == b.BITNET_ERR_NULL
    assert raw(w.ref(), p(x), T, p(y), p(q), p(s), p(ws), need - 1, None) == b.BITNET_ERR_BUFSIZE
    assert raw(w.ref(), p(x), 0, p(y), p(q), p(s), p(ws), need, None) == b.BITNET_ERR_SHAPE
    assert raw(w.ref(), p(x), T, p(y), p(q), p(s), p(ws), need, None) == b.BITNET_OK
    assert b.bitnet_get_device_error() == b.BITNET_OK


@pytest.mark.parametrize("rows,K,T", [(1000, 640, 300), (13824, 2560, 2048)])
def test_linear_ws_int32_sums_exact(rows, K, T):
    # Integer activations whose row absmax is 127 quantise to q = x with s = 1,
    # and unit scales make y the int32 sum itself: the fused quantise-and-
    # expand pre-pass and the pair GEMM must reproduce the oracle's sums.
    b = lib()
    tt = torch()
    seed = rows + 7 * T
    t = syn.ternary_uniform(seed, rows, K)
    sc = np.ones((rows, K // QK), dtype=np.float32)
    x = syn.integer_rows(seed + 1, T, K)
    rq, rs, _ = oracle.quant_act(x)
    assert np.all(rs == 1.0)
    pick = None
    if rows * T > 10**6:
        pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(seed, np.arange(48)) % np.uint64(rows)]))
        pick = pick.astype(np.int64)
    tp = t if pick is None else t[pick]
    sums = oracle.block_acc(oracle.pack_i2s(tp), K, rq).astype(np.int64).sum(axis=-1)
    w, _ = device_weight(t, sc)
    q = tt.empty(T * K, dtype=tt.int8, device="cuda")
    s = tt.empty(T, dtype=tt.float32, device="cuda")
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    b.bitnet_w2a8_linear_ws(w, cuda(x.reshape(-1)), T, y, q, s, _workspace(rows, K))
    assert b.bitnet_get_device_error() == b.BITNET_OK
    np.testing.assert_array_equal(to_np(q).reshape(T, K), rq)
    got = to_np(y).reshape(T, rows)
    got = got if pick is None else got[:, pick]
    assert np.array_equal(got, sums.astype(np.float32)), f"linear_ws {rows}x{K} T={T}: int32 sums differ"
