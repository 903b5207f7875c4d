"""Bit-exact int32 sums of the kernels the benchmark times.

With every block scale equal to 1.0 and every activation row an integer
vector whose largest magnitude is exactly 127, the quantiser's scale is
s = 127 / 127 = 1 and q = x, so each output of the fp32 epilogues the decode
and prefill kernels run (y = rowscale * sum * (1/s)) is the int32 sum itself,
exactly (|sum| <= 127 * K < 2^24).  Comparing y bit for bit with the oracle's
block accumulators summed in int64 therefore checks the integer product of
the timed kernels with no rounding in between -- an off-by-one anywhere in a
sum fails.  The product is the integer add / subtract / skip of the ternary
weights ("BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级功耗遥测", section
"三值权重与 1.58-bit 的由来").

Which kernel each case reaches (dispatch of the library, uniform rows):
  bitnet_w2a8_linear, B = 1, K <= 16384      -> batch-1 decode kernel, fused
  bitnet_w2a8_gemv,   B = 1, K <= 16384      -> batch-1 decode kernel
  bitnet_w2a8_gemv,   B = 2..7, K <= 16384   -> batched decode kernel
  bitnet_w2a8_gemv,   B = 8..64              -> tensor-core kernel
  bitnet_w2a8_gemv_lut                       -> table-lookup kernel
  bitnet_w2a8_gemm                           -> tcgen05 GEMM, uniform path
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from helpers import QK, cuda, device_weight, lib, to_np, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert lib().bitnet_get_device_error() == lib().BITNET_OK


def _case(rows, K, T, seed, pick=None):
    """Ternary weights with unit scales, integer activations with s = 1, and
    the exact int32 row sums (for the rows in `pick`, all tokens)."""
    t = syn.ternary_uniform(seed, rows, K)
    sc = np.ones((rows, K // QK), dtype=np.float32)
    x = syn.integer_rows(seed + 1, T, K)
    rq, rs, _ = oracle.quant_act(x)
    assert np.all(rs == 1.0) and np.array_equal(rq.astype(np.float32), x)
    tp = t if pick is None else t[pick]
    sums = oracle.block_acc(oracle.pack_i2s(tp), K, rq).astype(np.int64).sum(axis=-1)
    assert np.abs(sums).max() < 2**24
    return t, sc, x, rq, sums.astype(np.float32)


def _pick(rows, seed, n=48):
    p = np.concatenate([[0, rows - 1], syn.splitmix64(seed, np.arange(n)) % np.uint64(rows)])
    return np.unique(p).astype(np.int64)


def _assert_bits(y, want, what):
    y = np.asarray(y, dtype=np.float32)
    bad = y.view(np.uint32) != want.view(np.uint32)
    if bad.any():
        i = np.argwhere(bad)[:4]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} sums differ; first {i.tolist()} "
                             f"got {y[tuple(i.T)]} want {want[tuple(i.T)]}")


DECODE_SHAPES = [(256, 512), (3840, 2560), (13824, 2560), (2560, 6912),
                 (28672, 4096), (4096, 14336)]   # the last two stream weights through the ring


@pytest.mark.parametrize("rows,K", DECODE_SHAPES)
def test_decode_b1_fused_sums_exact(rows, K):
    tt = torch()
    t, sc, x, rq, sums = _case(rows, K, 1, seed=rows * 3 + K)
    w, _ = device_weight(t, sc)
    y = tt.empty(rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_linear(w, cuda(x.reshape(-1)), 1, y)
    _assert_bits(to_np(y).reshape(1, rows), sums, f"fused decode {rows}x{K}")


@pytest.mark.parametrize("rows,K", DECODE_SHAPES)
def test_decode_b1_sums_exact(rows, K):
    tt = torch()
    t, sc, x, rq, sums = _case(rows, K, 1, seed=rows * 5 + K)
    w, _ = device_weight(t, sc)
    y = tt.empty(rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_gemv(w, cuda(rq.reshape(-1)), tt.ones(1, device="cuda"), 1, y)
    _assert_bits(to_np(y).reshape(1, rows), sums, f"decode {rows}x{K}")


@pytest.mark.parametrize("B", [2, 3, 4, 8, 13, 16])
@pytest.mark.parametrize("rows,K", [(777, 1280), (13824, 2560), (28672, 4096)])
def test_decode_batched_sums_exact(rows, K, B):
    tt = torch()
    pick = _pick(rows, rows ^ B) if rows * K > 10**7 else None
    t, sc, x, rq, sums = _case(rows, K, B, seed=rows * 7 + K + B, pick=pick)
    w, _ = device_weight(t, sc)
    y = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_gemv(w, cuda(rq.reshape(-1)), tt.ones(B, device="cuda"), B, y)
    got = to_np(y).reshape(B, rows)
    _assert_bits(got if pick is None else got[:, pick], sums, f"batched decode {rows}x{K} B={B}")


@pytest.mark.parametrize("rows,K", [(300, 1024), (3840, 2560), (2560, 6912)])
def test_lut_sums_exact(rows, K):
    tt = torch()
    t, sc, x, rq, sums = _case(rows, K, 1, seed=rows * 11 + K)
    w, _ = device_weight(t, sc)
    y = tt.empty(rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_gemv_lut(w, cuda(rq.reshape(-1)), tt.ones(1, device="cuda"), y)
    _assert_bits(to_np(y).reshape(1, rows), sums, f"lut {rows}x{K}")


@pytest.mark.parametrize("rows,K,T", [(1000, 640, 33), (2560, 2560, 129), (13824, 2560, 2048)])
def test_gemm_uniform_sums_exact(rows, K, T):
    tt = torch()
    pick = _pick(rows, rows + T) if rows * T > 10**6 else None
    t, sc, x, rq, sums = _case(rows, K, T, seed=rows + 13 * K + T, pick=pick)
    w, _ = device_weight(t, sc)
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    lib().bitnet_w2a8_gemm(w, cuda(rq.reshape(-1)), tt.ones(T, device="cuda"), T, y)
    got = to_np(y).reshape(T, rows)
    _assert_bits(got if pick is None else got[:, pick], sums, f"gemm {rows}x{K} T={T}")
