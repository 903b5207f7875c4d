"""GPU parity of the small-batch paths for 2..64 tokens: the warp-MMA GEMV
(uniform rows; mma.sync m16n8k32 u8 x s8 with the code tiles as A fragments,
K split over a cluster), the general kernel and the GEMM's block-scale path
that bitnet_w2a8_gemv takes on per-block scales, and the two-kernel fused
linear (quantiser into the caller's q_out / s_out, then the GEMV).  Against
the oracle on the same seeded inputs: the int32 sums bit for bit (unit
scales, s = 1), y within the fp32-epilogue bound, q and s bit for bit; ragged
rows and K, split and unsplit K, zero rows; the kernel has no bounded waits,
so a wait limit of 1 changes nothing."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from helpers import QK, assert_close, assert_decode_close, cuda, device_weight, gpu_quant, lib, to_np, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert lib().bitnet_get_device_error() == lib().BITNET_OK


def _pick(rows, seed, n=48):
    if rows <= 2048:
        return np.arange(rows)
    p = np.concatenate([[0, rows - 1], syn.splitmix64(seed, np.arange(n)) % np.uint64(rows)])
    return np.unique(p).astype(np.int64)


def _guarded_gemv(w, q, s, B, rows, guard=64):
    tt = torch()
    buf = tt.full((B * rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    y = buf[guard:guard + B * rows]
    lib().bitnet_w2a8_gemv(w, q, s, B, y)
    b = to_np(buf)
    assert np.all(b[:guard] == 12345.0) and np.all(b[guard + B * rows:] == 12345.0), "output guard overwritten"
    return to_np(y).reshape(B, rows)


# (rows, K): ragged rows, K from one block to 14336 (K split 1..8 over the cluster)
SHAPES = [(1, 128), (17, 256), (128, 128), (129, 384), (777, 1280), (2560, 2560), (3840, 2560),
          (13824, 2560), (2560, 6912), (4096, 14336), (20480, 3200)]


@pytest.mark.parametrize("rows,K", SHAPES)
@pytest.mark.parametrize("B", [2, 3, 4, 8, 16, 17, 33, 64])
def test_mma_int32_sums_exact(rows, K, B):
    """Unit scales and integer activations with absmax 127 (s = 1): y is the
    exact int32 sum of every row and token."""
    tt = torch()
    t = syn.ternary_uniform(rows * 7 + K + B, rows, K)
    sc = np.ones((rows, K // QK), np.float32)
    x = syn.integer_rows(rows + 3 * K + B, B, K)
    rq, rs, _ = oracle.quant_act(x)
    assert np.all(rs == 1.0)
    w, _ = device_weight(t, sc)
    pick = _pick(rows, rows ^ B)
    want = oracle.block_acc(oracle.pack_i2s(t[pick]), K, rq).astype(np.int64).sum(-1).astype(np.float32)
    got = _guarded_gemv(w, cuda(rq.reshape(-1)), tt.ones(B, device="cuda"), B, rows)[:, pick]
    bad = got.view(np.uint32) != want.view(np.uint32)
    assert not bad.any(), f"{int(bad.sum())} sums differ, first {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("rows,K", [(777, 1280), (3840, 2560), (2560, 6912), (4096, 14336)])
@pytest.mark.parametrize("B", [4, 7, 16, 31, 64])
def test_mma_matches_oracle(rows, K, B):
    t = syn.ternary_uniform(rows * 3 + K + B, rows, K)
    sc = syn.positive_scales(rows + K + B, rows, K // QK, per_tensor=True)
    x = syn.activations(rows * 5 + B, B, K, outliers=True)
    x[B // 2] = 0.0                                  # an all-zero token row
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    rq, rs, _ = oracle.quant_act(x)
    pick = _pick(rows, rows + B)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    got = _guarded_gemv(w, q, s, B, rows)
    assert_decode_close(got[:, pick], ref, f"mma {rows}x{K} B={B}")
    assert np.all(got[B // 2] == 0.0)


@pytest.mark.parametrize("B", [4, 5, 8, 16])
def test_mma_agrees_with_general_kernel(B):
    """The general kernel (taken when accumulators are exported) on the same
    q, s: the same int32 sums, so y agrees within the fp32 epilogue bound."""
    tt = torch()
    rows, K = 1000, 1152
    t = syn.ternary_uniform(41 + B, rows, K)
    sc = syn.positive_scales(42 + B, rows, K // QK, per_tensor=True)
    x = syn.activations(43 + B, B, K)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    y_mma = _guarded_gemv(w, q, s, B, rows)
    y_g = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    acc = tt.empty(B * rows * (K // QK), dtype=tt.int32, device="cuda")
    lib().bitnet_w2a8_gemv_acc(w, q, s, B, y_g, acc)
    assert_decode_close(y_mma, to_np(y_g).reshape(B, rows).astype(np.float64), f"mma vs general B={B}")


@pytest.mark.parametrize("B", [17, 40, 64])
def test_block_scales_beyond_16_tokens_match_oracle(B):
    """Per-block scales at 17..64 tokens run the GEMM's block-scale path."""
    rows, K = 700, 1024
    t = syn.ternary_uniform(61 + B, rows, K)
    sc = syn.positive_scales(62 + B, rows, K // QK)
    x = syn.activations(63 + B, B, K, outliers=True)
    w, _ = device_weight(t, sc)
    assert not w.uniform
    q, s, _ = gpu_quant(x)
    rq, rs, _ = oracle.quant_act(x)
    got = _guarded_gemv(w, q, s, B, rows)
    assert_close(got, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), f"block scales B={B}")
    tt = torch()
    y2 = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    acc = tt.full((B * rows * (K // QK),), -7, dtype=tt.int32, device="cuda")
    lib().bitnet_w2a8_gemv_acc(w, q, s, B, y2, acc)
    np.testing.assert_array_equal(to_np(acc).reshape(B, rows, K // QK), oracle.block_acc(oracle.pack_i2s(t), K, rq))


@pytest.mark.parametrize("rows,K", [(777, 1280), (6144, 4096), (4096, 14336)])
@pytest.mark.parametrize("B", [2, 3, 4, 16, 24, 64])
@pytest.mark.parametrize("mode", ["tensor", "block"])
def test_linear_staged_matches_oracle(rows, K, B, mode):
    """bitnet_w2a8_linear with q_out / s_out: the quantiser, then the GEMV."""
    b = lib()
    tt = torch()
    t = syn.ternary_uniform(rows + K * 3 + B, rows, K)
    sc = syn.positive_scales(rows + B, rows, K // QK, per_tensor=(mode == "tensor"))
    x = syn.activations(rows * 11 + B, B, K, outliers=True)
    w, _ = device_weight(t, sc)
    q = tt.full((B * K,), 99, dtype=tt.int8, device="cuda")
    s = tt.full((B,), -1.0, dtype=tt.float32, device="cuda")
    y = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    b.bitnet_w2a8_linear(w, cuda(x.reshape(-1)), B, y, q, s)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(to_np(q).reshape(B, K), rq)
    np.testing.assert_array_equal(to_np(s).view(np.uint32), rs.view(np.uint32))
    pick = _pick(rows, rows * B)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    got = to_np(y).reshape(B, rows)[:, pick]
    if mode == "tensor":
        assert_decode_close(got, ref, f"staged linear {rows}x{K} B={B}")
    else:
        assert_close(got, ref, f"staged linear {rows}x{K} B={B} block scales")


def test_mma_has_no_waits_to_time_out():
    """The warp-MMA GEMV synchronises only with CTA and cluster barriers: with
    the bounded-wait limit at 1 it still completes, exactly, with no error."""
    b = lib()
    tt = torch()
    rows, K, B = 4096, 14336, 16
    t = syn.ternary_uniform(71, rows, K)
    sc = syn.positive_scales(72, rows, K // QK, per_tensor=True)
    x = syn.activations(73, B, K)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    y = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    y_ref = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    b.bitnet_w2a8_gemv(w, q, s, B, y_ref)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_set_wait_limit(1)
    try:
        b.bitnet_w2a8_gemv(w, q, s, B, y)
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st == b.BITNET_OK
    assert tt.equal(y, y_ref)
    rq, rs, _ = oracle.quant_act(x)
    pick = _pick(rows, 99)
    assert_decode_close(to_np(y).reshape(B, rows)[:, pick],
                        oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs), "mma GEMV, wait limit 1")
