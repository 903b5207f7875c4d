"""Bounded device waits: with the iteration cap forced to 1 the waits run out,
the kernel latches BITNET_ERR_TIMEOUT, waits (bounded) for its own copies (and,
in the GEMM, MMAs and tensor memory) and returns; nothing hangs, and the next
call on the same context is correct.  Covered: the GEMM, the batch-1 decode
kernel, the batched decode kernel and the table-lookup kernel.  No fault, trap
or hang is provoked."""
import numpy as np
import pytest

import oracle
from helpers import assert_close, assert_decode_close, device_weight, gpu_quant, lib, to_np, torch
import synthetic as syn

pytestmark = pytest.mark.gpu


def test_gemm_wait_timeout_is_reported_and_recoverable():
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    rows, K, T = 512, 1024, 256
    t = syn.ternary_uniform(77, rows, K)
    sc = syn.positive_scales(78, rows, K // 128, per_tensor=True)
    x = syn.activations(79, T, K)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    y = tt.empty(T * rows, dtype=tt.float32, device="cuda")
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_set_wait_limit(1)
    try:
        b.bitnet_w2a8_gemm(w, q, s, T, y)
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st == b.BITNET_ERR_TIMEOUT
    assert b.bitnet_get_device_error() == b.BITNET_OK      # the word was cleared
    b.bitnet_w2a8_gemm(w, q, s, T, y)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    rq, rs, _ = oracle.quant_act(x)
    assert_close(to_np(y).reshape(T, rows), oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), "after timeout")


def _forced_timeout(call, check, what):
    """Cap the waits at one try, launch four times, expect BITNET_ERR_TIMEOUT
    latched; then, with the default cap, the same call must be correct."""
    b = lib()
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_set_wait_limit(1)
    try:
        for _ in range(4):
            call()
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st == b.BITNET_ERR_TIMEOUT, f"{what}: {b.bitnet_status_string(st)}"
    assert b.bitnet_get_device_error() == b.BITNET_OK      # the word was cleared
    call()
    assert b.bitnet_get_device_error() == b.BITNET_OK
    check()


# 28672 x 4096: 1792 row tiles over the SMs, 13 per CTA, 26 tiles per warp --
# more than a warp's shared-memory slots, so the decode kernels stream tiles
# through the ring and wait on refills inside the product loop as well as on
# the first copies before griddepcontrol.wait.  With one try per wait, the
# first poll comes a CTA barrier after the copies were issued, far less than a
# copy's latency from HBM, so the waits run out and every warp takes the drain
# path (bounded waits for its own copies in flight, then return).
ROWS, K = 28672, 4096


def _weights(seed):
    t = syn.ternary_uniform(seed, ROWS, K)
    sc = syn.positive_scales(seed + 1, ROWS, K // 128, per_tensor=True)
    w, _ = device_weight(t, sc)
    return t, sc, w


def test_decode_b1_wait_timeout_is_reported_and_recoverable():
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    t, sc, w = _weights(81)
    x = syn.activations(83, 1, K)
    xd = tt.from_numpy(x.reshape(-1).copy()).cuda()
    y = tt.empty(ROWS, dtype=tt.float32, device="cuda")
    rq, rs, _ = oracle.quant_act(x)
    pick = np.arange(0, ROWS, 97)

    def check():
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        assert_decode_close(to_np(y).reshape(1, ROWS)[:, pick], ref, "batch-1 decode after timeout")

    _forced_timeout(lambda: b.bitnet_w2a8_linear(w, xd, 1, y), check, "batch-1 decode")


def test_decode_batched_wait_timeout_is_reported_and_recoverable():
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    B = 4
    t, sc, w = _weights(91)
    x = syn.activations(93, B, K)
    q, s, _ = gpu_quant(x)
    y = tt.empty(B * ROWS, dtype=tt.float32, device="cuda")
    rq, rs, _ = oracle.quant_act(x)
    pick = np.arange(5, ROWS, 101)

    def check():
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        assert_decode_close(to_np(y).reshape(B, ROWS)[:, pick], ref, "batched decode after timeout")

    _forced_timeout(lambda: b.bitnet_w2a8_gemv(w, q, s, B, y), check, "batched decode")


def test_lut_wait_timeout_is_reported_and_recoverable():
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    t, sc, w = _weights(97)
    x = syn.activations(99, 1, K)
    q, s, _ = gpu_quant(x)
    y = tt.empty(ROWS, dtype=tt.float32, device="cuda")
    rq, rs, _ = oracle.quant_act(x)
    pick = np.arange(7, ROWS, 89)

    def check():
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        assert_decode_close(to_np(y).reshape(1, ROWS)[:, pick], ref, "lut after timeout")

    _forced_timeout(lambda: b.bitnet_w2a8_gemv_lut(w, q, s, y), check, "table-lookup")
