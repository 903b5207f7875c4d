"""The GEMM's bounded mbarrier waits: with the iteration cap forced to 1 the
waits run out, the kernel latches BITNET_ERR_TIMEOUT, drains its own copies
and MMAs, frees tensor memory and returns; nothing hangs, and the next call
on the same context is correct.  No fault, trap or hang is provoked."""
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


def test_decode_wait_limit_returns_and_recovers():
    """The batch-1 decode kernel waits (bounded) on its weight copies.  With the
    cap at one try a wait may or may not run out, depending on whether the
    copy has landed; either way the call returns, a timeout is latched as
    BITNET_ERR_TIMEOUT, and the next call is correct."""
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    rows, K = 13824, 2560
    t = syn.ternary_uniform(81, rows, K)
    sc = syn.positive_scales(82, rows, K // 128, per_tensor=True)
    x = syn.activations(83, 1, K)
    w, _ = device_weight(t, sc)
    xd = tt.from_numpy(x.reshape(-1).copy()).cuda()
    y = tt.empty(rows, dtype=tt.float32, device="cuda")
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_set_wait_limit(1)
    try:
        for _ in range(4):
            b.bitnet_w2a8_linear(w, xd, 1, y)
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st in (b.BITNET_OK, b.BITNET_ERR_TIMEOUT)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    b.bitnet_w2a8_linear(w, xd, 1, y)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    rq, rs, _ = oracle.quant_act(x)
    assert_decode_close(to_np(y).reshape(1, rows), oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), "after limit")
