"""The allocation-free ternariser entry point.

Some callers cannot give the library device scratch memory: a host whose own
fixed pool already owns all of the GPU's memory, a binding with no device
allocator, or a serving loop that must not call cudaMalloc because it can
synchronise the whole device.  bitnet_ternarize_absmean_device_noalloc serves
them from a static device array inside the library.  This test calls it
through the C ABI twice in a row -- two different weight matrices, so the
second call runs on scratch the first one left behind -- and checks each
result against bitnet_ternarize_absmean_device given a caller-allocated
workspace: the packed codes and the scales must match bit for bit.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import synthetic as syn
from helpers import QK, cuda, lib, to_np, torch

pytestmark = pytest.mark.gpu


def _with_workspace(b, tt, w_d, rows, cols, mode):
    codes = tt.empty(rows * cols // 4, dtype=tt.uint8, device="cuda")
    scales = tt.empty(rows * cols // QK, dtype=tt.float32, device="cuda")
    ws = tt.empty(b.bitnet_ternarize_workspace_bytes(rows, cols), dtype=tt.uint8, device="cuda")
    b.bitnet_ternarize_absmean_device(w_d, rows, cols, mode, codes, scales, ws)
    return to_np(codes), to_np(scales)


def _no_alloc_via_c_abi(b, tt, w_d, rows, cols, mode):
    codes = tt.full((rows * cols // 4,), 0xEE, dtype=tt.uint8, device="cuda")
    scales = tt.full((rows * cols // QK,), -1.0, dtype=tt.float32, device="cuda")
    stream = ctypes.c_void_p(tt.cuda.current_stream().cuda_stream)
    st = b.library().bitnet_ternarize_absmean_device_noalloc(
        ctypes.c_void_p(w_d.data_ptr()), rows, cols, mode, ctypes.c_void_p(codes.data_ptr()),
        ctypes.c_void_p(scales.data_ptr()), stream)
    assert st == b.BITNET_OK, b.bitnet_last_error_detail()
    return to_np(codes), to_np(scales)


def test_no_alloc_matches_workspace_entry_point_twice_in_a_row():
    tt = torch()
    if not tt.cuda.is_available():
        pytest.skip("no CUDA device")
    b = lib()
    cases = [(3840, 2560, 0xA11), (1000, 640, 0xB22)]   # second call: smaller, new data
    for rows, cols, seed in cases:
        w_d = cuda(syn.normal_matrix(seed, rows, cols).reshape(-1))
        for mode in (b.BITNET_ABSMEAN_PER_TENSOR, b.BITNET_ABSMEAN_PER_BLOCK):
            want_c, want_s = _with_workspace(b, tt, w_d, rows, cols, mode)
            got_c, got_s = _no_alloc_via_c_abi(b, tt, w_d, rows, cols, mode)
            np.testing.assert_array_equal(got_c, want_c)
            np.testing.assert_array_equal(got_s, want_s)
    assert b.bitnet_get_device_error() == b.BITNET_OK


def test_no_alloc_rejects_bad_shapes_without_touching_the_gpu():
    b = lib()
    st = b.library().bitnet_ternarize_absmean_device_noalloc(16, 4, 100, 0, 16, 16, None)
    assert st == b.BITNET_ERR_SHAPE
