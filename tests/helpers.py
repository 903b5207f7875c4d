"""Shared helpers for the GPU tests: seeded inputs go to both the CUDA library
(through its C ABI binding) and the CPU oracle, never from one to the other."""
from __future__ import annotations

import numpy as np

import oracle
import synthetic as syn

QK = 128


def lib():
    import ternary_weight_absmax_b200 as b
    return b


def torch():
    import torch as _t
    return _t


def cuda(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def to_np(t):
    return t.detach().cpu().numpy()


def device_weight(t_host: np.ndarray, scales: np.ndarray):
    """Pack (library host packer), upload, repack.  Returns (Weight, codes)."""
    b = lib()
    rows, cols = t_host.shape
    codes = b.bitnet_pack_i2s(t_host)
    codes_d = cuda(codes.reshape(-1))
    scales_d = cuda(np.ascontiguousarray(scales, dtype=np.float32).reshape(-1))
    data = torch().empty(b.bitnet_repacked_bytes(rows, cols), dtype=torch().uint8, device="cuda")
    w = b.bitnet_repack_device(codes_d, scales_d, rows, cols, data)
    return w, codes


def gpu_quant(x: np.ndarray):
    """Library act-quant of host x -> (q_dev, s_dev, blocksum_dev)."""
    b = lib()
    T, K = x.shape
    tt = torch()
    xd = cuda(x.astype(np.float32))
    q = tt.empty(T * K, dtype=tt.int8, device="cuda")
    s = tt.empty(T, dtype=tt.float32, device="cuda")
    bs = tt.empty(T * (K // QK), dtype=tt.int32, device="cuda")
    b.bitnet_quant_act(xd, T, K, q, s, bs)
    return q, s, bs


def tolerance_ok(y, ref, rel=1e-6, abs_=1e-6):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.abs(y - ref) <= rel * np.abs(ref) + abs_


def assert_close(y, ref, what=""):
    ok = tolerance_ok(y, ref)
    if not np.all(ok):
        bad = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outside 1e-6*|ref|+1e-6; "
                             f"first {bad.tolist()} y={np.asarray(y)[tuple(bad.T)]} ref={np.asarray(ref)[tuple(bad.T)]}")


def assert_decode_close(y, ref, what=""):
    """Outputs of the batch-1 decode kernel (uniform rows), whose epilogue runs
    in fp32: rowscale * sum * (1/s) with three roundings, so within 3 * 2^-24
    of the exact value and within 4e-7 of the fp64 oracle (tighter than the
    1e-6*|ref| + 1e-6 bar, which it must also meet).  Zero sums give zero."""
    assert_close(y, ref, what)
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    zero = ref == 0.0
    assert np.all(y[zero] == 0.0), f"{what}: nonzero output where the oracle gives 0"
    rel = np.abs(y[~zero] - ref[~zero]) / np.abs(ref[~zero])
    assert rel.size == 0 or rel.max() <= 4e-7, f"{what}: relative error {rel.max():.3e} above 4e-7"
