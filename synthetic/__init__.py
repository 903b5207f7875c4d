"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the
W2A8 method's arithmetic (no ternarisation, no packing, no quantisation).
Both the CPU oracle and the CUDA library receive the arrays it returns.

Generator (counter based, so any element can be regenerated from its index):
  * splitmix64 on the counter ``seed + (i + 1) * 0x9E3779B97F4A7C15``;
  * 53-bit uniforms: u1 = ((z >> 11) + 1) * 2**-53 in (0, 1],
    u2 = (z >> 11) * 2**-53 in [0, 1);
  * Box-Muller in fp64 on the pair (2p, 2p+1): element 2p gets r*cos(theta),
    element 2p+1 gets r*sin(theta); the result is rounded once to fp32.

Seeds: ``seed_for(config, layer, matrix_id, kind)`` =
``0xB17E7 ^ (config << 40) ^ (layer << 24) ^ (matrix_id << 16) ^ kind``.
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

KIND_WEIGHT = 1
KIND_ACT = 2
KIND_OUTLIER = 3


def seed_for(config: int, layer: int = 0, matrix_id: int = 0, kind: int = KIND_WEIGHT) -> int:
    return (0xB17E7 ^ (config << 40) ^ (layer << 24) ^ (matrix_id << 16) ^ kind) & (2**64 - 1)


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """splitmix64 output for each counter value (uint64 array)."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + (counters.astype(np.uint64) + np.uint64(1)) * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * M1
        z = (z ^ (z >> np.uint64(27))) * M2
        z = z ^ (z >> np.uint64(31))
    return z


def normal_f32(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Elements [start, start+n) of the seeded N(0,1) stream, as float32."""
    if n <= 0:
        return np.zeros(0, dtype=np.float32)
    first_pair = start // 2
    last_pair = (start + n - 1) // 2
    pairs = np.arange(first_pair, last_pair + 1, dtype=np.uint64)
    z1 = splitmix64(seed, 2 * pairs)
    z2 = splitmix64(seed, 2 * pairs + np.uint64(1))
    u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0**-53
    u2 = (z2 >> np.uint64(11)).astype(np.float64) * 2.0**-53
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * np.pi * u2
    out = np.empty(2 * pairs.size, dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    off = start - 2 * first_pair
    return out[off:off + n].astype(np.float32)


def normal_matrix(seed: int, rows: int, cols: int) -> np.ndarray:
    return normal_f32(seed, rows * cols).reshape(rows, cols)


def outlier_channels(seed: int, K: int, frac: float = 0.01) -> np.ndarray:
    """floor(frac*K) channel indices, chosen by ranking splitmix64(seed, k)."""
    n = int(np.floor(frac * K))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    keys = splitmix64(seed, np.arange(K, dtype=np.uint64))
    return np.sort(np.argsort(keys, kind="stable")[:n]).astype(np.int64)


def activations(seed: int, T: int, K: int, outliers: bool = False, outlier_seed: int | None = None,
                factor: float = 20.0) -> np.ndarray:
    """fp32 N(0,1) activations [T][K]; optionally a fixed 1% of channels x factor."""
    x = normal_matrix(seed, T, K)
    if outliers:
        ch = outlier_channels(outlier_seed if outlier_seed is not None else seed ^ KIND_OUTLIER, K)
        x[:, ch] *= np.float32(factor)
    return x


def ternary_uniform(seed: int, rows: int, cols: int, p_zero: float = 0.31) -> np.ndarray:
    """Random values in {-1, 0, +1} drawn directly (for layout and corner tests)."""
    z = splitmix64(seed, np.arange(rows * cols, dtype=np.uint64))
    u = (z >> np.uint64(11)).astype(np.float64) * 2.0**-53
    t = np.where(u < p_zero, 0, np.where(u < p_zero + (1 - p_zero) / 2, -1, 1))
    return t.astype(np.int8).reshape(rows, cols)


def positive_scales(seed: int, rows: int, nb: int, uniform_per_row: bool = False,
                    per_tensor: bool = False) -> np.ndarray:
    """fp32 block scales [rows][nb] in [0.25, 4): 2**(4u - 2) for seeded uniforms u.

    per_tensor: one value for the whole matrix; uniform_per_row: one value per row.
    """
    n = 1 if per_tensor else (rows if uniform_per_row else rows * nb)
    z = splitmix64(seed, np.arange(n, dtype=np.uint64))
    u = (z >> np.uint64(11)).astype(np.float64) * 2.0**-53
    v = np.exp2(4.0 * u - 2.0).astype(np.float32)
    if per_tensor:
        return np.full((rows, nb), v[0], dtype=np.float32)
    if uniform_per_row:
        return np.repeat(v[:, None], nb, axis=1)
    return v.reshape(rows, nb)


def integer_rows(seed: int, T: int, K: int, peak: int = 127) -> np.ndarray:
    """fp32 rows [T][K] of integers drawn uniformly from [-peak, peak], with
    element (t, splitmix64 pick) of every row set to +-peak, so each row's
    largest magnitude is exactly `peak`."""
    z = splitmix64(seed, np.arange(T * K, dtype=np.uint64))
    x = ((z % np.uint64(2 * peak + 1)).astype(np.int64) - peak).reshape(T, K)
    pick = splitmix64(seed ^ 0x5EED, np.arange(T, dtype=np.uint64))
    col = (pick % np.uint64(K)).astype(np.int64)
    sign = np.where((pick >> np.uint64(32)) & np.uint64(1), -1, 1)
    x[np.arange(T), col] = sign * peak
    return x.astype(np.float32)


def _as_i64(v: int) -> int:
    """The two's-complement int64 with the same 64 bits as the uint64 v."""
    v &= 2**64 - 1
    return v - 2**64 if v >= 2**63 else v


def normal_device(seed: int, n: int, device, chunk: int = 1 << 24):
    """The same N(0,1) stream as normal_f32(seed, n), drawn with torch on
    `device` (for the benchmark's multi-gigabyte weight sets).  splitmix64 runs
    in int64 (wrapping multiply; right shifts masked to be logical); the
    Box-Muller step runs in fp64 with torch's log/cos/sin, so an element may
    differ from the host stream in its last fp32 bit."""
    import torch
    out = torch.empty(n, dtype=torch.float32, device=device)
    g, m1, m2 = _as_i64(int(GOLDEN)), _as_i64(int(M1)), _as_i64(int(M2))

    def lsr(z, k):
        return (z >> k) & ((1 << (64 - k)) - 1)

    def mix(cnt):
        z = cnt.add(1).mul_(g).add_(_as_i64(seed))
        z = (z ^ lsr(z, 30)).mul_(m1)
        z = (z ^ lsr(z, 27)).mul_(m2)
        return z ^ lsr(z, 31)

    for p0 in range(0, (n + 1) // 2, chunk):
        p1 = min((n + 1) // 2, p0 + chunk)
        pairs = torch.arange(p0, p1, dtype=torch.int64, device=device)
        u1 = (lsr(mix(2 * pairs), 11).double() + 1.0) * 2.0**-53
        u2 = lsr(mix(2 * pairs + 1), 11).double() * 2.0**-53
        r = torch.sqrt(-2.0 * torch.log(u1))
        th = 2.0 * torch.pi * u2
        pair_out = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).reshape(-1).float()
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = pair_out[: hi - lo]
    return out
