"""Pins for the CPU oracle, checked against what the pages and mathematics fix.

None of these compares the oracle with itself: the expected values come from
hand-worked bytes printed in ``tests/golden`` (with their page citations),
closed forms, invariants, exact library sums, and a brute-force fp64 matmul on
tiny shapes.  Each is chosen so that a plausible slip in the oracle (a wrong
shift, a swapped code, a transposed operand, a dropped scale, the wrong
rounding mode) fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synthetic as syn


# ---------------------------------------------------------------- i2_s pack --

def _hand_block(golden):
    rows = golden("i2s_hand_byte.txt")
    cols = int(rows[0][1])
    t = np.zeros((1, cols), dtype=np.int8)
    expected = None
    for r in rows[1:]:
        if r[0] == "weight":
            t[0, int(r[1])] = int(r[2])
        elif r[0] == "bytes":
            expected = np.array([int(v, 16) for v in r[1:]], dtype=np.uint8)
    return t, expected


def test_pack_hand_worked_byte(golden):
    t, expected = _hand_block(golden)
    codes = oracle.pack_i2s(t)
    assert codes.shape == (1, 32)
    np.testing.assert_array_equal(codes[0], expected)


def test_pack_closed_forms(golden):
    for value, byte in golden("i2s_closed_forms.txt"):
        for rows, cols in [(1, 128), (3, 512), (5, 2560)]:
            t = np.full((rows, cols), int(value), dtype=np.int8)
            codes = oracle.pack_i2s(t)
            assert codes.shape == (rows, cols // 4)
            assert np.all(codes == int(byte, 16)), (value, byte)


def test_row_stride(golden):
    for cols, bpr, spr in golden("row_stride.txt"):
        cols, bpr, spr = int(cols), int(bpr), int(spr)
        # Two rows that differ: row 1 must start exactly cols/4 bytes in.
        t = np.zeros((2, cols), dtype=np.int8)
        t[1, :] = 1
        codes = oracle.pack_i2s(t)
        flat = codes.reshape(-1)
        assert flat.size == 2 * bpr
        assert np.all(flat[:bpr] == 0x55) and np.all(flat[bpr:] == 0xAA)
        t2, sc = oracle.absmean_blocks(np.ones((1, cols), dtype=np.float32))
        assert sc.shape == (1, spr)


def test_pack_single_weight_positions():
    # A lone +1 at position i of a block sets code 2 at byte i%32, shift 6-2*(i//32);
    # every other 2-bit field of the block stays code 1.
    for i in [0, 1, 31, 32, 33, 63, 64, 95, 96, 127]:
        t = np.zeros((1, 256), dtype=np.int8)
        t[0, 128 + i] = 1
        codes = oracle.pack_i2s(t)[0]
        assert np.all(codes[:32] == 0x55)
        blk = codes[32:]
        shift = 6 - 2 * (i // 32)
        for b in range(32):
            want = 0x55
            if b == i % 32:
                want = (0x55 & ~(3 << shift)) | (2 << shift)
            assert blk[b] == want, (i, b, hex(blk[b]), hex(want))


def test_pack_unpack_round_trip():
    for seed, (rows, cols) in enumerate([(1, 128), (7, 384), (33, 2560), (16, 6912)]):
        t = syn.ternary_uniform(100 + seed, rows, cols)
        codes = oracle.pack_i2s(t)
        assert codes.dtype == np.uint8 and codes.shape == (rows, cols // 4)
        np.testing.assert_array_equal(oracle.unpack_i2s(codes, cols), t)


def test_pack_rejects_non_ternary():
    t = np.zeros((2, 128), dtype=np.int8)
    t[1, 5] = 2
    assert oracle.pack_status(t) == oracle.BAD_VALUE
    t[1, 5] = -2
    assert oracle.pack_status(t) == oracle.BAD_VALUE


def test_unpack_rejects_code_3():
    codes = np.full((2, 32), 0x55, dtype=np.uint8)
    codes[1, 7] = 0x57  # lowest field = 3
    assert oracle.unpack_status(codes, 128) == oracle.CORRUPT
    codes[1, 7] = 0xD5  # highest field = 3
    assert oracle.unpack_status(codes, 128) == oracle.CORRUPT


def test_shape_rejected():
    t = np.zeros((1, 100), dtype=np.int8)
    assert oracle.pack_status(t) == oracle.BAD_SHAPE


# ------------------------------------------------------------- absmean ternary --

def test_absmean_zero_fraction_matches_normal_closed_form():
    # For W ~ N(0,1), gamma -> E|W| = sqrt(2/pi) and t = 0 iff |W| < gamma/2, so the
    # zero fraction tends to 2*Phi(sqrt(2/pi)/2) - 1 = 0.3101 (binomial sd ~2e-4 here).
    w = syn.normal_f32(syn.seed_for(9, 0, 0), 1 << 22)
    t, g = oracle.absmean_tensor(w)
    expected = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    assert abs(expected - 0.3101) < 1e-4
    frac = float(np.mean(t == 0))
    assert 0.305 <= frac <= 0.315, frac
    assert abs(frac - expected) < 2e-3
    assert set(np.unique(t).tolist()) == {-1, 0, 1}
    assert abs(float(g) - math.sqrt(2 / math.pi)) < 2e-3


def test_absmean_gamma_is_exact_mean_rounded():
    for seed, n in [(1, 1000), (2, 4096 * 3), (3, 1 << 20)]:
        w = syn.normal_f32(seed, n) * np.float32(0.02)
        _, g = oracle.absmean_tensor(w)
        exact = math.fsum(abs(float(v)) for v in w) / n
        assert g == np.float32(exact), (g, exact)


def test_absmean_closed_forms():
    # |w| constant = c: gamma = c and t = sign(w).
    c = np.float32(0.37)
    sgn = np.where(syn.ternary_uniform(5, 4, 256, p_zero=0.0) > 0, 1, -1).astype(np.float32)
    t, g = oracle.absmean_tensor(sgn * c)
    assert g == c
    np.testing.assert_array_equal(t, sgn.astype(np.int8))
    # [2, 0, 0, 0] repeated: gamma = 0.5, t = [1, 0, 0, 0].
    w = np.tile(np.array([2, 0, 0, 0], dtype=np.float32), 64)
    t, g = oracle.absmean_tensor(w)
    assert g == np.float32(0.5)
    np.testing.assert_array_equal(t, np.tile(np.array([1, 0, 0, 0], dtype=np.int8), 64))


def test_absmean_ties_and_clamp():
    # mean |w| = 1 exactly, so w/gamma = w: 0.5 -> 0 and -0.5 -> 0 (ties to even),
    # 1.5 -> 2 -> clamped to 1, 2.5 -> 2 -> 1, 1.0 -> 1.
    w = np.array([0.5, -0.5, 1.5, 1.5, 2.5, 0.5, 0.5, 0.5, 1.0, -1.0, 1.0, -1.0], dtype=np.float32)
    t, g = oracle.absmean_tensor(w)
    assert g == np.float32(1.0)
    np.testing.assert_array_equal(t, np.array([0, 0, 1, 1, 1, 0, 0, 0, 1, -1, 1, -1], dtype=np.int8))


def test_absmean_all_zero_floor():
    t, g = oracle.absmean_tensor(np.zeros(512, dtype=np.float32))
    assert g == np.float32(1e-5)
    assert np.all(t == 0)


def test_absmean_blocks_scales():
    w = syn.normal_matrix(77, 3, 384)
    w[1, 128:256] = 0.0
    w[2, 256:] *= np.float32(10.0)
    t, sc = oracle.absmean_blocks(w)
    for o in range(3):
        for j in range(3):
            blk = w[o, 128 * j:128 * (j + 1)]
            exact = math.fsum(abs(float(v)) for v in blk) / 128
            want = max(np.float32(exact), np.float32(1e-5))
            assert sc[o, j] == want
    assert np.all(t[1, 128:256] == 0)


# ----------------------------------------------------------------- act quant --

def test_act_quant_ties_to_even(golden):
    rows = golden("act_quant_ties.txt")
    x = np.zeros((1, 128), dtype=np.float32)
    want = np.zeros(128, dtype=np.int8)
    for idx, xv, qv in rows:
        x[0, int(idx)] = np.float32(float(xv))
        want[int(idx)] = int(qv)
    q, s, bs = oracle.quant_act(x)
    assert s[0] == np.float32(1.0)
    np.testing.assert_array_equal(q[0], want)
    assert bs[0, 0] == int(want.astype(np.int64).sum())


def test_act_quant_extreme_and_bound():
    x = syn.activations(11, 6, 2560, outliers=True)
    x[3] *= np.float32(1e-3)
    q, s, bs = oracle.quant_act(x)
    for b in range(x.shape[0]):
        k = int(np.argmax(np.abs(x[b])))
        assert abs(int(q[b, k])) == 127 and np.sign(q[b, k]) == np.sign(x[b, k])
        # |x - q/s| <= 0.5/s (one rounding of the product; tiny slack for the fp32 multiply)
        err = np.abs(x[b].astype(np.float64) - q[b].astype(np.float64) / np.float64(s[b]))
        assert np.all(err <= 0.5 / np.float64(s[b]) * (1 + 1e-6))
        m = np.float64(np.max(np.abs(x[b])))
        assert abs(np.float64(s[b]) - 127.0 / m) <= 127.0 / m * 2**-23
    assert np.all(np.abs(q) <= 127)
    np.testing.assert_array_equal(bs, q.astype(np.int64).reshape(6, -1, 128).sum(-1))


def test_act_quant_all_zero_row():
    x = np.zeros((2, 256), dtype=np.float32)
    x[1, 3] = 1.0
    q, s, bs = oracle.quant_act(x)
    assert np.all(q[0] == 0) and np.all(bs[0] == 0)
    assert s[0] == np.float32(127.0) / np.float32(1e-5)
    assert q[1, 3] == 127 and s[1] == np.float32(127.0)


# ------------------------------------------------------ dot and the epilogue --

def _pack_rows(t):
    return oracle.pack_i2s(t)


def test_linear_all_zero_weights():
    x = syn.activations(3, 4, 512)
    q, s, _ = oracle.quant_act(x)
    codes = _pack_rows(np.zeros((9, 512), dtype=np.int8))
    sc = np.full((9, 4), 0.7, dtype=np.float32)
    y = oracle.linear(codes, sc, 512, q, s)
    assert np.all(y == 0.0)


@pytest.mark.parametrize("sign", [1, -1])
def test_linear_all_pm1_closed_form(sign):
    x = syn.activations(4, 3, 640 * 2)
    q, s, _ = oracle.quant_act(x)
    K = x.shape[1]
    g = np.float32(0.8125)
    codes = _pack_rows(np.full((5, K), sign, dtype=np.int8))
    sc = np.full((5, K // 128), g, dtype=np.float32)
    y = oracle.linear(codes, sc, K, q, s)
    for b in range(3):
        want = np.float32(sign * float(g) * int(q[b].astype(np.int64).sum()) / float(s[b]))
        assert np.all(y[b] == want)


def test_linear_single_weight():
    x = syn.activations(5, 2, 512)
    q, s, _ = oracle.quant_act(x)
    for o_star, k_star, v in [(0, 0, 1), (6, 511, -1), (3, 200, 1)]:
        t = np.zeros((7, 512), dtype=np.int8)
        t[o_star, k_star] = v
        sc = syn.normal_matrix(6, 7, 4).__abs__() + np.float32(0.1)
        y = oracle.linear(_pack_rows(t), sc, 512, q, s)
        for b in range(2):
            for o in range(7):
                want = 0.0
                if o == o_star:
                    want = v * float(sc[o, k_star // 128]) * int(q[b, k_star]) / float(s[b])
                assert y[b, o] == np.float32(want)


def test_linear_single_activation():
    # x = a * e_k: q_k = sign(a) * 127, s = 127/|a|, so y_o = t[o][k] * scale * a.
    K, rows = 384, 11
    t = syn.ternary_uniform(8, rows, K)
    sc = np.abs(syn.normal_matrix(9, rows, K // 128)) + np.float32(0.05)
    codes = _pack_rows(t)
    for k, a in [(0, 3.25), (200, -0.0078125), (383, 1000.0)]:
        x = np.zeros((1, K), dtype=np.float32)
        x[0, k] = a
        q, s, _ = oracle.quant_act(x)
        assert q[0, k] == (127 if a > 0 else -127)
        y = oracle.linear(codes, sc, K, q, s)
        for o in range(rows):
            want = t[o, k] * float(sc[o, k // 128]) * a
            assert abs(float(y[0, o]) - want) <= 1e-6 * abs(want) + 1e-30


def test_block_acc_matches_integer_matmul():
    rows, K, T = 37, 640, 5
    t = syn.ternary_uniform(12, rows, K)
    x = syn.activations(13, T, K, outliers=True)
    q, s, _ = oracle.quant_act(x)
    acc = oracle.block_acc(_pack_rows(t), K, q)
    ref = np.einsum("bjk,ojk->boj", q.astype(np.int64).reshape(T, K // 128, 128),
                    t.astype(np.int64).reshape(rows, K // 128, 128))
    np.testing.assert_array_equal(acc, ref)
    assert np.max(np.abs(acc)) <= 128 * 127


@pytest.mark.parametrize("rows,K,T", [(48, 384, 5), (17, 1024, 3), (256, 512, 1)])
def test_linear_brute_force_fp64(rows, K, T):
    # Dequantise both sides and multiply in fp64 with a library matmul.
    t = syn.ternary_uniform(20 + rows, rows, K)
    sc = (np.abs(syn.normal_matrix(21 + rows, rows, K // 128)) + np.float32(0.01)).astype(np.float32)
    x = syn.activations(22 + rows, T, K, outliers=True)
    q, s, _ = oracle.quant_act(x)
    y, y64 = oracle.linear(_pack_rows(t), sc, K, q, s, want_f64=True)
    w_deq = t.astype(np.float64) * np.repeat(sc.astype(np.float64), 128, axis=1)
    a_deq = q.astype(np.float64) / s.astype(np.float64)[:, None]
    ref = a_deq @ w_deq.T
    mag = np.abs(a_deq) @ np.abs(w_deq).T
    assert np.all(np.abs(y64 - ref) <= 1e-12 * mag + 1e-300)
    np.testing.assert_array_equal(y, y64.astype(np.float32))
