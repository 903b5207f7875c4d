"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the
same seeded inputs.  Integers (packed bytes, q, s, block accumulators) must be
bit-exact; fp32 outputs within 1e-6*|ref| + 1e-6 (and bit-exact where every
block scale of a row is equal, where the library's arithmetic is exact)."""
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


# ------------------------------------------------------------- act quant --

@pytest.mark.parametrize("T,K,outliers", [(1, 128, False), (1, 512, False), (1, 2560, True), (33, 2560, True),
                                          (4, 6912, True), (2, 14336, False), (7, 3200, True),
                                          (300, 1024, True), (3, 32768, True), (2, 32896, True),
                                          (1, 65536, False), (5, 384, True), (17, 4096, False)])
def test_quant_act_bit_exact(T, K, outliers):
    x = syn.activations(syn.seed_for(0, T, K % 997, syn.KIND_ACT), T, K, outliers=outliers)
    q, s, bs = gpu_quant(x)
    rq, rs, rbs = oracle.quant_act(x)
    np.testing.assert_array_equal(to_np(q).reshape(T, K), rq)
    np.testing.assert_array_equal(to_np(s).view(np.uint32), rs.view(np.uint32))
    np.testing.assert_array_equal(to_np(bs).reshape(T, K // QK), rbs)


def test_quant_act_special_rows(golden):
    K = 256
    x = np.zeros((6, K), dtype=np.float32)
    for idx, xv, _ in golden("act_quant_ties.txt"):       # row 0: ties to even
        x[0, int(idx)] = np.float32(float(xv))
    x[2] = syn.normal_f32(5, K) * np.float32(1e-30)          # below the 1e-5 floor
    x[3] = syn.normal_f32(6, K) * np.float32(1e30)           # huge
    x[4, 17] = -3.0                                          # single nonzero
    x[5] = syn.normal_f32(7, K)
    x[5, 100] = np.float32(65504.0)                       # one big outlier
    q, s, bs = gpu_quant(x)
    rq, rs, rbs = oracle.quant_act(x)
    np.testing.assert_array_equal(to_np(q).reshape(6, K), rq)
    np.testing.assert_array_equal(to_np(s), rs)
    np.testing.assert_array_equal(to_np(bs).reshape(6, K // QK), rbs)


def test_quant_act_without_blocksum():
    b = lib()
    tt = torch()
    x = syn.activations(44, 3, 640)
    q = tt.empty(3 * 640, dtype=tt.int8, device="cuda")
    s = tt.empty(3, dtype=tt.float32, device="cuda")
    b.bitnet_quant_act(cuda(x), 3, 640, q, s)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(to_np(q).reshape(3, 640), rq)
    np.testing.assert_array_equal(to_np(s), rs)


# ---------------------------------------------------------------- repack --

@pytest.mark.parametrize("rows,cols", [(1, 128), (17, 512), (256, 512), (1000, 640), (3840, 2560)])
@pytest.mark.parametrize("mode", ["tensor", "row", "block"])
def test_repack_round_trip_and_flags(rows, cols, mode):
    b = lib()
    tt = torch()
    t = syn.ternary_uniform(rows * 7 + cols, rows, cols)
    sc = syn.positive_scales(rows + 3, rows, cols // QK, uniform_per_row=(mode == "row"),
                             per_tensor=(mode == "tensor"))
    w, codes = device_weight(t, sc)
    np.testing.assert_array_equal(codes, oracle.pack_i2s(t))        # packed bytes bit-exact
    assert w.struct.layout_version == b.BITNET_LAYOUT_VERSION
    assert w.uniform == (mode != "block" or cols == QK)
    c2 = tt.empty(rows * cols // 4, dtype=tt.uint8, device="cuda")
    s2 = tt.empty(rows * cols // QK, dtype=tt.float32, device="cuda")
    b.bitnet_unrepack_device(w, c2, s2)
    np.testing.assert_array_equal(to_np(c2).reshape(rows, cols // 4), codes)
    np.testing.assert_array_equal(to_np(s2).reshape(rows, cols // QK), sc)


def test_repack_rejects_code3():
    b = lib()
    tt = torch()
    rows, cols = 40, 256
    codes = np.full((rows, cols // 4), 0x55, dtype=np.uint8)
    codes[37, 50] = 0x57
    data = tt.empty(b.bitnet_repacked_bytes(rows, cols), dtype=tt.uint8, device="cuda")
    with pytest.raises(b.BitnetError) as e:
        b.bitnet_repack_device(cuda(codes.reshape(-1)), cuda(np.ones(rows * 2, np.float32)), rows, cols, data)
    assert e.value.status == b.BITNET_ERR_CORRUPT


# ------------------------------------------------------------------ GEMV --

def _gemv_case(rows, K, B, mode, seed, outliers=True):
    t = syn.ternary_uniform(seed, rows, K)
    sc = syn.positive_scales(seed + 1, rows, K // QK, uniform_per_row=(mode == "row"),
                             per_tensor=(mode == "tensor"))
    x = syn.activations(seed + 2, B, K, outliers=outliers)
    return t, sc, x


def _run_gemv(t, sc, x, with_acc=False, guard=64):
    b = lib()
    tt = torch()
    rows, K = t.shape
    B = x.shape[0]
    w, codes = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ybuf = tt.full((B * rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    y = ybuf[guard:guard + B * rows]
    acc = None
    if with_acc:
        acc = tt.full((B * rows * (K // QK),), -7, dtype=tt.int32, device="cuda")
        b.bitnet_w2a8_gemv_acc(w, q, s, B, y, acc)
    else:
        b.bitnet_w2a8_gemv(w, q, s, B, y)
    yb = to_np(ybuf)
    assert np.all(yb[:guard] == 12345.0) and np.all(yb[guard + B * rows:] == 12345.0), "output guard overwritten"
    return w, codes, to_np(q).reshape(B, K), to_np(s), to_np(y).reshape(B, rows), \
        (to_np(acc).reshape(B, rows, K // QK) if acc is not None else None)


@pytest.mark.parametrize("rows,K,B,mode", [
    (256, 512, 1, "tensor"),      # the 256 x 512 single-GEMV workload
    (256, 512, 1, "block"),
    (1, 128, 1, "tensor"), (17, 128, 16, "block"), (1000, 640, 3, "block"), (33, 384, 5, "row"),
    (3840, 2560, 1, "tensor"), (2560, 2560, 1, "block"), (2560, 6912, 1, "tensor"),
    (2560, 2560, 4, "tensor"), (2560, 2560, 16, "tensor"), (2560, 2560, 16, "block"),
    (777, 1280, 2, "tensor"), (777, 1280, 8, "block"), (4096, 512, 1, "tensor"),
])
def test_gemv_matches_oracle(rows, K, B, mode):
    t, sc, x = _gemv_case(rows, K, B, mode, seed=rows * 31 + K + B)
    w, codes, q, s, y, acc = _run_gemv(t, sc, x, with_acc=True)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    np.testing.assert_array_equal(s, rs)
    ref_acc = oracle.block_acc(oracle.pack_i2s(t), K, rq)
    np.testing.assert_array_equal(acc, ref_acc)
    ref = oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs)
    assert_close(y, ref, f"gemv {rows}x{K} B={B} {mode}")
    if mode != "block":
        np.testing.assert_array_equal(y, ref)   # uniform rows: exact arithmetic end to end
    # The plain entry point (no accumulator export) gives the same y bit for
    # bit, except on uniform rows, where it runs a decode kernel and its fp32
    # epilogue.
    w2, _, _, _, y2, _ = _run_gemv(t, sc, x)
    if w2.uniform:   # every row's block scales equal (any mode when K = 128)
        assert_decode_close(y2, ref, f"decode gemv {rows}x{K} B={B}")
    else:
        np.testing.assert_array_equal(y2, y)


@pytest.mark.parametrize("B", list(range(1, 17)))
def test_gemv_every_batch_size(B):
    rows, K = 200, 768
    t, sc, x = _gemv_case(rows, K, B, "tensor", seed=900 + B)
    _, _, q, s, y, acc = _run_gemv(t, sc, x, with_acc=True)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(acc, oracle.block_acc(oracle.pack_i2s(t), K, rq))
    ref = oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs)
    np.testing.assert_array_equal(y, ref)
    _, _, _, _, y2, _ = _run_gemv(t, sc, x)     # plain entry point: the decode kernels
    assert_decode_close(y2, ref, f"decode gemv B={B}")


def test_gemv_degenerate_weights():
    rows, K, B = 64, 512, 2
    x = syn.activations(5, B, K)
    x[1] = 0.0                                   # all-zero activation row
    for val in (0, 1, -1):
        t = np.full((rows, K), val, dtype=np.int8)
        sc = np.full((rows, K // QK), 0.75, dtype=np.float32)
        _, _, q, s, y, _ = _run_gemv(t, sc, x)
        rq, rs, _ = oracle.quant_act(x)
        np.testing.assert_array_equal(y, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs))
        assert np.all(y[1] == 0.0)
        if val == 0:
            assert np.all(y == 0.0)


def test_gemv_deterministic():
    t, sc, x = _gemv_case(2560, 2560, 4, "block", seed=4242)
    b = lib()
    tt = torch()
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ys = []
    for _ in range(3):
        y = tt.empty(4 * 2560, dtype=tt.float32, device="cuda")
        b.bitnet_w2a8_gemv(w, q, s, 4, y)
        ys.append(to_np(y))
    np.testing.assert_array_equal(ys[0], ys[1])
    np.testing.assert_array_equal(ys[0], ys[2])


# Full-size layers, as the benchmark launches them; the oracle checks a seeded
# sample of output rows (all batch rows) one by one.
FULL_SHAPES = [(3840, 2560), (2560, 2560), (13824, 2560), (2560, 6912), (20480, 3200),
               (6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336)]


@pytest.mark.parametrize("rows,K", FULL_SHAPES)
@pytest.mark.parametrize("B", [1, 4, 16])
def test_gemv_full_size_sampled_rows(rows, K, B):
    t, sc, x = _gemv_case(rows, K, B, "tensor", seed=rows + K)
    _, codes, q, s, y, _ = _run_gemv(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(rows, np.arange(62)) % np.uint64(rows)]))
    pick = pick.astype(np.int64)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    if K <= 16384:                                   # the decode kernels
        assert_decode_close(y[:, pick], ref, f"decode gemv {rows}x{K} B={B}")
    else:
        np.testing.assert_array_equal(y[:, pick], ref)


# ------------------------------------------------------ device ternarise --

def _gpu_ternarize(w, mode):
    b = lib()
    tt = torch()
    rows, cols = w.shape
    codes = tt.empty(rows * cols // 4, dtype=tt.uint8, device="cuda")
    scales = tt.empty(rows * cols // QK, dtype=tt.float32, device="cuda")
    ws = tt.full((b.bitnet_ternarize_workspace_bytes(rows, cols),), 0xAB, dtype=tt.uint8, device="cuda")
    b.bitnet_ternarize_absmean_device(cuda(w.reshape(-1)), rows, cols, mode, codes, scales, ws)
    return to_np(codes).reshape(rows, cols // 4), to_np(scales).reshape(rows, cols // QK)


@pytest.mark.parametrize("rows,cols", [(1, 128), (256, 512), (1000, 640), (3840, 2560), (2560, 6912)])
def test_ternarize_per_block_bit_exact(rows, cols):
    w = syn.normal_matrix(syn.seed_for(2, 0, rows % 251, syn.KIND_WEIGHT), rows, cols)
    w[0, :128] = 0.0                                             # all-zero block -> 1e-5 floor
    codes, scales = _gpu_ternarize(w, lib().BITNET_ABSMEAN_PER_BLOCK)
    t, sc = oracle.absmean_blocks(w)
    np.testing.assert_array_equal(scales, sc)
    np.testing.assert_array_equal(codes, oracle.pack_i2s(t))


@pytest.mark.parametrize("rows,cols", [(256, 512), (3840, 2560), (13824, 2560), (4096, 14336)])
def test_ternarize_per_tensor(rows, cols):
    # gamma is an fp64 sum rounded to fp32; the library adds in a fixed tree
    # order and the oracle left to right, so the two gammas may differ by one
    # fp32 ulp in rare cases.  Then, and only then, codes may differ, and only
    # where |W/gamma| sits at a rounding boundary.
    w = syn.normal_matrix(syn.seed_for(3, 0, rows % 251, syn.KIND_WEIGHT), rows, cols)
    codes, scales = _gpu_ternarize(w, lib().BITNET_ABSMEAN_PER_TENSOR)
    t, g = oracle.absmean_tensor(w)
    assert np.all(scales == scales.flat[0])
    g_gpu = scales.flat[0]
    assert abs(int(g_gpu.view(np.int32)) - int(np.float32(g).view(np.int32))) <= 1
    if g_gpu == g:
        np.testing.assert_array_equal(codes, oracle.pack_i2s(t))
    else:
        t_gpu = oracle.unpack_i2s(codes, cols)
        diff = t_gpu != t
        r = np.abs(w[diff] / np.float32(g))
        assert np.all(np.abs(r - np.round(r - 0.5) - 0.5) < 1e-6)


def test_ternarize_zero_fraction():
    rows, cols = 4096, 4096
    w = syn.normal_matrix(17, rows, cols)
    codes, _ = _gpu_ternarize(w, lib().BITNET_ABSMEAN_PER_TENSOR)
    frac = float(np.mean(oracle.unpack_i2s(codes, cols) == 0))
    assert 0.305 <= frac <= 0.315


# ------------------------------------------------------------------ GEMM --

def _run_gemm(t, sc, x, with_acc=False, guard=64):
    b = lib()
    tt = torch()
    rows, K = t.shape
    T = x.shape[0]
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ybuf = tt.full((T * rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    y = ybuf[guard:guard + T * rows]
    acc = None
    if with_acc:
        acc = tt.full((T * rows * (K // QK),), -7, dtype=tt.int32, device="cuda")
        b.bitnet_w2a8_gemm_acc(w, q, s, T, y, acc)
    else:
        b.bitnet_w2a8_gemm(w, q, s, T, y)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    yb = to_np(ybuf)
    assert np.all(yb[:guard] == 12345.0) and np.all(yb[guard + T * rows:] == 12345.0), "output guard overwritten"
    return w, to_np(q).reshape(T, K), to_np(s), to_np(y).reshape(T, rows), \
        (to_np(acc).reshape(T, rows, K // QK) if acc is not None else None)


@pytest.mark.parametrize("rows,K,T,mode", [
    (256, 512, 40, "tensor"), (256, 512, 40, "block"),
    (1, 128, 1, "tensor"), (17, 128, 33, "block"), (100, 384, 129, "tensor"), (1000, 640, 200, "row"),
    (300, 256, 512, "tensor"), (2560, 2560, 256, "tensor"), (2560, 2560, 256, "block"),
])
def test_gemm_matches_oracle(rows, K, T, mode):
    t, sc, x = _gemv_case(rows, K, T, mode, seed=rows * 17 + K + T)
    _, q, s, y, _ = _run_gemm(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    ref = oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs)
    assert_close(y, ref, f"gemm {rows}x{K} T={T} {mode}")


@pytest.mark.parametrize("rows,K,T", [(64, 256, 1), (200, 384, 130), (513, 1280, 77)])
def test_gemm_block_accumulators_bit_exact(rows, K, T):
    t, sc, x = _gemv_case(rows, K, T, "block", seed=rows + 5 * K + T)
    _, q, s, y, acc = _run_gemm(t, sc, x, with_acc=True)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(acc, oracle.block_acc(oracle.pack_i2s(t), K, rq))
    assert_close(y, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), "gemm_acc y")


def test_gemm_agrees_with_gemv_on_small_batches():
    rows, K = 2560, 2560
    for T in (1, 5, 16):
        t, sc, x = _gemv_case(rows, K, T, "tensor", seed=31 + T)
        _, _, _, _, yg, _ = _run_gemv(t, sc, x)
        _, _, _, ym, _ = _run_gemm(t, sc, x)
        assert_close(ym, yg, f"gemm vs gemv T={T}")


@pytest.mark.parametrize("rows,K,T", [(13824, 2560, 512), (2560, 6912, 512), (13824, 2560, 2048),
                                      (2560, 6912, 2048), (28672, 4096, 1024), (4096, 14336, 1024)])
def test_gemm_full_size_sampled(rows, K, T):
    # Full-size prefill as the benchmark launches it; the oracle checks a
    # seeded sample of output rows for every token.
    t, sc, x = _gemv_case(rows, K, T, "tensor", seed=rows ^ K ^ T, outliers=True)
    _, q, s, y, _ = _run_gemm(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(rows + T, np.arange(30)) % np.uint64(rows)]))
    pick = pick.astype(np.int64)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    assert_close(y[:, pick], ref, f"gemm full {rows}x{K} T={T}")


def test_gemm_zero_tokens_is_a_no_op():
    b = lib()
    tt = torch()
    t, sc, x = _gemv_case(64, 256, 1, "tensor", seed=3)
    w, _ = device_weight(t, sc)
    y = tt.full((64,), 5.0, device="cuda")
    q = tt.zeros(256, dtype=tt.int8, device="cuda")
    s = tt.ones(1, device="cuda")
    b.bitnet_w2a8_gemm(w, q, s, 0, y)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    assert np.all(to_np(y) == 5.0)


# ---------------------------------------------------- fused decode linear --

def _run_linear(t, sc, x, with_acc=False, guard=64):
    b = lib()
    tt = torch()
    rows, K = t.shape
    B = x.shape[0]
    w, _ = device_weight(t, sc)
    xd = cuda(x.astype(np.float32).reshape(-1))
    ybuf = tt.full((B * rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    y = ybuf[guard:guard + B * rows]
    q = tt.full((B * K,), 99, dtype=tt.int8, device="cuda")
    s = tt.full((B,), -1.0, dtype=tt.float32, device="cuda")
    acc = None
    if with_acc:
        acc = tt.full((B * rows * (K // QK),), -7, dtype=tt.int32, device="cuda")
        b.bitnet_w2a8_linear_acc(w, xd, B, y, acc, q, s)
    else:
        b.bitnet_w2a8_linear(w, xd, B, y, q, s)
    yb = to_np(ybuf)
    assert np.all(yb[:guard] == 12345.0) and np.all(yb[guard + B * rows:] == 12345.0), "output guard overwritten"
    return to_np(q).reshape(B, K), to_np(s), to_np(y).reshape(B, rows), \
        (to_np(acc).reshape(B, rows, K // QK) if acc is not None else None)


@pytest.mark.parametrize("rows,K,B,mode", [
    (256, 512, 1, "tensor"), (256, 512, 1, "block"), (1, 128, 1, "tensor"), (17, 128, 16, "block"),
    (1000, 640, 3, "block"), (3840, 2560, 1, "tensor"), (2560, 6912, 1, "tensor"), (2560, 2560, 16, "tensor"),
    (777, 1280, 8, "row"), (4096, 14336, 4, "tensor"), (2560, 14336, 16, "block"),
])
def test_linear_matches_oracle_and_gemv(rows, K, B, mode):
    t, sc, x = _gemv_case(rows, K, B, mode, seed=rows * 13 + K + B)
    q, s, y, acc = _run_linear(t, sc, x, with_acc=True)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    np.testing.assert_array_equal(s.view(np.uint32), rs.view(np.uint32))
    np.testing.assert_array_equal(acc, oracle.block_acc(oracle.pack_i2s(t), K, rq))
    ref = oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs)
    assert_close(y, ref, f"linear {rows}x{K} B={B} {mode}")
    if mode != "block":
        np.testing.assert_array_equal(y, ref)
    wg, _, _, _, yg, _ = _run_gemv(t, sc, x)           # same arithmetic as quant_act + gemv
    q2, s2, y2, _ = _run_linear(t, sc, x)              # plain entry point, q_out / s_out given
    np.testing.assert_array_equal(q2, rq)
    # B = 1: the fused decode kernel; B >= 2: the quantiser, then the GEMV's
    # own dispatch on the same q, s -- the same y as the GEMV, bit for bit.
    np.testing.assert_array_equal(y2, yg)
    if wg.uniform and (K <= 16384 or B >= 8):          # decode or tensor-core kernels: fp32 epilogue
        assert_decode_close(yg, ref, f"gemv {rows}x{K} B={B}")
    else:                                              # the general kernel: exact
        np.testing.assert_array_equal(yg, y)


@pytest.mark.parametrize("B", list(range(1, 17)))
def test_linear_every_batch_size(B):
    rows, K = 300, 1024
    t, sc, x = _gemv_case(rows, K, B, "tensor", seed=1700 + B)
    q, s, y, _ = _run_linear(t, sc, x)                 # q_out / s_out given: fp32-epilogue kernels
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    ref = oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs)
    assert_decode_close(y, ref, f"linear B={B}")


def test_linear_optional_outputs_and_zero_rows():
    b = lib()
    tt = torch()
    rows, K, B = 64, 512, 3
    t, sc, x = _gemv_case(rows, K, B, "tensor", seed=91)
    x[1] = 0.0
    w, _ = device_weight(t, sc)
    y = tt.empty(B * rows, dtype=tt.float32, device="cuda")
    b.bitnet_w2a8_linear(w, cuda(x.reshape(-1)), B, y)            # no q/s outputs
    rq, rs, _ = oracle.quant_act(x)
    got = to_np(y).reshape(B, rows)
    np.testing.assert_array_equal(got, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs))
    assert np.all(got[1] == 0.0)


@pytest.mark.parametrize("rows,K", [(3840, 2560), (13824, 2560), (2560, 6912), (28672, 4096), (4096, 14336)])
@pytest.mark.parametrize("B", [1, 16])
def test_linear_full_size_sampled_rows(rows, K, B):
    t, sc, x = _gemv_case(rows, K, B, "tensor", seed=rows + 3 * K + B)
    q, s, y, _ = _run_linear(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(rows ^ B, np.arange(40)) % np.uint64(rows)]))
    pick = pick.astype(np.int64)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    assert_decode_close(y[:, pick], ref, f"linear {rows}x{K} B={B}")


# ------------------------------------------------ table-lookup GEMV variant --

def _run_lut(t, sc, x, guard=64):
    b = lib()
    tt = torch()
    rows, K = t.shape
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    ybuf = tt.full((rows + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    y = ybuf[guard:guard + rows]
    b.bitnet_w2a8_gemv_lut(w, q, s, y)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    yb = to_np(ybuf)
    assert np.all(yb[:guard] == 12345.0) and np.all(yb[guard + rows:] == 12345.0), "output guard overwritten"
    return to_np(q).reshape(1, K), to_np(s), to_np(y).reshape(1, rows)


@pytest.mark.parametrize("rows,K,mode", [
    (256, 512, "tensor"), (1, 128, "tensor"), (17, 256, "row"), (300, 1024, "tensor"), (777, 1280, "row"),
    (3840, 2560, "tensor"), (2560, 6912, "tensor"), (4096, 8192, "tensor"), (7109, 640, "tensor"),
])
def test_lut_gemv_matches_oracle(rows, K, mode):
    t, sc, x = _gemv_case(rows, K, 1, mode, seed=rows * 7 + K)
    q, s, y = _run_lut(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(q, rq)
    assert_decode_close(y, oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs), f"lut {rows}x{K}")


def test_lut_gemv_full_size_sampled_rows():
    rows, K = 13824, 2560
    t, sc, x = _gemv_case(rows, K, 1, "tensor", seed=4711)
    q, s, y = _run_lut(t, sc, x)
    rq, rs, _ = oracle.quant_act(x)
    pick = np.unique(np.concatenate([[0, rows - 1], syn.splitmix64(rows, np.arange(60)) % np.uint64(rows)]))
    pick = pick.astype(np.int64)
    ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
    assert_decode_close(y[:, pick], ref, "lut full size")


def test_lut_gemv_rejects_block_scales():
    b = lib()
    tt = torch()
    t, sc, x = _gemv_case(64, 512, 1, "block", seed=5)
    w, _ = device_weight(t, sc)
    q, s, _ = gpu_quant(x)
    y = tt.empty(64, dtype=tt.float32, device="cuda")
    with pytest.raises(b.BitnetError) as e:
        b.bitnet_w2a8_gemv_lut(w, q, s, y)
    assert e.value.status == b.BITNET_ERR_UNSUPPORTED
