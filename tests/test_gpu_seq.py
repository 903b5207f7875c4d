"""GPU parity of bitnet_w2a8_linear_seq, the persistent kernel that runs a list
of batch-1 decode linears: every entry against the oracle (the fp32 decode
epilogue's tolerance), against bitnet_w2a8_linear called once per entry (bit
for bit: the same arithmetic), and with unit scales and s = 1 against the
exact int32 sums.  Lists without waits, chains where each x is part of the
previous y, mixed waves, ragged shapes, repeated calls on one workspace and a
forced timeout are covered."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from helpers import QK, assert_decode_close, cuda, device_weight, lib, to_np, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert lib().bitnet_get_device_error() == lib().BITNET_OK


def _weights(shapes, seed, unit=False):
    out = []
    for i, (rows, K) in enumerate(shapes):
        t = syn.ternary_uniform(seed + 17 * i, rows, K)
        sc = np.ones((rows, K // QK), np.float32) if unit else \
            syn.positive_scales(seed + 17 * i + 1, rows, K // QK, per_tensor=True)
        w, _ = device_weight(t, sc)
        out.append((t, sc, w))
    return out


def _workspace(n):
    tt = torch()
    return tt.zeros(lib().bitnet_w2a8_linear_seq_workspace_bytes(n), dtype=tt.uint8, device="cuda")


def _guarded(n, guard=32):
    tt = torch()
    buf = tt.full((n + 2 * guard,), 12345.0, dtype=tt.float32, device="cuda")
    return buf, buf[guard:guard + n]


def _check_guard(buf, n, guard=32):
    b = to_np(buf)
    assert np.all(b[:guard] == 12345.0) and np.all(b[guard + n:] == 12345.0), "output guard overwritten"


def _pick(rows, seed, n=40):
    if rows <= 4096:
        return np.arange(rows)
    p = np.concatenate([[0, rows - 1], syn.splitmix64(seed, np.arange(n)) % np.uint64(rows)])
    return np.unique(p).astype(np.int64)


INDEP = [(256, 512), (1, 128), (17, 128), (300, 1024), (777, 1280), (3840, 2560), (2560, 2560),
         (13824, 2560), (2560, 6912), (4096, 14336), (100, 16384)]


def test_seq_independent_matches_oracle_and_per_call():
    b = lib()
    tt = torch()
    ws = _weights(INDEP, 5100)
    xs, ys, bufs = [], [], []
    for i, (rows, K) in enumerate(INDEP):
        xs.append(syn.activations(syn.seed_for(1, i, 0, syn.KIND_ACT), 1, K, outliers=True))
        buf, y = _guarded(rows)
        bufs.append(buf)
        ys.append(y)
    xd = [cuda(x.reshape(-1)) for x in xs]
    b.bitnet_w2a8_linear_seq([(w, xd[i], ys[i], -1) for i, (_, _, w) in enumerate(ws)])
    assert b.bitnet_get_device_error() == b.BITNET_OK
    for i, ((rows, K), (t, sc, w)) in enumerate(zip(INDEP, ws)):
        _check_guard(bufs[i], rows)
        got = to_np(ys[i]).reshape(1, rows)
        rq, rs, _ = oracle.quant_act(xs[i])
        pick = _pick(rows, rows + i)
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        assert_decode_close(got[:, pick], ref, f"seq {rows}x{K}")
        y1 = tt.empty(rows, dtype=tt.float32, device="cuda")
        b.bitnet_w2a8_linear(w, xd[i], 1, y1)
        np.testing.assert_array_equal(got.reshape(-1), to_np(y1))


def test_seq_int32_sums_exact():
    """Unit scales and integer x with absmax 127 (s = 1): y is the int32 sum."""
    b = lib()
    shapes = [(3840, 2560), (2560, 2560), (13824, 2560), (2560, 6912), (777, 1280), (28672, 4096)]
    ws = _weights(shapes, 6100, unit=True)
    xs = [syn.integer_rows(6200 + i, 1, K) for i, (_, K) in enumerate(shapes)]
    ys = [torch().empty(rows, dtype=torch().float32, device="cuda") for rows, _ in shapes]
    b.bitnet_w2a8_linear_seq([(w, cuda(xs[i].reshape(-1)), ys[i], -1) for i, (_, _, w) in enumerate(ws)])
    for i, ((rows, K), (t, _, _)) in enumerate(zip(shapes, ws)):
        rq, rs, _ = oracle.quant_act(xs[i])
        assert rs[0] == 1.0
        pick = _pick(rows, 77 + i, 200)
        want = oracle.block_acc(oracle.pack_i2s(t[pick]), K, rq).astype(np.int64).sum(-1).astype(np.float32)
        got = to_np(ys[i]).reshape(1, rows)[:, pick]
        np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


def _chain(shapes, seed, calls=1, mode="seq"):
    """Each entry's x is the first K entries of the previous entry's y."""
    b = lib()
    tt = torch()
    ws = _weights(shapes, seed)
    ys = [tt.empty(rows, dtype=tt.float32, device="cuda") for rows, _ in shapes]
    x0 = cuda(syn.activations(seed + 999, 1, shapes[0][1], outliers=True).reshape(-1))
    xs = [x0] + [ys[i - 1][:K] for i, (_, K) in enumerate(shapes) if i > 0]
    for prev, (rows, K) in zip(shapes, shapes[1:]):
        assert prev[0] >= K
    work = _workspace(len(shapes))
    for _ in range(calls):
        if mode == "seq":
            b.bitnet_w2a8_linear_seq([(w, xs[i], ys[i], i - 1) for i, (_, _, w) in enumerate(ws)], work)
        else:
            for i, (_, _, w) in enumerate(ws):
                b.bitnet_w2a8_linear(w, xs[i], 1, ys[i])
    assert b.bitnet_get_device_error() == b.BITNET_OK
    assert np.all(to_np(work) == 0), "workspace not left zeroed"
    return ws, xs, ys


# A 2B-shaped layer chain: QKV -> O reads the first 2560 of QKV's y, gate+up
# reads O's y, down reads the first 6912 of gate+up's y, the next QKV reads
# down's y.
CHAIN = [(3840, 2560), (2560, 2560), (13824, 2560), (2560, 6912)] * 3 + [(3840, 2560)]


def test_seq_chain_matches_oracle_per_link_and_per_call():
    ws, xs, ys = _chain(CHAIN, 7100, calls=2)
    _, xs1, ys1 = _chain(CHAIN, 7100, mode="per_call")
    for i, ((rows, K), (t, sc, w)) in enumerate(zip(CHAIN, ws)):
        x = to_np(xs[i]).reshape(1, K)            # the input this link actually read
        rq, rs, _ = oracle.quant_act(x)
        pick = _pick(rows, 300 + i)
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        got = to_np(ys[i]).reshape(1, rows)
        assert_decode_close(got[:, pick], ref, f"chain link {i} {rows}x{K}")
        np.testing.assert_array_equal(got.reshape(-1), to_np(ys1[i]))


def test_seq_mixed_waves_and_ragged():
    """Entries 0, 1, 4 wait for nothing; 2 waits for 0, 3 for 2, 5 for 1."""
    b = lib()
    tt = torch()
    shapes = [(1000, 640), (513, 1280), (700, 1000 // 128 * 128), (33, 640), (5000, 384), (129, 512)]
    deps = [-1, -1, 0, 2, -1, 1]
    ws = _weights(shapes, 8100)
    ys = [tt.empty(rows, dtype=tt.float32, device="cuda") for rows, _ in shapes]
    xs = []
    for i, ((rows, K), d) in enumerate(zip(shapes, deps)):
        xs.append(cuda(syn.activations(8200 + i, 1, K).reshape(-1)) if d < 0 else ys[d][:K])
    work = _workspace(len(shapes))
    for _ in range(3):
        b.bitnet_w2a8_linear_seq([(w, xs[i], ys[i], deps[i]) for i, (_, _, w) in enumerate(ws)], work)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    for i, ((rows, K), (t, sc, w)) in enumerate(zip(shapes, ws)):
        x = to_np(xs[i]).reshape(1, K)
        rq, rs, _ = oracle.quant_act(x)
        assert_decode_close(to_np(ys[i]).reshape(1, rows), oracle.linear(oracle.pack_i2s(t), sc, K, rq, rs),
                            f"mixed entry {i}")


def test_seq_full_step_sampled_rows():
    """The benchmark's step: 30 layers x (QKV, O, gate+up, down), every linear
    with its own input, one call."""
    b = lib()
    tt = torch()
    shapes = [(3840, 2560), (2560, 2560), (13824, 2560), (2560, 6912)]
    layers = 30
    # Weights repeat every 5 layers to bound host-side packing time; every
    # linear still has its own input and output.
    uniq = _weights(shapes * 5, 9100)
    entries, xs, ys = [], [], []
    for l in range(layers):
        for m, (rows, K) in enumerate(shapes):
            x = syn.activations(syn.seed_for(1, l, m, syn.KIND_ACT), 1, K, outliers=True)
            y = tt.empty(rows, dtype=tt.float32, device="cuda")
            xs.append(x)
            ys.append(y)
            entries.append((uniq[(l % 5) * 4 + m][2], cuda(x.reshape(-1)), y, -1))
    b.bitnet_w2a8_linear_seq(entries)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    for i in range(0, layers * 4, 7):
        rows, K = shapes[i % 4]
        t, sc, _ = uniq[((i // 4) % 5) * 4 + i % 4]
        rq, rs, _ = oracle.quant_act(xs[i])
        pick = _pick(rows, 500 + i, 24) if rows > 4096 else np.arange(0, rows, 37)
        ref = oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs)
        assert_decode_close(to_np(ys[i]).reshape(1, rows)[:, pick], ref, f"step linear {i}")


def test_seq_wait_timeout_is_reported_and_recoverable():
    b = lib()
    shapes = [(28672, 4096), (4096, 14336), (28672, 4096)]
    ws, xs, ys = _chain(shapes, 9900)
    work = _workspace(len(shapes))
    entries = [(w, xs[i], ys[i], i - 1) for i, (_, _, w) in enumerate(ws)]
    b.bitnet_set_wait_limit(1)
    try:
        for _ in range(3):
            b.bitnet_w2a8_linear_seq(entries, work)
        st = b.bitnet_get_device_error()
    finally:
        b.bitnet_set_wait_limit(0)
    assert st == b.BITNET_ERR_TIMEOUT
    assert np.all(to_np(work) == 0), "workspace not left zeroed after a timeout"
    b.bitnet_w2a8_linear_seq(entries, work)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    for i, ((rows, K), (t, sc, w)) in enumerate(zip(shapes, ws)):
        x = to_np(xs[i]).reshape(1, K)
        rq, rs, _ = oracle.quant_act(x)
        pick = _pick(rows, 40 + i)
        assert_decode_close(to_np(ys[i]).reshape(1, rows)[:, pick],
                            oracle.linear(oracle.pack_i2s(t[pick]), sc[pick], K, rq, rs), f"after timeout {i}")
