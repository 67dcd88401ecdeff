"""GPU parity of the fused GEMV on the fixed-width lane layout (bs_fw_gemv) through the C ABI.

The kernel accumulates in fp32 in its own fixed order; the oracle computes y = W x in
float64 from its own decode. Every product of two BF16 values is exact in fp32, so the only
error is the fp32 rounding of the running sums, at most about K * 2^-24 times the sum of
|w_k x_k| over a row of K terms. An escaped weight enters as its placeholder plus a
correction, which adds the placeholder's |w x| to that sum. The test allows twice that bound.
Integer-valued cases whose partial sums stay below 2^24 must match exactly.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _gauss(n, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    return ((rng.standard_normal(n) * scale).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f64(words):
    return (np.asarray(words, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _dev(words):
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int16).copy()).cuda()


def _tolerance(w, x, table0):
    """Per output: 2 * K * 2^-24 * (sum |w x| + sum over escapes of |w_placeholder x|)."""
    rows, cols = w.shape
    wf, xf = _f64(w), _f64(x).reshape(-1, cols)
    s = np.abs(xf) @ np.abs(wf).T
    coded = np.isin(w >> 7, np.array(oracle.fw_info(oracle.fw_encode(w))["table"]))
    ph = _f64((table0 << 7) | (w & 0x7F)) * (~coded)
    s += np.abs(xf) @ np.abs(ph).T
    return 2.0 * cols * 2.0 ** -24 * s + 1e-30


def _run(products, batch):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = []
    items = []
    for w, x in products:
        rows, cols = w.shape
        fw, info = bs.fw_transcode(_dev(w.reshape(-1)))
        y = torch.empty((batch, rows), dtype=torch.float32, device="cuda")
        items.append((fw, info, rows, cols, _dev(x.reshape(batch, cols)), y))
        ys.append(y)
    bs.fw_gemv(items, err)
    torch.cuda.synchronize()
    return [y.cpu().numpy().astype(np.float64) for y in ys], int(err.item()), items


SHAPES = [(8, 256), (33, 512), (300, 3584), (2048, 3584), (96, 14336)]


@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("batch", [1, 3, 8])
def test_gemv_matches_oracle(rows, cols, batch):
    w = _gauss(rows * cols, seed=rows + cols).reshape(rows, cols)
    x = _gauss(batch * cols, seed=batch, scale=1.0).reshape(batch, cols)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0
    blob = oracle.fw_encode(w)
    ref = oracle.fw_gemv(blob, rows, cols, x)
    tol = _tolerance(w, x, oracle.fw_info(blob)["table"][0])
    assert items[0][1].n_exc > 0
    assert np.all(np.abs(y - ref) <= tol), float(np.max(np.abs(y - ref) / tol))


@pytest.mark.parametrize("rows,cols", [(3584, 4096), (3584, 14336)])
def test_gemv_rows_split_between_warps_are_exact_sums(rows, cols):
    # o- and down-projection shapes: a CTA holds 12-13 rows and its 8 warps share their tiles,
    # so most warps end inside a row and hand their piece to the warp that starts it; the
    # outputs are fixed sums, the same bits on every call
    batch = 2
    w = _gauss(rows * cols, seed=rows ^ cols).reshape(rows, cols)
    x = _gauss(batch * cols, seed=77, scale=1.0).reshape(batch, cols)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0
    blob = oracle.fw_encode(w)
    ref = oracle.fw_gemv(blob, rows, cols, x)
    assert np.all(np.abs(y - ref) <= _tolerance(w, x, oracle.fw_info(blob)["table"][0]))
    fw, info, _, _, xd, _ = items[0]
    for _ in range(3):
        y2 = torch.empty((batch, rows), dtype=torch.float32, device="cuda")
        e2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        bs.fw_gemv([(fw, info, rows, cols, xd, y2)], e2)
        torch.cuda.synchronize()
        assert int(e2.item()) == 0
        assert np.array_equal(y2.cpu().numpy().view(np.uint32), y.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("batch", [2, 4, 5, 6, 7])
def test_gemv_every_batch_instance(batch):
    # one kernel instance per batch size; rows of 20 tiles (cols 5120) take groups of 10
    rows, cols = 200, 5120
    w = _gauss(rows * cols, seed=55).reshape(rows, cols)
    x = _gauss(batch * cols, seed=56 + batch, scale=1.0).reshape(batch, cols)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0 and items[0][1].n_exc > 0
    blob = oracle.fw_encode(w)
    ref = oracle.fw_gemv(blob, rows, cols, x)
    assert np.all(np.abs(y - ref) <= _tolerance(w, x, oracle.fw_info(blob)["table"][0]))


def test_gemv_many_escapes_per_group():
    rows, cols = 40, 1024
    w = _gauss(rows * cols, seed=3, scale=1.0).reshape(rows, cols)
    w ^= ((np.arange(w.size) % 3 == 0).astype(np.uint16) << 14).reshape(rows, cols)  # exponents everywhere
    x = _gauss(2 * cols, seed=4, scale=1.0).reshape(2, cols)
    (y,), err, items = _run([(w, x)], 2)
    assert err == 0
    assert items[0][1].n_exc > 64 * rows          # far more than 64 escapes per group (a row here)
    ref = oracle.fw_gemv(oracle.fw_encode(w), rows, cols, x)
    finite = np.isfinite(ref)
    assert np.array_equal(np.isfinite(y), finite)
    tol = _tolerance(w, x, oracle.fw_info(oracle.fw_encode(w))["table"][0])
    assert np.all(np.abs(y[finite] - ref[finite]) <= tol[finite])


def test_gemv_integer_case_is_exact():
    # small integers: every partial sum stays below 2^24, so fp32 sums are exact
    rows, cols = 64, 768
    rng = np.random.default_rng(9)
    wv = rng.integers(-8, 9, size=(rows, cols)).astype(np.float32)
    wv[rng.random((rows, cols)) < 0.02] *= 1024.0                       # rarer exponents: escapes
    w = (wv.view(np.uint32) >> 16).astype(np.uint16)
    x = (rng.integers(-4, 5, size=(4, cols)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    (y,), err, items = _run([(w, x)], 4)
    assert err == 0 and items[0][1].n_exc > 0
    assert np.array_equal(y, oracle.fw_gemv(oracle.fw_encode(w), rows, cols, x))


def test_gemv_several_products_in_one_call():
    # q, k, v-like projections sharing one x
    cols, batch = 3584, 1
    x = _gauss(cols, seed=21, scale=1.0).reshape(1, cols)
    ws = [_gauss(r * cols, seed=r).reshape(r, cols) for r in (4096, 2048, 2048)]
    ys, err, _ = _run([(w, x) for w in ws], batch)
    assert err == 0
    for w, y in zip(ws, ys):
        blob = oracle.fw_encode(w)
        ref = oracle.fw_gemv(blob, w.shape[0], cols, x)
        assert np.all(np.abs(y - ref) <= _tolerance(w, x, oracle.fw_info(blob)["table"][0]))


def test_gemv_large_matrix_sampled_rows():
    # 65536 x 3584 (235 M weights): rows sampled against float64 products of the originals
    rows, cols = 65536, 3584
    g = torch.Generator(device="cuda").manual_seed(5)
    wt = (torch.randn(rows * cols, device="cuda", generator=g) * 0.02).to(torch.bfloat16).view(torch.int16)
    xt = torch.randn(cols, device="cuda", generator=g).to(torch.bfloat16).view(torch.int16)
    fw, info = bs.fw_transcode(wt)
    y = torch.empty((1, rows), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bs.fw_gemv([(fw, info, rows, cols, xt.view(1, cols), y)], err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sample = np.random.default_rng(0).choice(rows, 64, replace=False)
    w = wt.view(rows, cols)[torch.from_numpy(sample).cuda()].cpu().numpy().view(np.uint16)
    x = xt.cpu().numpy().view(np.uint16)
    ref = _f64(w) @ _f64(x)
    got = y[0].cpu().numpy()[sample].astype(np.float64)
    tol = 2.0 * cols * 2.0 ** -24 * (np.abs(_f64(w)) @ np.abs(_f64(x)) + 64.0 * np.abs(_f64(x)).max())
    assert np.all(np.abs(got - ref) <= tol)


def test_gemv_corrupt_tile_exc_is_flagged():
    rows, cols = 16, 1024
    w = _gauss(rows * cols, seed=8, scale=1.0).reshape(rows, cols)
    blob = bytearray(oracle.fw_encode(w))
    info = bs.fw_parse(np.frombuffer(bytes(blob), np.uint8)[:96], len(blob))
    te = 96 + 352 * info.n_tiles
    blob[te + 4: te + 8] = (info.n_exc + 3).to_bytes(4, "little")
    d = torch.from_numpy(np.frombuffer(bytes(blob), np.uint8).copy()).cuda()
    x = _dev(_gauss(cols, seed=1, scale=1.0).reshape(1, cols))
    y = torch.full((1, rows), -7.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bs.fw_gemv([(d, info, rows, cols, x, y)], err)
    torch.cuda.synchronize()
    assert int(err.item()) & 1
    assert torch.isfinite(y).all()


def test_gemv_special_weights_follow_ieee():
    # inf, -inf and NaN weights (rare exponents, so they escape): each output must match the
    # float64 product's class (nan, +inf, -inf) and, where finite, its value
    rows, cols = 24, 512
    w = _gauss(rows * cols, seed=13).reshape(rows, cols)
    w[3, 7] = 0x7F80             # +inf
    w[5, 100] = 0xFF80           # -inf
    w[9, 300] = 0x7FC1           # NaN
    w[11, 0] = 0x7F80
    w[11, 1] = 0xFF80            # inf + -inf in one row: NaN
    x = _gauss(cols, seed=14, scale=1.0).reshape(1, cols)
    x[0, 300] = 0x3F80
    (y,), err, _ = _run([(w, x)], 1)
    assert err == 0
    ref = oracle.fw_gemv(oracle.fw_encode(w), rows, cols, x)
    assert np.array_equal(np.isnan(y), np.isnan(ref))
    assert np.array_equal(np.isposinf(y), np.isposinf(ref)) and np.array_equal(np.isneginf(y), np.isneginf(ref))
    fin = np.isfinite(ref)
    tol = _tolerance(w, x, oracle.fw_info(oracle.fw_encode(w))["table"][0])
    assert np.all(np.abs(y[fin] - ref[fin]) <= tol[fin])


@pytest.mark.parametrize("resident", [False, True])
def test_gemv_back_to_back_calls_keep_stream_order(resident):
    # A call may be scheduled while the one before it on the stream finishes. Here the second
    # call's y is the first call's x (the same bytes), so the second must not write before the
    # first has read; a third call then writes its y over the same bytes, so the last writer
    # must win. Results are compared bit for bit with the calls made one at a time.
    cols, rows1, rows2 = 3584, 4096, 1792  # y2 (1792 fp32) takes exactly x1's 3584 BF16 words
    w1 = _gauss(rows1 * cols, seed=101).reshape(rows1, cols)
    w2 = _gauss(rows2 * cols, seed=102).reshape(rows2, cols)
    w3 = _gauss(rows2 * cols, seed=103).reshape(rows2, cols)
    x1 = _dev(_gauss(cols, seed=104, scale=1.0))
    x2 = _dev(_gauss(cols, seed=105, scale=1.0))
    fws = [bs.fw_transcode(_dev(w.reshape(-1))) for w in (w1, w2, w3)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call(k, rows, x, y):
        fw, info = fws[k]
        bs.fw_gemv([(fw, info, rows, cols, x.view(1, cols), y.view(1, rows))], err, layouts_resident=resident)

    alone = []
    for k, rows, x in ((0, rows1, x1), (1, rows2, x2), (2, rows2, x2)):
        y = torch.empty(rows, dtype=torch.float32, device="cuda")
        call(k, rows, x, y)
        torch.cuda.synchronize()
        alone.append(y.clone())
    shared = torch.empty(cols, dtype=torch.int16, device="cuda")   # x1, then y2 and y3
    y1 = torch.empty(rows1, dtype=torch.float32, device="cuda")
    for _ in range(20):
        shared.copy_(x1)
        call(0, rows1, shared, y1)
        call(1, rows2, x2, shared.view(torch.float32))
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int32), alone[0].view(torch.int32))
        assert torch.equal(shared.view(torch.float32).view(torch.int32), alone[1].view(torch.int32))
        call(1, rows2, x2, shared.view(torch.float32))
        call(2, rows2, x2, shared.view(torch.float32))
        torch.cuda.synchronize()
        assert torch.equal(shared.view(torch.float32).view(torch.int32), alone[2].view(torch.int32))
    assert int(err.item()) == 0
