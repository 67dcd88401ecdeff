"""GPU parity of the tensor-core product on the fixed-width lane layout (bs_fw_gemm) through
the C ABI.

The kernel decodes W (tile by tile, exceptions patched in) into shared memory and multiplies it
with the tokens on the tensor cores (BF16 operands, FP32 accumulation); the oracle computes
Y = X W^T in float64 from its own decode. Every product of two BF16 values is exact in FP32,
so the only error is the FP32 accumulation, whose order the tensor cores fix; the test allows
4 * K * 2^-24 times the sum of |w x| over a row, twice the bound of a sequential FP32 sum.
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
    x = torch.from_numpy((rng.standard_normal(n) * scale).astype(np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _f64(words):
    return (np.asarray(words, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _dev(words):
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int16).copy()).cuda()


def _run(products, batch):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys, items = [], []
    for w, x in products:
        rows, cols = w.shape
        fw, info = bs.fw_transcode(_dev(w.reshape(-1)))
        y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device="cuda")
        items.append((fw, info, rows, cols, _dev(x.reshape(batch, cols)), y))
        ys.append(y)
    bs.fw_gemm(items, err)
    torch.cuda.synchronize()
    return [y.cpu().numpy().astype(np.float64) for y in ys], int(err.item()), items


def _check(w, x, y):
    rows, cols = w.shape
    ref = oracle.fw_gemv(oracle.fw_encode(w), rows, cols, x)
    tol = 4.0 * cols * 2.0 ** -24 * (np.abs(_f64(x).reshape(-1, cols)) @ np.abs(_f64(w)).T) + 1e-30
    assert np.all(np.abs(y - ref) <= tol), float(np.max(np.abs(y - ref) / tol))


@pytest.mark.parametrize("rows,cols", [(128, 256), (256, 512), (384, 3584)])
@pytest.mark.parametrize("batch", [9, 16, 33, 64, 100])
def test_gemm_matches_oracle(rows, cols, batch):
    w = _gauss(rows * cols, seed=rows + cols).reshape(rows, cols)
    x = _gauss(batch * cols, seed=batch, scale=1.0).reshape(batch, cols)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0 and items[0][1].n_exc > 0
    _check(w, x, y)


def test_gemm_integer_case_is_exact():
    # small integers: every partial sum stays below 2^24, so the FP32 sums are exact in any order
    rows, cols, batch = 256, 1024, 24
    rng = np.random.default_rng(9)
    wv = rng.integers(-8, 9, size=(rows, cols)).astype(np.float32)
    wv[rng.random((rows, cols)) < 0.02] *= 1024.0                       # rarer exponents: escapes
    w = (wv.view(np.uint32) >> 16).astype(np.uint16)
    x = (rng.integers(-4, 5, size=(batch, cols)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0 and items[0][1].n_exc > 0
    assert np.array_equal(y, oracle.fw_gemv(oracle.fw_encode(w), rows, cols, x))


def test_gemm_many_escapes_and_several_products():
    # a matrix whose weights escape far more often than usual, next to q, k, v-like products
    cols, batch = 1024, 20
    x = _gauss(batch * cols, seed=4, scale=1.0).reshape(batch, cols)
    esc = _gauss(128 * cols, seed=3, scale=1.0).reshape(128, cols)
    esc ^= ((np.arange(esc.size) % 3 == 0).astype(np.uint16) << 13).reshape(128, cols)   # exponents everywhere
    ws = [esc] + [_gauss(r * cols, seed=r).reshape(r, cols) for r in (512, 256, 256)]
    ys, err, items = _run([(w, x) for w in ws], batch)
    assert err == 0 and items[0][1].n_exc > 32 * 128
    for w, y in zip(ws, ys):
        _check(w, x, y)


def test_gemm_agrees_with_the_gemv_and_dense_products():
    # the same product through bs_fw_gemm, through bs_fw_gemv (batch 8) and as a dense matmul
    rows, cols, batch = 512, 3584, 8
    w = _gauss(rows * cols, seed=31).reshape(rows, cols)
    x = _gauss(batch * cols, seed=32, scale=1.0).reshape(batch, cols)
    (y,), err, items = _run([(w, x)], batch)
    assert err == 0
    y2 = torch.empty((batch, rows), dtype=torch.float32, device="cuda")
    fw, info = items[0][0], items[0][1]
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    bs.fw_gemv([(fw, info, rows, cols, items[0][4], y2)], err2)
    dense = (_dev(x).view(torch.bfloat16).float() @ _dev(w).view(torch.bfloat16).float().T)
    torch.cuda.synchronize()
    assert int(err2.item()) == 0
    tol = torch.from_numpy(4.0 * cols * 2.0 ** -24 * (np.abs(_f64(x)) @ np.abs(_f64(w)).T)).cuda()
    assert torch.all((torch.from_numpy(y).cuda() - y2.double()).abs() <= tol)
    assert torch.all((torch.from_numpy(y).cuda() - dense.double()).abs() <= tol)


def test_gemm_refuses_rows_off_the_block():
    w = _gauss(100 * 256, seed=1).reshape(100, 256)
    x = _gauss(16 * 256, seed=2, scale=1.0).reshape(16, 256)
    fw, info = bs.fw_transcode(_dev(w.reshape(-1)))
    y = torch.empty((16, 100), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(bs.BsError) as e:
        bs.fw_gemm([(fw, info, 100, 256, _dev(x), y)], err)
    assert e.value.code == bs.E_ARG


def test_gemm_corrupt_tile_exc_is_flagged():
    rows, cols, batch = 128, 1024, 16
    w = _gauss(rows * cols, seed=8, scale=1.0).reshape(rows, cols)
    blob = bytearray(oracle.fw_encode(w))
    info = bs.fw_parse(np.frombuffer(bytes(blob), np.uint8)[:96], len(blob))
    te = 96 + 352 * info.n_tiles
    blob[te + 4: te + 8] = (info.n_exc + 3).to_bytes(4, "little")
    d = torch.from_numpy(np.frombuffer(bytes(blob), np.uint8).copy()).cuda()
    x = _dev(_gauss(batch * cols, seed=1, scale=1.0).reshape(batch, cols))
    y = torch.full((batch, rows), -7.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bs.fw_gemm([(d, info, rows, cols, x, y)], err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1
    assert torch.isfinite(y).all()


def test_gemm_without_and_with_k_split():
    # 297 row blocks fill the GPU (one CTA each, the sums written directly); 3 row blocks with
    # a long K are split over many CTAs that add their parts with atomics
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    batch = 16
    for rows, cols in ((128 * (2 * sms + 1), 256), (384, 256 * 56)):
        w = _gauss(rows * cols, seed=rows).reshape(rows, cols)
        x = _gauss(batch * cols, seed=cols, scale=1.0).reshape(batch, cols)
        (y,), err, _ = _run([(w, x)], batch)
        assert err == 0
        _check(w, x, y)


def test_gemm_items_of_different_shapes_and_tables_in_one_call():
    # one launch shares the (row block, tile) units of all items evenly among its CTAs, so a CTA
    # can cover the end of one item and the start of the next, with a different code table and
    # row length; rows of a single tile (cols 256) make many short runs per CTA
    batch = 24
    shapes = [(384, 256), (1280, 3584), (256, 1024), (640, 256), (128, 7168)]
    scales = [0.02, 1.0, 0.003, 0.5, 0.05]
    ws = [_gauss(r * c, seed=100 + k, scale=sc).reshape(r, c) for k, ((r, c), sc) in enumerate(zip(shapes, scales))]
    xs = [_gauss(batch * c, seed=200 + k, scale=1.0).reshape(batch, c) for k, (_, c) in enumerate(shapes)]
    tables = {tuple(oracle.fw_info(oracle.fw_encode(w))["table"]) for w in ws}
    assert len(tables) >= 3
    ys, err, _ = _run(list(zip(ws, xs)), batch)
    assert err == 0
    for w, x, y in zip(ws, xs, ys):
        _check(w, x, y)
