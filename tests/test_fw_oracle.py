"""Pins of the fixed-width lane layout oracle (oracle/fworacle.c).

What pins it (each independent of the oracle's own code):
* the two layouts of sections 10.1 and 10.2, derived by hand (tests/golden/lane_*.hex);
* a hand-derived plane C block, which fixes the 24-bit lane packing and every step's bit;
* the code table against a numpy lexsort of the counts (the tie rule);
* the escape count and the size against a numpy count;
* a round trip on every 16-bit pattern, and on ragged lengths;
* each malformed field, which must be refused.
"""
import os
import struct

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lane_golden(name):
    out = bytearray()
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("zeros"):
                out += bytes(int(line.split()[1]))
            else:
                out += bytes(int(x, 16) for x in line.split())
    return bytes(out)


SEVENTEEN = np.array([(i << 7) | i for i in range(17)], np.uint16)
CASES = [("lane_one_weight.hex", np.array([0x3F80], np.uint16), 464),
         ("lane_seventeen.hex", SEVENTEEN, 496)]


@pytest.mark.parametrize("fname,words,size", CASES)
def test_golden_encode(fname, words, size):
    want = _lane_golden(fname)
    assert len(want) == size
    assert oracle.fw_encode(words) == want


@pytest.mark.parametrize("fname,words,size", CASES)
def test_golden_decode(fname, words, size):
    got = oracle.fw_decode(_lane_golden(fname))
    assert np.array_equal(got, words)


def test_plane_c_block_by_hand():
    # Lanes 0, 1 and 31 hold weights with fraction t << 4 at step t (h = t, u = 0); every
    # other weight is 1.0. Lane field by hand: even steps 0,2,4,6 carry h = 0,2,4,6 at bits
    # 0,3,6,9 -> 0x000D10; odd steps 1,3,5,7 carry h = 1,3,5,7 at bits 12,15,18,21 ->
    # 0xF59000. The field 0xF59D10 sits at bit 24j: bytes 3j..3j+2 = 10 9d f5.
    w = np.full(256, 0x3F80, np.uint16)
    for j in (0, 1, 31):
        for t in range(8):
            w[8 * j + t] = 0x3F80 | (t << 4)
    blob = oracle.fw_encode(w)
    c = blob[96 + 128 + 128: 96 + 128 + 128 + 96]
    want = bytearray(96)
    for j in (0, 1, 31):
        want[3 * j: 3 * j + 3] = bytes([0x10, 0x9D, 0xF5])
    assert c == bytes(want)
    assert np.array_equal(oracle.fw_decode(blob), w)


def _table_by_sort(words):
    s = words.astype(np.int64) >> 7
    cnt = np.bincount(s, minlength=512)
    present = np.nonzero(cnt)[0]
    order = present[np.lexsort((present, -cnt[present]))]  # by count down, then s up
    top = [int(v) for v in order[:16]]
    return top + [0] * (16 - len(top)), len(top)


def _gaussian_bf16(n, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    f = (rng.standard_normal(n) * scale).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_table_tie_rule_against_sort(seed):
    rng = np.random.default_rng(seed)
    # few symbols with many equal counts, so that the tie rule decides the order
    s = rng.choice(np.arange(0, 512, 7), size=23, replace=False)
    counts = rng.integers(1, 4, size=s.size)
    w = np.repeat(s, counts).astype(np.uint16) << 7
    w = w | rng.integers(0, 128, size=w.size).astype(np.uint16)
    rng.shuffle(w)
    assert oracle.fw_table(w) == _table_by_sort(w)


def test_table_short_alphabet():
    w = np.array([0x4000, 0x4001, 0x3F80, 0x4002], np.uint16)   # s = 128 three times, 127 once
    assert oracle.fw_table(w) == ([128, 127] + [0] * 14, 2)


@pytest.mark.parametrize("n", [0, 1, 255, 256, 257, 1000, 4099])
def test_size_and_escapes_against_count(n):
    w = _gaussian_bf16(n, seed=n)
    table, k = _table_by_sort(w)
    n_exc = int(np.count_nonzero(~np.isin(w >> 7, table[:k])))
    blob = oracle.fw_encode(w)
    info = oracle.fw_info(blob)
    assert info["n_exc"] == n_exc
    assert info["n_tiles"] == (n + 255) // 256
    assert len(blob) == info["total_bytes"] == oracle.fw_bytes(n, n_exc)
    assert np.array_equal(oracle.fw_decode(blob), w)


def test_every_pattern_round_trips():
    w = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    blob = oracle.fw_encode(w)
    info = oracle.fw_info(blob)
    # each s occurs 128 times: the table is s = 0..15 and every other weight escapes
    assert info["table"] == list(range(16))
    assert info["n_exc"] == (1 << 16) - 16 * 128
    assert np.array_equal(oracle.fw_decode(blob), w)
    rng = np.random.default_rng(7)
    p = rng.permutation(w)[: (1 << 16) - 77]
    assert np.array_equal(oracle.fw_decode(oracle.fw_encode(p)), p)


def test_tile_exc_counts_escapes_per_tile():
    rng = np.random.default_rng(3)
    w = _gaussian_bf16(256 * 5 + 9, seed=3, scale=1.0)   # wide exponent spread: many escapes
    blob = oracle.fw_encode(w)
    info = oracle.fw_info(blob)
    table = info["table"]
    esc = ~np.isin(w >> 7, table)
    nt = info["n_tiles"]
    off = 96 + 352 * nt
    te = np.frombuffer(blob, np.uint32, nt + 1, off)
    per_tile = [int(esc[256 * t: 256 * (t + 1)].sum()) for t in range(nt)]
    assert te.tolist() == list(np.concatenate([[0], np.cumsum(per_tile)]))
    assert np.array_equal(oracle.fw_decode(blob), w)
    del rng


def test_empty_tensor():
    blob = oracle.fw_encode(np.zeros(0, np.uint16))
    assert len(blob) == 96 + 16
    assert oracle.fw_info(blob)["n_tiles"] == 0
    assert oracle.fw_decode(blob).size == 0


def test_bits_per_weight_near_card_figure():
    # The card's runtime accounting: about 11.36 bits per weight resident. Gaussian-shaped
    # BF16 weights should land near it (11.125 fixed plus 24 bits per escape).
    w = _gaussian_bf16(1 << 20, seed=11)
    bits = 8 * len(oracle.fw_encode(w)) / w.size
    assert 11.2 < bits < 11.6, bits


def _corrupt(blob, off, fmt, value):
    b = bytearray(blob)
    struct.pack_into(fmt, b, off, value)
    return bytes(b)


def test_refuses_malformed_headers():
    w = _gaussian_bf16(700, seed=5, scale=1.0)
    blob = oracle.fw_encode(w)
    info = oracle.fw_info(blob)
    bad = [
        (_corrupt(blob, 0, "<B", ord("X")), oracle.E_FORMAT),             # magic
        (_corrupt(blob, 8, "<I", 2), oracle.E_VERSION),                   # version
        (_corrupt(blob, 12, "<I", 32), oracle.E_FORMAT),                  # header_bytes
        (_corrupt(blob, 24, "<Q", info["n_tiles"] + 1), oracle.E_FORMAT),  # n_tiles
        (_corrupt(blob, 32, "<Q", 701), oracle.E_FORMAT),                 # n_exc > n_elems
        (_corrupt(blob, 40, "<Q", len(blob) + 16), oracle.E_FORMAT),      # total_bytes
        (_corrupt(blob, 50, "<B", 1), oracle.E_FORMAT),                   # reserved
        (_corrupt(blob, 64 + 2 * 3, "<H", 512), oracle.E_FORMAT),         # table entry
        (blob[:-16], oracle.E_FORMAT),                                    # short buffer
    ]
    for b, code in bad:
        with pytest.raises(oracle.OracleError) as e:
            oracle.fw_decode(b)
        assert e.value.code == code


def test_refuses_bad_exception_lists():
    w = _gaussian_bf16(256 * 3 + 40, seed=9, scale=1.0)
    blob = oracle.fw_encode(w)
    info = oracle.fw_info(blob)
    nt, ne = info["n_tiles"], info["n_exc"]
    assert ne > 8
    te = 96 + 352 * nt
    pos = te + ((4 * (nt + 1) + 15) // 16) * 16
    t1 = struct.unpack_from("<I", blob, te + 4)[0]
    t2 = struct.unpack_from("<I", blob, te + 8)[0]
    assert 1 < t1 < t2
    last_tile_first = struct.unpack_from("<I", blob, te + 4 * (nt - 1))[0]
    assert last_tile_first < ne
    bad = [
        _corrupt(blob, te, "<I", 1),                     # tile_exc[0] != 0
        _corrupt(blob, te + 4, "<I", t2 + 1),            # decreasing
        _corrupt(blob, te + 4 * nt, "<I", ne - 1),       # does not end at n_exc
        _corrupt(blob, pos + 1, "<B", blob[pos]),        # positions of tile 0 not ascending
        _corrupt(blob, pos + ne - 1, "<B", 255),         # last tile: position past the tensor
    ]
    for b in bad:
        with pytest.raises(oracle.OracleError) as e:
            oracle.fw_decode(b)
        assert e.value.code == oracle.E_CORRUPT


# ---------------------------------------------------------------- y = W x on the layout
def _bf(v):
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_gemv_oracle_closed_form():
    # rows: all 1.0; all 2.0; 1.0 except one weight of 2^20; and 1.0 except 2^(k-8) at
    # column k < 20. Row 3 has 20 + 1 distinct exponents in all, so some of its weights
    # escape. x = 1, 2, ..., 256 (exact in BF16) for the first three rows, and all ones for
    # row 3 in a second product.
    cols = 256
    w = np.full((4, cols), 0x3F80, np.uint16)
    w[1, :] = 0x4000
    w[2, 99] = _bf(2.0 ** 20)
    w[3, :20] = _bf(2.0 ** (np.arange(20) - 8))
    blob = oracle.fw_encode(w)
    assert oracle.fw_info(blob)["n_exc"] >= 1
    x = _bf(np.arange(1, cols + 1))
    y = oracle.fw_gemv(blob, 4, cols, x)
    assert y[:3].tolist() == [32896.0, 65792.0, 32896.0 + (2.0 ** 20 - 1) * 100]
    ones = np.full(cols, 0x3F80, np.uint16)
    y1 = oracle.fw_gemv(blob, 4, cols, ones)
    assert y1[3] == (2.0 ** 20 - 1) * 2.0 ** -8 + (cols - 20)


def test_gemv_oracle_matches_definition_on_the_originals():
    rows, cols = 37, 512
    w = _gaussian_bf16(rows * cols, seed=4, scale=1.0).reshape(rows, cols)
    x = _gaussian_bf16(3 * cols, seed=5).reshape(3, cols)
    blob = oracle.fw_encode(w)
    assert oracle.fw_info(blob)["n_exc"] > 0
    f = lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(oracle.fw_gemv(blob, rows, cols, x), f(x) @ f(w).T)
