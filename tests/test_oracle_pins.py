"""Pins of the oracle against facts that do not come from the oracle itself.

* Containers derived by hand: one weight with constant nibbles (tests/golden/one_weight.hex),
  two weights with stored nibbles (tests/golden/two_weights.hex), and sixteen weights whose
  lanes emit different words at the same steps, which fixes the (step, lane) order of the
  interleaved stream (tests/golden/interleave_sixteen.hex and, for kind JOINT,
  tests/golden/joint_interleave_sixteen.hex).
* The NVLC model card's field split and bitwise reconstruction: every 16-bit pattern
  round-trips (this covers +-0, subnormals, +-inf and NaN payloads).
* rANS exactness: brute force over tiny alphabets, where the decode must invert the
  encode and the end state must be L. The code length must equal the model's ideal
  cost sum(log2(2^P/Q)) plus the 16 bits of the start state L, within the rANS rounding
  bound of log2(1 + 2^(P-16)) bits per step.
* The quantiser: closed forms, plus optimality against exhaustive search on small cases.
* The route rule: the Pearson-statistic threshold at its exact boundary.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

L = 1 << 16


def _golden_bytes(path):
    hexs = []
    with open(path) as fh:
        for line in fh:
            hexs.append(line.split("#", 1)[0])
    return bytes.fromhex("".join("".join(hexs).split()))


# ---------------------------------------------------------------- golden container
GOLDEN = [("one_weight.hex", [0x3F80], 704, 0x10), ("two_weights.hex", [0x3F80, 0x3F81], 832, 0x00)]


@pytest.mark.parametrize("fname,words,size,nib_mode", GOLDEN)
def test_golden_encode(golden_dir, fname, words, size, nib_mode):
    want = _golden_bytes(os.path.join(golden_dir, fname))
    assert len(want) == size
    got = oracle.encode([("w", np.array(words, np.uint16), "bf16")], force_rans=True)
    assert got == want


@pytest.mark.parametrize("fname,words,size,nib_mode", GOLDEN)
def test_golden_decode(golden_dir, fname, words, size, nib_mode):
    c = _golden_bytes(os.path.join(golden_dir, fname))
    assert oracle.validate(c) == 1
    ti = oracle.info(c, 0)
    assert (ti["kind"], ti["ns"], ti["nh"], ti["n_chunks"], ti["name"], ti["nib_mode"]) == (0, 11, 5, 1, "w", nib_mode)
    assert oracle.decode(c, 0).tolist() == words


# ---------------------------------------------------------------- the interleaved stream
# Sixteen weights whose lanes 0 and 1 emit different words at the same steps (0 and 4), derived
# by hand in the comments of tests/golden/interleave_sixteen.hex (kind RANS, ns 1, nh 3) and
# tests/golden/joint_interleave_sixteen.hex (kind JOINT, nj 12).
SIXTEEN = np.array([0x3F80 + 16 * h for h in range(8)] + [0x4000 + 16 * h for h in range(8)], np.uint16)
INTERLEAVE = [("interleave_sixteen.hex", dict(ns=1, nh=3), 768, [0x00010000, 0x00010008],
               [0x4321, 0xCBA9], [0x0765, 0x0FED]),
              ("joint_interleave_sixteen.hex", dict(model="joint", nj=12), 576, [0x00010043, 0x000108CB],
               [0x2107, 0xA90F], [0x6500, 0xED00])]


def _chunk0(c):
    ti = oracle.info(c, 0)
    e = ti["data_offset"]
    off = int.from_bytes(c[e:e + 8], "little")
    nw = int.from_bytes(c[e + 8:e + 12], "little")
    return off, nw


@pytest.mark.parametrize("fname,kw,size,states,step0,step4", INTERLEAVE)
def test_interleave_golden_encode_and_decode(golden_dir, fname, kw, size, states, step0, step4):
    want = _golden_bytes(os.path.join(golden_dir, fname))
    assert len(want) == size
    assert oracle.encode([("w", SIXTEEN, "bf16")], force_rans=True, **kw) == want
    assert np.array_equal(oracle.decode(want, 0), SIXTEEN)
    off, nw = _chunk0(want)
    st = np.frombuffer(want[off:off + 128], "<u4")
    words = np.frombuffer(want[off + 128:off + 128 + 2 * nw], "<u2")
    assert nw == 64 and st[:2].tolist() == states and set(st[2:].tolist()) == {0x00010000}
    # (step, lane) order: step 0's 32 words, then step 4's
    assert words[:2].tolist() == step0 and words[32:34].tolist() == step4
    assert not words[2:32].any() and not words[34:].any()


@pytest.mark.parametrize("fname,kw,size,states,step0,step4", INTERLEAVE)
def test_interleave_order_is_what_decodes(golden_dir, fname, kw, size, states, step0, step4):
    # Any other order of the same words fails: lane order swapped within a step, or the two
    # steps' blocks swapped. Each variant either fails the end check or decodes other weights.
    c = _golden_bytes(os.path.join(golden_dir, fname))
    off, nw = _chunk0(c)
    w0 = off + 128
    words = bytearray(c[w0:w0 + 2 * nw])
    lanes = words[2:4] + words[0:2] + words[4:]
    steps = words[64:] + words[:64]
    for variant in (lanes, steps):
        bad = c[:w0] + bytes(variant) + c[w0 + 2 * nw:]
        try:
            out = oracle.decode(bad, 0)
        except oracle.OracleError as e:
            assert e.code == oracle.E_CORRUPT
        else:
            assert not np.array_equal(out, SIXTEEN)


def test_checksum_published_splitmix64_outputs():
    # splitmix64 seeded with 0 produces e220a8397b1dcdaf, 6e789e6aa1b965f4, 06c45d188009454f
    g = 0x9E3779B97F4A7C15
    assert oracle.mix64(0) == 0xE220A8397B1DCDAF
    assert oracle.mix64(g) == 0x6E789E6AA1B965F4
    assert oracle.mix64((2 * g) % (1 << 64)) == 0x06C45D188009454F


def test_checksum_is_position_sensitive_sum():
    w = np.array([5, 7, 9], np.uint16)
    parts = [oracle.mix64((i << 16) | int(v)) for i, v in enumerate(w)]
    assert oracle.checksum(w) == sum(parts) % (1 << 64)
    assert oracle.checksum(w[::-1].copy()) != oracle.checksum(w)
    assert oracle.checksum(np.zeros(0, np.uint16)) == 0
    b = np.array([1, 2], np.uint8)
    assert oracle.checksum(b) == (oracle.mix64(1) + oracle.mix64((1 << 8) | 2)) % (1 << 64)


def test_one_weight_defaults_to_stored():
    c = oracle.encode([("w", np.array([0x3F80], np.uint16), "bf16")])
    assert oracle.info(c, 0)["kind"] == oracle.KIND_STORED
    assert oracle.decode(c, 0).tolist() == [0x3F80]


# ---------------------------------------------------------------- every bit pattern
def test_all_patterns_one_tensor():
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    c = oracle.encode([("all", w, "bf16")], force_rans=True)
    assert oracle.info(c, 0)["kind"] == oracle.KIND_RANS
    assert np.array_equal(oracle.decode(c, 0), w)


def test_all_patterns_single_element_tensors():
    # 65,536 one-weight tensors: each has a one-symbol s-model (zero-width s code).
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    items = [(f"p{k}", w[k:k + 1], "bf16") for k in range(65536)]
    c = oracle.encode(items, force_rans=True)
    arr = np.frombuffer(c, np.uint8)
    assert oracle.validate(arr) == 65536
    for k in range(0, 65536):
        assert int(oracle.decode(arr, k)[0]) == k


def test_field_split_closed_form():
    # w == (s << 7) | f with s = w >> 7 (9 bits) and f = w & 0x7F (7 bits).
    w = np.arange(65536, dtype=np.uint32)
    s, f = w >> 7, w & 0x7F
    assert s.max() == 511 and f.max() == 127
    assert np.array_equal((s << 7) | f, w)
    # sign is bit 8 of s, exponent its low 8 bits: 1.0 = 0x3F80 -> sign 0, exponent 127
    assert (0x3F80 >> 7) == 127 and (0xBF80 >> 7) == 256 + 127


# ---------------------------------------------------------------- brute force, one lane
def _tables(fs_dict, ns, route=None, fh=None):
    Fs = np.zeros(512, np.uint32)
    for k, v in fs_dict.items():
        Fs[k] = v
    assert Fs.sum() == 1 << ns
    r = np.full(256, 0xFF, np.uint8)
    if route:
        for e, idx in route.items():
            r[e] = idx
    Fh = np.zeros((0, 8), np.uint32) if fh is None else np.asarray(fh, np.uint32)
    return Fs, r, Fh


def _ideal_bits(words, Fs, ns, route, Fh, nh):
    """sum over weights of log2(2^P / Q), Q = Fs[s] * qh: the model's cost of (s, h)."""
    bits = 0.0
    for w in words:
        s, h = int(w) >> 7, (int(w) >> 4) & 7
        r = int(route[s & 0xFF])
        qh = (1 << nh) // 8 if r == 0xFF else int(Fh[r][h])
        bits += ns + nh - math.log2(int(Fs[s]) * qh)
    return bits


TINY_MODELS = []
# three s symbols (exponents 1, 2 and the sign-flipped 1), ns = 4, nh = 5
_fh = np.zeros((1, 8), np.uint32)
_fh[0, 0], _fh[0, 1], _fh[0, 5], _fh[0, 6] = 20, 9, 2, 1   # sums to 32 = 2^5, a skewed route for e = 2
TINY_MODELS.append(dict(fs={1: 9, 2: 6, 257: 1}, ns=4, route={2: 0}, fh=_fh, nh=5,
                        alphabet=[(1 << 7) | (3 << 4) | 5, (2 << 7) | (1 << 4) | 9, (257 << 7) | 0]))
TINY_MODELS.append(dict(fs={1: 1, 2: 1, 3: 2}, ns=2, route=None, fh=None, nh=3,
                        alphabet=[(1 << 7) | 0, (2 << 7) | (7 << 4) | 15, (3 << 7) | (4 << 4) | 1]))
# P = 16, the largest precision: one symbol of frequency 1 at ns = 12 and a table with a
# frequency-1 entry, so Q = 1 costs 16 bits and every step of it emits a word
_fh2 = np.zeros((2, 8), np.uint32)
_fh2[0, :] = 2            # flat over the eight values, sums to 16
_fh2[1, 3], _fh2[1, 7] = 15, 1
TINY_MODELS.append(dict(fs={10: 4095, 300: 1}, ns=12, route={10: 0, 300 & 0xFF: 1}, fh=_fh2, nh=4,
                        alphabet=[(10 << 7) | (3 << 4) | 7, (300 << 7) | (3 << 4) | 9, (300 << 7) | (7 << 4)]))


@pytest.mark.parametrize("mi", range(len(TINY_MODELS)))
def test_bruteforce_tiny_alphabets(mi):
    m = TINY_MODELS[mi]
    Fs, route, Fh = _tables(m["fs"], m["ns"], m["route"], m["fh"])
    alphabet = m["alphabet"]
    P = m["ns"] + m["nh"]
    n_seq = 0
    for S in range(0, 9):
        for seq in itertools.product(alphabet, repeat=S):
            words = np.array(seq, np.uint16)
            x0, wd, tags = oracle.lane_encode(Fs, m["ns"], route, Fh, m["nh"], words)
            assert L <= x0 < (1 << 32)
            assert np.all(np.diff(tags.astype(np.int64)) > 0)   # at most one word per step
            st, out, fin = oracle.lane_decode(Fs, m["ns"], route, Fh, m["nh"], x0, wd, words & 15, S)
            assert st == 0 and fin == L
            assert np.array_equal(out, words)
            # code length: log2(x0) + 16*n_words = 16 + ideal bits, up to rANS rounding
            ideal = _ideal_bits(words, Fs, m["ns"], route, Fh, m["nh"])
            got = math.log2(x0) + 16 * wd.size
            assert abs(got - 16 - ideal) <= 1e-6 + S * math.log2(1 + 2.0 ** (P - 16)), (seq, got, ideal)
            n_seq += 1
    assert n_seq == sum(3 ** k for k in range(9))


def test_bruteforce_code_length_is_tight_at_low_precision():
    # With P = 6 the rounding bound is S*log2(1 + 2^-10): the length must match the model.
    m = TINY_MODELS[1]
    Fs, route, Fh = _tables(m["fs"], m["ns"], m["route"], m["fh"])
    words = np.array(m["alphabet"] * 20, np.uint16)
    x0, wd, _ = oracle.lane_encode(Fs, m["ns"], route, Fh, m["nh"], words)
    ideal = _ideal_bits(words, Fs, m["ns"], route, Fh, m["nh"])
    assert abs(math.log2(x0) + 16 * wd.size - 16 - ideal) < 0.1


def test_lane_decode_detects_wrong_state():
    m = TINY_MODELS[0]
    Fs, route, Fh = _tables(m["fs"], m["ns"], m["route"], m["fh"])
    words = np.array(m["alphabet"] * 3, np.uint16)
    x0, wd, _ = oracle.lane_encode(Fs, m["ns"], route, Fh, m["nh"], words)
    # Decoding is a bijection on (state, words): a different start state either fails the
    # end check or decodes to a different message; it can never reproduce the original.
    for delta in (1, 2, 3, 1 << 12, 1 << 20):
        st, out, fin = oracle.lane_decode(Fs, m["ns"], route, Fh, m["nh"], x0 ^ delta, wd, words & 15, words.size)
        assert st == oracle.E_CORRUPT or not np.array_equal(out, words)
        assert (st == oracle.E_CORRUPT) == (fin != L or st == oracle.E_CORRUPT)


# ---------------------------------------------------------------- quantiser
def test_quantise_exact_proportions():
    assert oracle.quantise([1, 1, 2], 2048).tolist() == [512, 512, 1024]
    assert oracle.quantise([0, 5, 0, 15], 16).tolist() == [0, 4, 0, 12]


def test_quantise_single_symbol_gets_all():
    assert oracle.quantise([0, 0, 7, 0], 4096).tolist() == [0, 0, 4096, 0]


def test_quantise_tie_goes_to_lowest():
    # floor((2*1*4 + 3) / 6) = 1 each; one slot left, all ratios 1/3 tie -> index 0
    assert oracle.quantise([1, 1, 1], 4).tolist() == [2, 1, 1]


def test_quantise_rare_symbols_keep_one_slot():
    c = [10 ** 9, 1, 1, 1]
    q = oracle.quantise(c, 16)
    assert q.tolist() == [13, 1, 1, 1]


def test_quantise_too_many_symbols():
    with pytest.raises(oracle.OracleError):
        oracle.quantise([1, 1, 1], 2)


def _cost(c, q, M):
    return sum(ci * (math.log2(M) - math.log2(qi)) for ci, qi in zip(c, q) if ci)


def _best_cost(c, M):
    K = len(c)
    best = float("inf")
    present = [k for k in range(K) if c[k]]
    for parts in itertools.product(range(1, M + 1), repeat=len(present)):
        if sum(parts) != M:
            continue
        q = [0] * K
        for k, v in zip(present, parts):
            q[k] = v
        best = min(best, _cost(c, q, M))
    return best


def test_quantise_near_optimal_small_cases():
    rng = np.random.default_rng(5)
    for _ in range(40):
        K = int(rng.integers(2, 5))
        c = [int(v) for v in rng.integers(0, 60, K)]
        if sum(1 for v in c if v) < 1:
            continue
        M = 16
        q = oracle.quantise(c, M).tolist()
        assert sum(q) == M and all((qi >= 1) == (ci > 0) for qi, ci in zip(q, c))
        # greedy first-order moves reach the exhaustive optimum within 0.5% of total cost
        assert _cost(c, q, M) <= _best_cost(c, M) * 1.005 + 1e-9


def test_quantise_invariants_random():
    rng = np.random.default_rng(1)
    for M in (128, 1024, 4096):
        for _ in range(20):
            c = rng.integers(0, 1000, 512) * (rng.random(512) < 0.2)
            if c.sum() == 0:
                continue
            q = oracle.quantise(c, M)
            assert int(q.sum()) == M
            assert np.array_equal(q > 0, c > 0)


# ---------------------------------------------------------------- route rule
def _ceh_with(counts, e=40):
    ceh = np.zeros((256, 8), np.uint64)
    ceh[e, : len(counts)] = counts
    return ceh


def test_route_threshold_boundary():
    # chi2*n = 8*S - n^2 over the eight top-bit counts; candidate iff 8*S - n^2 > 256*n.
    r, re = oracle.choose_routes(_ceh_with([16] * 8))      # flat: chi2 = 0
    assert r[40] == 0xFF and re.size == 0
    # all mass on one value: 8*n^2 - n^2 = 7*n^2 > 256*n iff n > 36.57
    r, re = oracle.choose_routes(_ceh_with([37]))
    assert r[40] == 0 and re.tolist() == [40]
    r, re = oracle.choose_routes(_ceh_with([36]))          # 7*36 = 252 < 256
    assert r[40] == 0xFF
    # exactly on the boundary is not a candidate: n = 64, S = 48^2 + 16^2 = 2560,
    # 8*2560 - 64^2 = 16384 = 256*64
    r, _ = oracle.choose_routes(_ceh_with([48, 16]))
    assert r[40] == 0xFF
    r, _ = oracle.choose_routes(_ceh_with([49, 15]))       # 8*2626 - 4096 = 16912 > 16384
    assert r[40] == 0


def test_route_ranking_and_limit():
    ceh = np.zeros((256, 8), np.uint64)
    for e, k in ((10, 1000), (20, 3000), (30, 2000)):
        ceh[e, 0] = k            # one-hot rows: chi2 = 7 * n
    r, re = oracle.choose_routes(ceh, max_routes=2)
    assert re.tolist() == [20, 30]                       # the two largest chi2, in ascending e
    assert r[20] == 0 and r[30] == 1 and r[10] == 0xFF
    r, re = oracle.choose_routes(ceh, max_routes=0)
    assert re.size == 0
    with pytest.raises(oracle.OracleError):
        oracle.choose_routes(ceh, max_routes=16)


# ---------------------------------------------------------------- nibble modes
def test_nibble_modes():
    # constant low nibble -> no nibble words; any other -> stored, and both round-trip
    for words, mode in (([0x3F85] * 300, 0x15), ([0x3F80, 0x3F8F] * 150, 0x00)):
        w = np.array(words, np.uint16)
        c = oracle.encode([("w", w, "bf16")], force_rans=True)
        ti = oracle.info(c, 0)
        assert ti["nib_mode"] == mode
        assert np.array_equal(oracle.decode(c, 0), w)
        nib_bytes = 0 if mode else 128 * 2     # n_c = 300 weights -> B = 2 blocks
        assert ti["coded_bytes"] >= ti["model_bytes"] + 16 + 128 + nib_bytes
