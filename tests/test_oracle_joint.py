"""Pins of the oracle's JOINT kind: one quantised table
over the pairs j = (s << 3) | h, decoded with one lookup per weight.

What pins it:
* two containers derived by hand (tests/golden/joint_two_weights.hex and, for the word order,
  tests/golden/joint_interleave_sixteen.hex);
* every 16-bit pattern and a size sweep round-trip;
* a closed form: pairs with power-of-two frequencies cost exactly log2(2^nj / F) bits each,
  so the word count is fixed up to the lanes' start and end states;
* Gibbs' inequality and the 0.5% overhead gate against the empirical entropy;
* every malformed JOINT field is refused.
"""
import itertools
import math
import os
import struct

import numpy as np
import pytest

import oracle
import synthetic as S
from tests.entropy import conditional_entropy_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    hexs = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            hexs.append(line.split("#", 1)[0])
    return bytes.fromhex("".join("".join(hexs).split()))


def _words(spec):
    return S.words_numpy(S.generate(spec, "cpu"))


def _roundtrip(items, **kw):
    c = oracle.encode(items, model="joint", **kw)
    arr = np.frombuffer(c, np.uint8)
    assert oracle.validate(arr) == len(items)
    for k, (_, a, _) in enumerate(items):
        assert np.array_equal(oracle.decode(arr, k), a), items[k][0]
    return arr


def test_golden_encode_and_decode():
    want = _golden("joint_two_weights.hex")
    w = np.array([0x3F80, 0x3F90], np.uint16)
    got = oracle.encode([("w", w, "bf16")], model="joint", force_rans=True)
    assert got == want
    assert np.array_equal(oracle.decode(want, 0), w)
    ti = oracle.info(want, 0)
    assert (ti["kind"], ti["ns"], ti["nh"], ti["n_routes"], ti["nib_mode"]) == (oracle.KIND_JOINT, 13, 0, 0, 0x10)


# Single-lane JOINT models for the brute force: (nj, {pair j: Fj}). The first has power-of-two
# frequencies, so lane states land exactly on the renormalisation bound Fj << (32 - nj) and an
# off-by-one comparison there breaks the round trip; the second codes two pairs of frequency 1
# at the largest precision; the third has frequencies with no common power of two.
TINY_JOINT = [
    (8, {1016: 128, 1017: 64, 3000: 64}),
    (13, {1016: 8190, 1017: 1, 2047: 1}),
    (10, {5: 700, 1016: 300, 4095: 24}),
]
L = 1 << 16


@pytest.mark.parametrize("mi", range(len(TINY_JOINT)))
def test_bruteforce_tiny_joint_alphabets(mi):
    """Every sequence of length <= 8 over three pairs: decode inverts encode, the lane ends at
    L, at most one word leaves per step, and the code length log2(start state) + 16 * words
    is 16 + sum log2(2^nj / F) within the rANS rounding bound log2(1 + 2^(nj - 16)) per step."""
    nj, freqs = TINY_JOINT[mi]
    Fj = np.zeros(4096, np.uint32)
    for j, f in freqs.items():
        Fj[j] = f
    assert Fj.sum() == 1 << nj
    pairs = sorted(freqs)
    n_seq = 0
    for S in range(0, 9):
        for seq in itertools.product(pairs, repeat=S):
            words = np.array([(j << 4) | ((5 * t + 3) & 15) for t, j in enumerate(seq)], np.uint16)
            x0, wd, tags = oracle.joint_lane_encode(Fj, nj, words)
            assert L <= x0 < (1 << 32)
            assert np.all(np.diff(tags.astype(np.int64)) > 0)
            st, out, fin = oracle.joint_lane_decode(Fj, nj, x0, wd, words & 15, S)
            assert st == 0 and fin == L
            assert np.array_equal(out, words)
            ideal = sum(nj - math.log2(freqs[j]) for j in seq)
            got = math.log2(x0) + 16 * wd.size
            assert abs(got - 16 - ideal) <= 1e-6 + S * math.log2(1 + 2.0 ** (nj - 16)), (seq, got, ideal)
            n_seq += 1
    assert n_seq == sum(3 ** k for k in range(9))


def test_joint_lane_hits_the_bound_exactly():
    # Under the first model pair 1016 has frequency 128 of 2^8 and cumulative 0, so encoding it
    # maps x to (x / 128) * 256 + x % 128, which doubles a state that is a multiple of 128.
    # From L = 2^16, fifteen weights reach 2^31 = 128 << (32 - 8), the bound itself, so the
    # sixteenth (step 0) must emit the low word 0 and continue from 2^15, ending at 2^16.
    nj, freqs = TINY_JOINT[0]
    Fj = np.zeros(4096, np.uint32)
    for j, f in freqs.items():
        Fj[j] = f
    words = np.full(16, 1016 << 4, np.uint16)
    x0, wd, tags = oracle.joint_lane_encode(Fj, nj, words)
    assert wd.tolist() == [0] and tags.tolist() == [0]
    assert x0 == 1 << 16
    # fifteen weights stay below the bound and emit nothing
    x15, wd15, _ = oracle.joint_lane_encode(Fj, nj, words[:15])
    assert x15 == 1 << 31 and wd15.size == 0
    st, out, fin = oracle.joint_lane_decode(Fj, nj, x0, wd, words & 15, 16)
    assert st == 0 and fin == L and np.array_equal(out, words)


def test_joint_lane_refuses_bad_tables():
    Fj = np.zeros(4096, np.uint32)
    Fj[7] = 255                       # sums to 255, not 2^8
    with pytest.raises(oracle.OracleError):
        oracle.joint_lane_encode(Fj, 8, np.array([7 << 4], np.uint16))
    Fj[7] = 256
    with pytest.raises(oracle.OracleError):   # a pair of frequency 0
        oracle.joint_lane_encode(Fj, 8, np.array([8 << 4], np.uint16))
    with pytest.raises(oracle.OracleError):   # precision outside 8..13
        oracle.joint_lane_encode(Fj, 7, np.array([7 << 4], np.uint16))


def test_every_pattern_round_trips():
    w = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(3)
    arr = _roundtrip([("all", w, "bf16"), ("shuffled", rng.permutation(w), "bf16")], force_rans=True)
    assert oracle.info(arr, 0)["kind"] == oracle.KIND_JOINT


def test_sizes_and_edges():
    rng = np.random.default_rng(11)
    sizes = list(range(1, 300)) + [1023, 1024, 1025, 65535, 65536, 65537, 2 * 65536 + 255]
    items = []
    for n in sizes:
        x = (rng.standard_normal(n) * 0.02).astype(np.float32)
        items.append((f"n{n}", (x.view(np.uint32) >> 16).astype(np.uint16), "bf16"))
    arr = _roundtrip(items, force_rans=True)
    for k, n in enumerate(sizes):
        assert oracle.info(arr, k)["n_chunks"] == -(-n // 65536)


@pytest.mark.parametrize("nj", [8, 10, 12, 13])
@pytest.mark.parametrize("log2_chunk", [8, 16])
def test_precisions_and_chunks(nj, log2_chunk):
    w = _words(S.workload("tensor_1m")[0]).reshape(-1)[:90_001]
    if nj < 10:   # keep the pair alphabet below 2^nj
        w = np.where(np.arange(w.size) % 3 == 0, 0x3C00, 0xBC31).astype(np.uint16)
    arr = _roundtrip([("w", w, "bf16")], nj=nj, log2_chunk=log2_chunk, force_rans=True)
    assert oracle.info(arr, 0)["ns"] == nj


@pytest.mark.parametrize("nj", [7, 14, 0])
def test_precision_out_of_range(nj):
    with pytest.raises(oracle.OracleError):
        oracle.encode([("w", np.ones(10, np.uint16), "bf16")], model="joint", nj=nj)


def test_power_of_two_frequencies_closed_form():
    # four pairs with counts in proportion 1/2, 1/4, 1/8, 1/8 quantise exactly (4096, 2048,
    # 1024, 1024 of 8192). Each weight then multiplies the state by exactly 2, 4, 8 or 8, i.e.
    # costs exactly 1, 2, 3 or 3 bits: 1.75 bits per weight. Over the chunk's 65536 slots the
    # 32 lanes take 2048 steps each and start from 2^16, so lane j's word count is
    # floor((16 + bits_j - 16) / 16) within one word: the total is 65536 * 1.75 / 16 = 7168
    # words, up to 32 (one partial word per lane).
    n = 65536
    pattern = np.array([0x3F80] * 4 + [0x3F90] * 2 + [0x3FA0, 0x3FB0], np.uint16)
    w = np.tile(pattern, n // 8)
    arr = _roundtrip([("w", w, "bf16")], force_rans=True)
    ti = oracle.info(arr, 0)
    n_words = int.from_bytes(arr[ti["data_offset"] + 8: ti["data_offset"] + 12].tobytes(), "little")
    assert 7168 - 32 <= n_words <= 7168


def test_gibbs_and_half_percent_gate():
    total_bits = total_h = 0.0
    for name in ("tensor_1m", "gemma2_layer"):
        for s in S.workload(name):
            w = _words(s)
            c = oracle.encode([(s.name, w, "bf16")], model="joint", force_rans=True)
            ti = oracle.info(c, 0)
            h = conditional_entropy_bits(w)                   # total bits of the tensor
            bits = 8.0 * ti["coded_bytes"]
            assert bits >= h, s.name                          # Gibbs' inequality
            total_bits += bits
            total_h += h
    assert total_bits / total_h - 1 < 0.005, total_bits / total_h - 1


def test_edge_mix_kinds():
    specs = S.workload("edge_mix")
    items = [(s.name, _words(s), "raw" if s.is_raw else "bf16") for s in specs]
    arr = _roundtrip(items)
    kinds = {s.name: oracle.info(arr, k)["kind"] for k, s in enumerate(specs)}
    assert kinds["uniform16"] == oracle.KIND_STORED
    assert kinds["raw_span"] == oracle.KIND_RAW
    assert kinds["t3"] == kinds["outliers"] == kinds["zeros"] == kinds["ones"] == oracle.KIND_JOINT


def _bad(c, off, fmt, v):
    b = bytearray(c)
    struct.pack_into(fmt, b, off, v)
    return np.frombuffer(bytes(b), np.uint8)


def test_refuses_malformed_joint_fields():
    c = _golden("joint_two_weights.hex")
    d, m = 64, 224
    bad = [
        _bad(c, d + 4, "<B", 7),             # nj below 8
        _bad(c, d + 4, "<B", 14),            # nj above 13
        _bad(c, d + 5, "<B", 3),             # nh must be 0
        _bad(c, d + 6, "<B", 1),             # n_routes must be 0
        _bad(c, d + 0, "<B", 4),             # unknown kind
        _bad(c, m + 0, "<H", 0),             # no pairs
        _bad(c, m + 2, "<H", 1),             # reserved
        _bad(c, m + 8, "<H", 1016),          # pairs not ascending
        _bad(c, m + 4, "<H", 4096),          # pair out of range
        _bad(c, m + 6, "<H", 0),             # zero frequency
        _bad(c, m + 6, "<H", 4095),          # does not sum to 2^nj
        _bad(c, d + 40, "<Q", 16),           # model_bytes != 4 + 4 * n_pairs
    ]
    for k, b in enumerate(bad):
        with pytest.raises(oracle.OracleError) as e:
            oracle.validate(b)
        assert e.value.code == oracle.E_FORMAT, k


def test_corrupt_state_is_detected():
    c = bytearray(_golden("joint_two_weights.hex"))
    c[256] ^= 0x10                           # lane 0's start state
    with pytest.raises(oracle.OracleError) as e:
        oracle.decode(np.frombuffer(bytes(c), np.uint8), 0)
    assert e.value.code == oracle.E_CORRUPT


def test_too_many_pairs_for_the_precision_is_stored():
    # 1100 distinct pairs do not fit the 1024 slots of nj = 10, so the tensor is STORED even
    # when the encoder is told never to fall back; nj = 11 has room and codes it JOINT
    w = ((np.arange(1100 * 3) % 1100).astype(np.uint16) << 4) | 5
    for nj, kind in ((10, oracle.KIND_STORED), (11, oracle.KIND_JOINT)):
        arr = _roundtrip([("w", w, "bf16")], nj=nj, force_rans=True)
        assert oracle.info(arr, 0)["kind"] == kind, nj


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover
    given = None

if given is not None:
    @settings(max_examples=60, deadline=None)
    @given(st.integers(1, 5000), st.integers(1, 4096), st.integers(0, 2 ** 32 - 1),
           st.sampled_from(["factored", "joint"]), st.sampled_from([8, 12, 16]))
    def test_random_tensors_round_trip(n, alphabet, seed, model, log2_chunk):
        # words drawn from a random alphabet of up to 4096 patterns, some of them skewed:
        # every container validates and decodes back, and the coded size obeys Gibbs
        rng = np.random.default_rng(seed)
        pool = rng.integers(0, 1 << 16, size=alphabet, dtype=np.uint32).astype(np.uint16)
        p = rng.dirichlet(np.full(alphabet, 0.3))
        w = pool[rng.choice(alphabet, size=n, p=p)]
        arr = np.frombuffer(oracle.encode([("w", w, "bf16")], model=model, log2_chunk=log2_chunk,
                                          force_rans=True), np.uint8)
        assert oracle.validate(arr) == 1
        assert np.array_equal(oracle.decode(arr, 0), w)
        ti = oracle.info(arr, 0)
        if ti["kind"] in (oracle.KIND_JOINT, oracle.KIND_RANS):
            assert 8.0 * ti["coded_bytes"] >= conditional_entropy_bits(w)
