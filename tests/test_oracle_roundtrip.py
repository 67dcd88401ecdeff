"""Oracle round trips on the workloads' distributions, the size gates, and host-made faults.

The size gates compare against the empirical entropy H(s) + H(f|s) of the data itself
(tests/entropy.py):
* Gibbs' inequality: the coded size is never below it;
* overhead: the coded size is within 0.5% of it on the aggregate of the dense workloads.
"""
import numpy as np
import pytest

import oracle
import synthetic as S
from tests.entropy import conditional_entropy_bits


def _words(spec):
    return S.words_numpy(S.generate(spec, "cpu"))


def _roundtrip(items, **kw):
    c = oracle.encode(items, **kw)
    arr = np.frombuffer(c, np.uint8)
    assert oracle.validate(arr) == len(items)
    for k, (_, a, _) in enumerate(items):
        got = oracle.decode(arr, k)
        assert got.dtype == a.dtype and got.shape == a.shape
        assert np.array_equal(got, a), items[k][0]
    return arr


def test_sizes_every_n_up_to_1025_and_edges():
    rng = np.random.default_rng(7)
    sizes = list(range(0, 1026)) + [4095, 4096, 4097, 65535, 65536, 65537, 3 * 65536 + 255]
    items = []
    for n in sizes:
        x = (rng.standard_normal(n) * 0.02).astype(np.float32)
        w = (x.view(np.uint32) >> 16).astype(np.uint16)          # truncation is fine for a size sweep
        items.append((f"n{n}", w, "bf16"))
    arr = _roundtrip(items, force_rans=True)
    for k, n in enumerate(sizes):
        ti = oracle.info(arr, k)
        if n == 0:
            assert ti["kind"] == oracle.KIND_STORED and ti["data_bytes"] == 0
        else:
            assert ti["kind"] == oracle.KIND_RANS and ti["n_chunks"] == -(-n // 65536)


@pytest.mark.parametrize("log2_chunk", [8, 12, 16, 17])
def test_chunk_sizes(log2_chunk):
    w = _words(S.workload("tensor_1m")[0])[:300_001]
    _roundtrip([("w", w, "bf16")], log2_chunk=log2_chunk)


@pytest.mark.parametrize("ns,nh", [(1, 3), (8, 3), (8, 5), (11, 5), (12, 4), (12, 3), (11, 3)])
def test_precisions(ns, nh):
    w = _words(S.workload("tensor_1m")[0]).reshape(-1)[:70_000]
    if ns < 9:   # fewer than 512 slots: keep the alphabet small enough to fit
        w = np.where(np.arange(w.size) % 2 == 0, 0x3C00, 0xBC31).astype(np.uint16)
    _roundtrip([("w", w, "bf16")], ns=ns, nh=nh, force_rans=True)


@pytest.mark.parametrize("ns,nh", [(13, 3), (12, 5), (11, 6), (11, 2), (0, 5)])
def test_precisions_out_of_range(ns, nh):
    with pytest.raises(oracle.OracleError):
        oracle.encode([("w", np.ones(10, np.uint16), "bf16")], ns=ns, nh=nh)


def test_edge_mix_roundtrip_and_kinds():
    specs = S.workload("edge_mix")
    items = [(s.name, _words(s), "raw" if s.is_raw else "bf16") for s in specs]
    arr = _roundtrip(items)
    kinds = {s.name: oracle.info(arr, k)["kind"] for k, s in enumerate(specs)}
    assert kinds["uniform16"] == oracle.KIND_STORED       # incompressible -> stored
    assert kinds["raw_span"] == oracle.KIND_RAW
    assert kinds["t3"] == kinds["outliers"] == kinds["zeros"] == kinds["ones"] == oracle.KIND_RANS
    # degenerate tensors: only the lane flush remains (32 states + at most a word per step);
    # their nibbles are constant, so no nibble words are stored
    for nm in ("zeros", "ones"):
        ti = oracle.info(arr, [s.name for s in specs].index(nm))
        assert ti["nib_mode"] == 0x10
        assert ti["coded_bytes"] < 0.02 * 2 * ti["n_elems"]


def test_uniform16_forced_rans_roundtrip():
    s = S.workload("edge_mix")[4]
    w = _words(s)
    arr = _roundtrip([(s.name, w, "bf16")], force_rans=True)
    ti = oracle.info(arr, 0)
    bits = ti["coded_bytes"] * 8 / w.size
    assert 16.0 <= bits <= 16.1                             # incompressible: ~16 bits + flush


def test_gibbs_lower_bound_every_tensor():
    specs = [s for s in S.workload("edge_mix") if not s.is_raw] + S.workload("tensor_1m")
    for s in specs:
        w = _words(s)
        c = oracle.encode([(s.name, w, "bf16")], force_rans=True)
        ti = oracle.info(c, 0)
        if ti["kind"] != oracle.KIND_RANS:
            continue
        assert ti["coded_bytes"] * 8 >= conditional_entropy_bits(w) * (1 - 1e-9), s.name


@pytest.mark.parametrize("name", ["tensor_1m", "gemma2_layer"])
def test_overhead_within_half_percent(name):
    specs = [s for s in S.workload(name) if not s.is_raw]
    arrs = [_words(s) for s in specs]
    c = oracle.encode([(s.name, a, "bf16") for s, a in zip(specs, arrs)])
    coded = sum(oracle.info(c, k)["coded_bytes"] for k in range(len(specs)))
    h = sum(conditional_entropy_bits(a) for a in arrs)
    assert coded * 8 >= h
    assert coded * 8 <= 1.005 * h, (coded * 8 / sum(a.size for a in arrs), h / sum(a.size for a in arrs))


# ---------------------------------------------------------------- host-made faults
def _container():
    w = _words(S.workload("tensor_1m")[0]).reshape(-1)[:200_000]
    return w, bytearray(oracle.encode([("w", w, "bf16")]))


def test_fault_payload_bitflips_are_detected():
    # A flip that desynchronises a lane fails the end check (E_CORRUPT from the chunk).
    # A flip inside a near-uniform fraction can change one weight and stay in sync; the
    # per-tensor checksum catches those. Flips in padding change nothing.
    w, c = _container()
    ti = oracle.info(bytes(c), 0)
    first_chunk = int.from_bytes(c[ti["data_offset"]:ti["data_offset"] + 8], "little")
    rng = np.random.default_rng(3)
    outcomes = {"chunk": 0, "checksum": 0, "none": 0}
    for _ in range(60):
        bad = bytearray(c)
        pos = int(rng.integers(first_chunk, len(c) - 16))
        bad[pos] ^= 1 << int(rng.integers(0, 8))
        out = np.zeros(w.size, np.uint16)
        st = oracle.decode_chunks(bytes(bad), 0, 0, ti["n_chunks"], out)
        if st:
            assert st == oracle.E_CORRUPT
            outcomes["chunk"] += 1
            continue
        if np.array_equal(out, w):
            outcomes["none"] += 1
            continue
        with pytest.raises(oracle.OracleError) as e:
            oracle.decode(bytes(bad), 0)
        assert e.value.code == oracle.E_CORRUPT
        outcomes["checksum"] += 1
    assert outcomes["chunk"] > 0 and outcomes["checksum"] > 0


def test_fault_truncation_and_header():
    _, c = _container()
    for cut in (0, 10, 63, 64, 500, len(c) - 16):
        with pytest.raises(oracle.OracleError):
            oracle.validate(bytes(c[:cut]))
    bad = bytearray(c)
    bad[0] ^= 0xFF
    with pytest.raises(oracle.OracleError) as e:
        oracle.validate(bytes(bad))
    assert e.value.code == oracle.E_FORMAT
    for version in (1, 3):           # version 1 (64-bit states) is not read by version-2 decoders
        bad = bytearray(c)
        bad[8] = version
        with pytest.raises(oracle.OracleError) as e:
            oracle.validate(bytes(bad))
        assert e.value.code == oracle.E_VERSION


def test_fault_table_sum_and_offsets():
    _, c = _container()
    ti = oracle.info(bytes(c), 0)
    bad = bytearray(c)
    bad[ti["model_offset"] + 6] ^= 1                       # first s frequency
    with pytest.raises(oracle.OracleError):
        oracle.validate(bytes(bad))
    bad = bytearray(c)
    bad[ti["data_offset"] + 2] ^= 0x40                     # chunk 0 offset far out of range
    with pytest.raises(oracle.OracleError):
        oracle.validate(bytes(bad))
    bad = bytearray(c)
    bad[ti["data_offset"]] ^= 0x04                         # unaligned chunk offset
    with pytest.raises(oracle.OracleError):
        oracle.validate(bytes(bad))


def test_fault_reserved_fields():
    # a nonzero reserved field makes a container invalid: the RANS model's second u16, the
    # directory entry's reserved u64, the header's reserved u64
    _, c = _container()
    ti = oracle.info(bytes(c), 0)
    dir_off = int.from_bytes(bytes(c[24:32]), "little")
    for off in (ti["model_offset"] + 2, dir_off + 72, 56):
        bad = bytearray(c)
        bad[off] = 1
        with pytest.raises(oracle.OracleError) as e:
            oracle.validate(bytes(bad))
        assert e.value.code == oracle.E_FORMAT
