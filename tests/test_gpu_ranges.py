"""GPU parity of bs_decode_ranges: parts of tensors, in whole chunks, through the C ABI.

* Every tensor of workloads 1, 2 and 4, cut into ranges of mixed lengths (chunk-aligned
  for coded kinds, arbitrary for STORED and RAW), decodes to exactly the matching slice
  of its original, for both coded kinds.
* A checkpoint cut into fixed-size batches of chunks, batches crossing tensor boundaries
  and splitting tensors, one call per batch, reassembles bit-exact.
* Misaligned or out-of-range requests are refused before anything is launched.
* A corrupt chunk inside a range is reported with the tensor's own chunk index.
Words are compared as 16-bit integers.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _host(t):
    a = t.detach().cpu().contiguous().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _items(specs):
    arrs = [S.words_numpy(S.generate(s, "cpu")).reshape(-1) for s in specs]
    return arrs, [(s.name, a, "raw" if s.is_raw else "bf16") for s, a in zip(specs, arrs)]


def _out(plan, idx, count):
    raw = plan.info(idx)["kind"] == bs.KIND_RAW
    return torch.empty(max(count, 0), dtype=torch.uint8 if raw else torch.int16, device="cuda:0")


def _cuts(n, C, coded, rng):
    """Split [0, n) into ranges: multiples of C for coded kinds (the last may be ragged)."""
    cuts, b = [], 0
    while b < n:
        if coded:
            cnt = int(rng.integers(1, 4)) * C
        else:
            cnt = int(rng.integers(1, max(2, n // 3 + 1)))
        cnt = min(cnt, n - b)
        cuts.append((b, cnt))
        b += cnt
    return cuts


@pytest.mark.parametrize("model", ["factored", "joint"])
def test_ranges_reassemble_every_tensor(model):
    specs = S.workload("tensor_1m") + S.workload("edge_mix")
    arrs, items = _items(specs)
    c = oracle.encode(items, log2_chunk=12, model=model)
    plan = bs.Plan(c, device="cuda:0")
    rng = np.random.default_rng(1)
    for k, a in enumerate(arrs):
        info = plan.info(k)
        coded = info["kind"] in (bs.KIND_RANS, bs.KIND_JOINT)
        cuts = _cuts(a.size, 1 << 12, coded, rng)
        ranges = [(k, b, cnt, _out(plan, k, cnt)) for b, cnt in cuts]
        rng.shuffle(ranges)
        plan.decode_ranges(ranges)
        plan.check()
        got = np.zeros_like(a)
        for _, b, cnt, o in ranges:
            got[b:b + cnt] = _host(o)
        assert np.array_equal(got, a), specs[k].name


def test_fixed_size_batches_across_tensors():
    # batches of 7 chunks of 4096 weights, the way a checkpoint is decoded a fixed amount
    # of output at a time: batches end inside tensors and the next one continues them
    specs = S.workload("gemma2_layer")
    arrs, items = _items(specs)
    C = 1 << 12
    c = oracle.encode(items, log2_chunk=12, model="joint")
    plan = bs.Plan(c, device="cuda:0")
    assert any(a.size % (7 * C) for a in arrs)          # batches do split tensors
    got = [np.full_like(a, 0x5555) for a in arrs]
    units = [(k, b, min(C, a.size - b)) for k, a in enumerate(arrs) for b in range(0, a.size, C)]
    for i in range(0, len(units), 7):                   # one batch: 7 chunks, one call
        ranges = []
        for k, b, cnt in units[i:i + 7]:                # runs of one tensor become one range
            if ranges and ranges[-1][0] == k:
                ranges[-1] = (k, ranges[-1][1], ranges[-1][2] + cnt)
            else:
                ranges.append((k, b, cnt))
        outs = plan.decode_ranges([(k, b, cnt, _out(plan, k, cnt)) for k, b, cnt in ranges])
        for (k, b, cnt), o in zip(ranges, outs):
            got[k][b:b + cnt] = _host(o)
    plan.check()
    for k, a in enumerate(arrs):
        assert np.array_equal(got[k], a), specs[k].name


def test_refused_requests():
    specs = S.workload("tensor_1m")
    arrs, items = _items(specs)
    c = oracle.encode(items + [("raw", np.arange(100, dtype=np.uint8), "raw")], log2_chunk=12, model="joint")
    plan = bs.Plan(c, device="cuda:0")
    n = arrs[0].size
    C = 1 << 12
    bad = [
        ((0, 100, C, _out(plan, 0, C)), bs.E_ARG),              # begin not on a chunk
        ((0, 0, C + 5, _out(plan, 0, C + 5)), bs.E_ARG),        # end inside a chunk
        ((0, n - C, 2 * C, _out(plan, 0, 2 * C)), bs.E_ARG),    # past the end
        ((0, 0, C, _out(plan, 0, C - 1)), bs.E_SIZE),           # out_bytes
        ((1, 90, 20, _out(plan, 1, 20)), bs.E_ARG),             # RAW past the end
        ((2, 0, 1, _out(plan, 0, 1)), bs.E_ARG),                # no such tensor
    ]
    for r, code in bad:
        with pytest.raises(bs.BsError) as e:
            plan.decode_ranges([r])
        assert e.value.code == code, r[:3]
    # a coded range into a 16-byte-misaligned output
    buf = torch.empty(C + 8, dtype=torch.int16, device="cuda:0")
    with pytest.raises(bs.BsError) as e:
        plan.decode_ranges([(0, 0, C, buf[1:C + 1])])
    assert e.value.code == bs.E_ARG
    # the same check on the whole-tensor call for a JOINT tensor
    big = torch.empty(n + 8, dtype=torch.int16, device="cuda:0")
    with pytest.raises(bs.BsError) as e:
        plan.decode(0, big[1:n + 1])
    assert e.value.code == bs.E_ARG
    # empty ranges are fine anywhere inside the tensor, RAW ranges may start anywhere
    o = _out(plan, 1, 30)
    plan.decode_ranges([(0, C, 0, _out(plan, 0, 0)), (0, 77, 0, _out(plan, 0, 0)), (0, n, 0, _out(plan, 0, 0)),
                        (1, 37, 30, o)])
    plan.check()
    assert np.array_equal(_host(o), np.arange(37, 67, dtype=np.uint8))


def test_corrupt_chunk_reported_with_its_tensor_index():
    specs = S.workload("tensor_1m")
    arrs, items = _items(specs)
    c = bytearray(oracle.encode(items, log2_chunk=12, model="joint"))
    ti = oracle.info(bytes(c), 0)
    e0 = ti["data_offset"] + 16 * 37
    off = int.from_bytes(c[e0:e0 + 8], "little")
    c[off + 4 * 3 + 2] ^= 0x08                      # chunk 37, lane 3's start state
    plan = bs.Plan(bytes(c), device="cuda:0")
    C = 1 << 12
    plan.decode_ranges([(0, 32 * C, 8 * C, _out(plan, 0, 8 * C))])
    with pytest.raises(bs.BsError) as e:
        plan.check()
    assert e.value.code == bs.E_CORRUPT
    assert e.value.first_bad == 37
    # a range that leaves chunk 37 out decodes clean
    o = _out(plan, 0, 32 * C)
    plan.decode_ranges([(0, 0, 32 * C, o)])
    plan.check()
    assert np.array_equal(_host(o), arrs[0][:32 * C])


def test_decode_geometry():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = S.words_numpy(S.generate(S.workload("tensor_1m")[0], "cpu")).reshape(-1)
    items = [("joint", w, "bf16"), ("u", np.arange(1 << 16, dtype=np.uint32).astype(np.uint16), "bf16")]
    plan = bs.Plan(oracle.encode(items, model="joint"), device="cuda:0")
    assert plan.info(1)["kind"] == bs.KIND_STORED
    assert plan.decode_geometry(0) == (64, sms)       # JOINT, 4-byte entries: 32 warps of 2 chunks, one CTA per SM
    assert plan.decode_geometry(1) == (0, sms)
    fplan = bs.Plan(oracle.encode(items[:1]), device="cuda:0")
    assert fplan.decode_geometry(0) == (48, sms)      # RANS, default precisions: 24 warps of 2
    gplan = bs.Plan(oracle.encode(items[:1], ns=10, nh=4), device="cuda:0")
    assert gplan.decode_geometry(0) == (40, sms)      # other precisions: 20 warps of 2
    # a JOINT tensor with a pair of frequency above 255 keeps 8-byte entries: 28 warps of 2
    skew = np.full(5000, 0x3F80, np.uint16)
    skew[::7] = 0x3F90
    jplan = bs.Plan(oracle.encode([("skew", skew, "bf16")], model="joint", force_rans=True), device="cuda:0")
    assert jplan.info(0)["kind"] == bs.KIND_JOINT and jplan.decode_geometry(0) == (56, sms)
    with pytest.raises(bs.BsError) as e:
        plan.decode_geometry(2)
    assert e.value.code == bs.E_ARG
