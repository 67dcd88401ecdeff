"""bs_decode_tensor_noalloc: decoding without a caller workspace.

Some callers cannot allocate device memory. Examples are a plugin inside another runtime
whose allocator owns the whole GPU, or a callback where an allocation would synchronise the
device. For them, libbs keeps the decode tables and the error block in a static device array
instead of a workspace.

This test calls that entry point through the C ABI and checks its output against the
regular bs_decode_tensor on the same container, bit-exact (the tolerance of every decode
test here), on two calls in a row. The file sorts last so that a run stopping at the first
failure has already run everything else.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _container():
    specs = S.workload("tensor_1m") + [s for s in S.workload("edge_mix") if s.name in ("ragged", "one", "raw_span")]
    arrs = [S.words_numpy(S.generate(s, "cpu")) for s in specs]
    c = oracle.encode([(s.name, a, "raw" if s.is_raw else "bf16") for s, a in zip(specs, arrs)])
    return specs, arrs, c


def test_noalloc_matches_regular_decode_twice():
    specs, arrs, c = _container()
    plan = bs.Plan(c, device="cuda:0")
    d_c = plan.d_container
    for k in [0, 1, 0, 3]:       # two calls in a row on tensor 0, then others, then 0 again
        want = plan.decode(k)
        got = plan.empty_output(k)
        got.fill_(0x55)
        bs.decode_noalloc(c, d_c, k, got)
        torch.cuda.synchronize()
        assert torch.equal(got, want), specs[k].name
        a = got.cpu().numpy()
        a = a.view(np.uint16) if a.dtype == np.int16 else a
        assert np.array_equal(a.reshape(arrs[k].shape), arrs[k])
    plan.check()


def test_noalloc_reports_corrupt_chunk_and_oversized_tables():
    specs, arrs, c = _container()
    bad = bytearray(c)
    ti = oracle.info(c, 0)
    e0 = ti["data_offset"] + 16 * 3
    off = int.from_bytes(bad[e0:e0 + 8], "little")
    bad[off + 4 * 7 + 2] ^= 0x20                       # chunk 3, lane 7's start state, bit 21
    d_bad = torch.from_numpy(np.frombuffer(bytes(bad), np.uint8).copy()).cuda()
    out = torch.empty(arrs[0].shape, dtype=torch.int16, device="cuda:0")
    with pytest.raises(bs.BsError) as e:
        bs.decode_noalloc(bytes(bad), d_bad, 0, out)
    assert e.value.code == bs.E_CORRUPT
    # a clean call right after: the shared error block starts from zero again
    d_c = torch.from_numpy(np.frombuffer(c, np.uint8).copy()).cuda()
    bs.decode_noalloc(c, d_c, 0, out)
    assert np.array_equal(out.cpu().numpy().view(np.uint16).reshape(arrs[0].shape), arrs[0])
    # the largest tables a valid container has (ns = 12 and 15 routes: 32 KiB + 2 KiB) fit
    # the static array: 16 exponents, each with a skewed top-bit distribution
    w = np.concatenate([((e << 7) | ((np.arange(1000) % 3) << 4) | (np.arange(1000) % 16)).astype(np.uint16)
                        for e in range(100, 116)])
    big = oracle.encode([("skewed", w, "bf16")], ns=12, nh=4, max_routes=15)
    assert oracle.info(big, 0)["n_routes"] == 15
    d_big = torch.from_numpy(np.frombuffer(big, np.uint8).copy()).cuda()
    out = torch.empty(w.size, dtype=torch.int16, device="cuda:0")
    bs.decode_noalloc(big, d_big, 0, out)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
    # a directory entry with ns = 13 is refused before any device work
    bad = bytearray(big)
    dir_off = int.from_bytes(bad[24:32], "little")
    bad[dir_off + 4] = 13
    with pytest.raises(bs.BsError) as e:
        bs.decode_noalloc(bytes(bad), d_big, 0, out)
    assert e.value.code == bs.E_FORMAT


@pytest.mark.parametrize("model,compact", [("joint", True), ("joint", False), ("factored", None)])
def test_noalloc_matches_regular_decode_for_each_table_kind(model, compact):
    # Both entry points validate with the same rules and build their tables with the same
    # builder; the no-alloc one keeps them in the static array. Checked on two calls in a row
    # for the JOINT tables with 4-byte entries (every frequency at most 255) and 8-byte ones,
    # and for the largest factored tables (ns = 12, 15 routes).
    rng = np.random.default_rng(3)
    if model == "factored":
        w = np.concatenate([((e << 7) | ((np.arange(20000) % 3) << 4) | (np.arange(20000) % 16)).astype(np.uint16)
                            for e in range(100, 116)])
        c = oracle.encode([("t", w, "bf16")], ns=12, nh=4, max_routes=15, log2_chunk=12)
        assert oracle.info(c, 0)["n_routes"] == 15
    else:
        x = rng.standard_normal(300_000).astype(np.float32) * 0.02
        w = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
        if not compact:
            w[::3] = 0x3F80                    # one pair takes a third of the slots: F above 255
        c = oracle.encode([("t", w, "bf16")], model="joint", log2_chunk=12)
    plan = bs.Plan(c, device="cuda:0")
    want = plan.decode(0)
    for _ in range(2):
        got = plan.empty_output(0)
        got.fill_(0x55)
        bs.decode_noalloc(c, plan.d_container, 0, got)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
    assert np.array_equal(S.words_numpy(want).reshape(-1), w)
    plan.check()
