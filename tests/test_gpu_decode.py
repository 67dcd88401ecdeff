"""GPU parity: the CUDA decode path against the original words and the oracle.

The oracle encodes each container. libbs decodes it on the device through the C ABI.
Outputs are compared bit-exact as 16-bit integers (never as bf16, since NaN != NaN):
against the original words and against the oracle's decode of the same container.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _host(t: torch.Tensor) -> np.ndarray:
    a = t.detach().cpu().contiguous().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _decode_all(container, n):
    plan = bs.Plan(container, device="cuda:0")
    outs = plan.decode_batch(range(n))
    plan.check()
    return plan, [_host(o) for o in outs]


def _items(specs):
    arrs = [S.words_numpy(S.generate(s, "cpu")) for s in specs]
    return arrs, [(s.name, a, "raw" if s.is_raw else "bf16") for s, a in zip(specs, arrs)]


def test_tensor_1m_bit_exact():
    arrs, items = _items(S.workload("tensor_1m"))
    c = oracle.encode(items)
    plan, outs = _decode_all(c, 1)
    assert np.array_equal(outs[0].reshape(arrs[0].shape), arrs[0])
    assert np.array_equal(outs[0].reshape(arrs[0].shape), oracle.decode(c, 0))
    plan.verify(0, plan.decode(0))


@pytest.mark.parametrize("force_rans", [False, True])
def test_edge_mix_bit_exact(force_rans):
    specs = S.workload("edge_mix")
    arrs, items = _items(specs)
    c = oracle.encode(items, force_rans=force_rans)
    plan, outs = _decode_all(c, len(specs))
    for k, (s, a) in enumerate(zip(specs, arrs)):
        assert np.array_equal(outs[k].reshape(a.shape), a), s.name
        plan.verify(k, plan.decode(k))


def test_every_bit_pattern():
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(0)
    items = [("all", w, "bf16"), ("shuffled", rng.permutation(w), "bf16")]
    items += [(f"p{k}", w[k:k + 1], "bf16") for k in range(0, 65536, 97)]   # ±0, subnormals, inf, NaNs
    items += [(f"s{k}", w[k:k + 1], "bf16") for k in (0x0000, 0x8000, 0x0001, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF)]
    c = oracle.encode(items, force_rans=True)
    _, outs = _decode_all(c, len(items))
    for k, (_, a, _) in enumerate(items):
        assert np.array_equal(outs[k], a)


def test_sizes_and_multiple_launches():
    # 1033 tensors: more RANS tensors than one launch carries (500), every tail length
    rng = np.random.default_rng(11)
    sizes = list(range(1, 1026)) + [4095, 4096, 4097, 65535, 65536, 65537, 3 * 65536 + 255]
    items = []
    for n in sizes:
        x = (rng.standard_normal(n) * 0.03).astype(np.float32)
        items.append((f"n{n}", (x.view(np.uint32) >> 16).astype(np.uint16), "bf16"))
    c = oracle.encode(items, force_rans=True)
    _, outs = _decode_all(c, len(items))
    for k, (_, a, _) in enumerate(items):
        assert np.array_equal(outs[k], a), sizes[k]


@pytest.mark.parametrize("log2_chunk,ns,nh", [(8, 11, 5), (12, 11, 3), (16, 1, 3), (16, 8, 5), (17, 12, 3),
                                               (20, 11, 5), (16, 12, 4)])
def test_parameters(log2_chunk, ns, nh):
    w = S.words_numpy(S.generate(S.workload("tensor_1m")[0], "cpu")).reshape(-1)[:700_001].copy()
    if ns < 9:
        w = np.where(np.arange(w.size) % 3 == 0, 0x3C00, 0xBC31).astype(np.uint16)
    c = oracle.encode([("w", w, "bf16")], log2_chunk=log2_chunk, ns=ns, nh=nh, force_rans=True)
    _, outs = _decode_all(c, 1)
    assert np.array_equal(outs[0], w)


@pytest.mark.parametrize("ns,nh", [(11, 5), (12, 4)])
def test_largest_tables(ns, nh):
    # 15 routes (16 fraction rows with UNIFORM) and, at ns = 12, the largest s-table (32 KiB):
    # the most shared memory any valid container asks for
    w = np.concatenate([((e << 7) | ((np.arange(3000) % (3 + e % 5)) << 4) | (np.arange(3000) % 16)).astype(np.uint16)
                        for e in range(90, 110)])
    c = oracle.encode([("skewed", w, "bf16")], ns=ns, nh=nh, max_routes=15)
    assert oracle.info(c, 0)["n_routes"] == 15
    _, outs = _decode_all(c, 1)
    assert np.array_equal(outs[0], w)


def test_gemma2_layer_bit_exact():
    specs = S.workload("gemma2_layer")
    arrs, items = _items(specs)
    c = oracle.encode(items)
    plan, outs = _decode_all(c, len(specs))
    for k, a in enumerate(arrs):
        assert np.array_equal(outs[k].reshape(a.shape), a), specs[k].name


def test_streams_concurrent_disjoint_outputs():
    arrs, items = _items(S.workload("edge_mix")[:2] + S.workload("tensor_1m"))
    c = oracle.encode(items)
    plan = bs.Plan(c, device="cuda:0")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    o = [plan.empty_output(k) for k in range(3)]
    plan.decode(0, o[0], stream=s1)
    plan.decode(1, o[1], stream=s2)
    plan.decode(2, o[2], stream=s1)
    torch.cuda.synchronize()
    plan.check()
    for k, a in enumerate(arrs):
        assert np.array_equal(_host(o[k]).reshape(a.shape), a)


def test_corrupt_chunk_is_reported():
    # host-made fault: a flipped bit in chunk 2's start state
    arrs, items = _items(S.workload("tensor_1m"))
    c = bytearray(oracle.encode(items))
    ti = oracle.info(bytes(c), 0)
    e2 = ti["data_offset"] + 16 * 2
    off2 = int.from_bytes(c[e2:e2 + 8], "little")
    c[off2 + 4 * 5 + 2] ^= 0x10                        # lane 5's state, bit 20
    plan = bs.Plan(bytes(c), device="cuda:0")
    plan.decode(0)
    with pytest.raises(bs.BsError) as e:
        plan.check()
    assert e.value.code == bs.E_CORRUPT and e.value.first_bad == (0 << 40) | 2
    assert oracle.decode_chunks(bytes(c), 0, 2, 3, np.zeros(arrs[0].size, np.uint16)) == oracle.E_CORRUPT
    plan.check()                                        # the error word was cleared


def test_in_sync_flip_caught_by_checksum():
    # a flip in a stored nibble changes one weight without any desync: the checksum catches it
    w = np.full(70_000, 0x3C00, np.uint16) | (np.arange(70_000, dtype=np.uint16) & 0x7F)   # one exponent, flat
    c = bytearray(oracle.encode([("w", w, "bf16")], force_rans=True))
    ti = oracle.info(bytes(c), 0)
    assert ti["nib_mode"] == 0
    e0 = ti["data_offset"]
    off0 = int.from_bytes(c[e0:e0 + 8], "little")
    c[off0 + 128 + 4 * 40 + 1] ^= 0x04                  # nibble word 40 (block 1, lane 8), bit 10
    plan = bs.Plan(bytes(c), device="cuda:0")
    out = plan.decode(0)
    plan.check()
    got = _host(out)
    assert int(np.count_nonzero(got != w)) == 1         # weight 256 + 8*8 + 4: its nibble's bit 2
    assert int(got[256 + 64 + 4]) == int(w[256 + 64 + 4]) ^ 0x4
    with pytest.raises(bs.BsError) as e:
        plan.verify(0, out)
    assert e.value.code == bs.E_CORRUPT


def test_bad_arguments():
    arrs, items = _items(S.workload("tensor_1m"))
    c = oracle.encode(items)
    plan = bs.Plan(c, device="cuda:0")
    small = torch.empty(10, dtype=torch.int16, device="cuda:0")
    with pytest.raises(bs.BsError) as e:
        plan.decode(0, small)
    assert e.value.code == bs.E_SIZE
    buf = torch.empty(arrs[0].size + 8, dtype=torch.int16, device="cuda:0")
    with pytest.raises(bs.BsError) as e:
        plan.decode(0, buf[1:1 + arrs[0].size])      # misaligned output
    assert e.value.code == bs.E_ARG
    with pytest.raises(bs.BsError):
        bs.Plan(c[:-16], device="cuda:0")


def _golden(name):
    import os
    hexs = []
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as fh:
        for line in fh:
            hexs.append(line.split("#", 1)[0])
    return bytes.fromhex("".join("".join(hexs).split()))


@pytest.mark.parametrize("name", ["one_weight.hex", "two_weights.hex", "interleave_sixteen.hex",
                                  "joint_two_weights.hex", "joint_interleave_sixteen.hex"])
def test_hand_derived_containers(name):
    # the containers derived by hand in the golden files' comments, decoded on the device;
    # the interleave pair fixes the (step, lane) order in which the warp takes the words
    c = _golden(name)
    want = oracle.decode(c, 0)
    plan, outs = _decode_all(c, 1)
    assert np.array_equal(outs[0].reshape(-1), want.reshape(-1))
    if "sixteen" in name:
        assert outs[0].reshape(-1).tolist() == [0x3F80 + 16 * h for h in range(8)] + [0x4000 + 16 * h for h in range(8)]
