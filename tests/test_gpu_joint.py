"""GPU parity of the JOINT kind (one table over the pairs (s, h)) through the C ABI.

* Containers the oracle encodes decode bit-exact on the device, against the originals and
  against the oracle's own decode: nj = 13 (the compile-time kernel instance) and 8..12
  (the generic one), several chunk sizes with ragged tails, and every 16-bit pattern.
* The device encoder writes the oracle's bytes for the JOINT kind.
* The no-alloc entry point and the layer streamer decode JOINT tensors.
* A corrupt chunk is reported.
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
    arrs = [S.words_numpy(S.generate(s, "cpu")) for s in specs]
    return arrs, [(s.name, a, "raw" if s.is_raw else "bf16") for s, a in zip(specs, arrs)]


def _decode_all(c, n):
    plan = bs.Plan(c, device="cuda:0")
    outs = plan.decode_batch(range(n))
    plan.check()
    return plan, [_host(o) for o in outs]


def test_tensor_1m_and_gemma2_layer():
    specs = S.workload("tensor_1m") + S.workload("gemma2_layer")
    arrs, items = _items(specs)
    c = oracle.encode(items, model="joint")
    plan, outs = _decode_all(c, len(specs))
    for k, a in enumerate(arrs):
        assert plan.info(k)["kind"] == bs.KIND_JOINT
        assert np.array_equal(outs[k].reshape(a.shape), a), specs[k].name
    assert np.array_equal(outs[0].reshape(arrs[0].shape), oracle.decode(c, 0))
    plan.verify(0, plan.decode(0))


@pytest.mark.parametrize("force_rans", [False, True])
def test_edge_mix(force_rans):
    specs = S.workload("edge_mix")
    arrs, items = _items(specs)
    c = oracle.encode(items, model="joint", force_rans=force_rans)
    plan, outs = _decode_all(c, len(specs))
    for k, (s, a) in enumerate(zip(specs, arrs)):
        assert np.array_equal(outs[k].reshape(a.shape), a), s.name
        plan.verify(k, plan.decode(k))


def test_every_bit_pattern():
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(0)
    items = [("all", w, "bf16"), ("shuffled", rng.permutation(w), "bf16")]
    items += [(f"p{k}", w[k:k + 1], "bf16") for k in range(0, 65536, 211)]
    c = oracle.encode(items, model="joint", force_rans=True)
    _, outs = _decode_all(c, len(items))
    for (nm, a, _), o in zip(items, outs):
        assert np.array_equal(o, a), nm


@pytest.mark.parametrize("nj,log2_chunk", [(8, 12), (10, 16), (12, 8), (13, 17), (13, 9)])
def test_precisions_and_ragged_chunks(nj, log2_chunk):
    w = S.words_numpy(S.generate(S.workload("tensor_1m")[0], "cpu")).reshape(-1)[: 3 * (1 << 16) + 77]
    if nj < 10:   # keep the pair alphabet below 2^nj
        w = np.where(np.arange(w.size) % 3 == 0, 0x3C00, 0xBC31).astype(np.uint16)
    c = oracle.encode([("w", w, "bf16")], model="joint", nj=nj, log2_chunk=log2_chunk, force_rans=True)
    _, outs = _decode_all(c, 1)
    assert np.array_equal(outs[0], w)


@pytest.mark.parametrize("kw", [dict(), dict(nj=10), dict(nj=13, log2_chunk=12), dict(force_rans=True)])
def test_device_encoder_matches_oracle_bytes(kw):
    specs = S.workload("edge_mix") + S.workload("tensor_1m")
    gen = [S.generate(s, "cpu") for s in specs]          # one draw, copied to the device
    cpu = [S.words_numpy(t) for t in gen]
    dev = [(s.name, t.to("cuda:0")) for s, t in zip(specs, gen)]
    _, h_c = bs.encode(dev, host_copy=True, model="joint", **kw)
    want = oracle.encode([(s.name, a, "raw" if s.is_raw else "bf16") for s, a in zip(specs, cpu)], model="joint",
                         **kw)
    assert bytes(h_c.tobytes()) == want


def test_device_encoder_round_trip_gemma2_layer():
    specs = S.workload("gemma2_layer")
    dev = [(s.name, S.generate(s, "cuda:0")) for s in specs]
    d_c, _ = bs.encode(dev, model="joint")
    plan = bs.Plan(d_container=d_c)
    outs = plan.decode_batch(range(len(specs)))
    plan.check()
    for (nm, t), o in zip(dev, outs):
        assert torch.equal(o.reshape(-1), t.reshape(-1)), nm


def test_noalloc_decodes_joint_tensors():
    specs = S.workload("tensor_1m") + [s for s in S.workload("edge_mix") if s.name in ("ragged", "one")]
    arrs, items = _items(specs)
    for nj in (13, 10):
        c = oracle.encode(items, model="joint", nj=nj, force_rans=True)
        plan = bs.Plan(c, device="cuda:0")
        for k, a in enumerate(arrs):
            got = plan.empty_output(k)
            got.fill_(0x55)
            bs.decode_noalloc(c, plan.d_container, k, got)
            torch.cuda.synchronize()
            assert np.array_equal(_host(got).reshape(a.shape), a), (nj, specs[k].name)


def test_streamer_with_a_joint_container():
    specs = S.workload("gemma2_9b", layers=2) + S.workload("edge_mix")
    dev = [(s.name, S.generate(s, "cuda:0")) for s in specs]
    _, h_c = bs.encode(dev, host_copy=True, model="joint")
    key = lambda name: name.split(".")[1] if name.startswith("layers.") else "misc"
    st = bs.Streamer(h_c, key)
    for g in list(range(st.n_groups)) * 2:
        outs = st.acquire(g)
        for k, o in zip(st.members[g], outs):
            assert torch.equal(o.reshape(-1), dev[k][1].reshape(-1)), specs[k].name
        st.release(g)
    st.check()


def test_corrupt_chunk_is_reported():
    specs = S.workload("tensor_1m")
    arrs, items = _items(specs)
    c = bytearray(oracle.encode(items, model="joint"))
    ti = oracle.info(bytes(c), 0)
    e0 = ti["data_offset"] + 16 * 5
    off = int.from_bytes(c[e0:e0 + 8], "little")
    c[off + 4 * 9 + 2] ^= 0x08                       # chunk 5, lane 9's start state
    plan = bs.Plan(bytes(c), device="cuda:0")
    plan.decode(0)
    with pytest.raises(bs.BsError) as e:
        plan.check()
    assert e.value.code == bs.E_CORRUPT
    assert e.value.first_bad == 5
