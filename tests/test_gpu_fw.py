"""GPU parity of the fixed-width lane layout through the C ABI.

* The device transcoder (bs_fw_measure + bs_fw_write) must produce the oracle's bytes
  exactly.
* The decode kernel (bs_fw_decode) must give back the original words exactly, both from the
  oracle's layout and from the device's.
* A corrupt exception list must raise the error flag without any write outside the output.
Words are compared as 16-bit integers.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gauss(n, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    return ((rng.standard_normal(n) * scale).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _case(name):
    if name == "one":
        return np.array([0x3F80], np.uint16)
    if name == "seventeen":
        return np.array([(i << 7) | i for i in range(17)], np.uint16)
    if name == "every_pattern":      # escapes everywhere: far more than 32 per tile
        return np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if name == "constant":
        return np.full(1000, 0xBC00, np.uint16)
    if name.startswith("gauss"):
        n = int(name[5:])
        return _gauss(n, n)
    if name == "wide":               # exponent spread wide enough that many tiles escape
        return _gauss(300_001, 5, scale=1.0) ^ (np.arange(300_001) % 3 == 0).astype(np.uint16) << 14
    raise KeyError(name)


CASES = ["one", "seventeen", "every_pattern", "constant", "gauss255", "gauss256", "gauss257", "gauss4099",
         "gauss1048653", "wide"]


def _dev(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(w.view(np.int16).copy()).cuda()


def _decode(fws, infos, ns, pad=0):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bigs = [torch.full((n + 2 * pad,), 0x5A5A, dtype=torch.int16, device="cuda") for n in ns]
    outs = [b[pad: pad + n] for b, n in zip(bigs, ns)]
    bs.fw_decode(fws, infos, outs, err)
    torch.cuda.synchronize()
    return [o.cpu().numpy().view(np.uint16) for o in outs], int(err.item()), bigs


@pytest.mark.parametrize("name", CASES)
def test_transcode_matches_oracle_bytes(name):
    w = _case(name)
    fw, info = bs.fw_transcode(_dev(w))
    want = oracle.fw_encode(w)
    assert info.total_bytes == len(want)
    assert fw.cpu().numpy().tobytes() == want


@pytest.mark.parametrize("name", CASES)
def test_decode_round_trip(name):
    w = _case(name)
    blob = oracle.fw_encode(w)
    d_blob = torch.from_numpy(np.frombuffer(blob, np.uint8).copy()).cuda()
    info = bs.fw_parse(np.frombuffer(blob, np.uint8)[:96], len(blob))
    fw, info2 = bs.fw_transcode(_dev(w))
    (a, b), err, _ = _decode([d_blob, fw], [info, info2], [w.size, w.size])
    assert err == 0
    assert np.array_equal(a, w)
    assert np.array_equal(b, w)


def _golden(name):
    out = bytearray()
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            out += bytes(int(line.split()[1])) if line.startswith("zeros") else bytes(int(x, 16) for x in line.split())
    return bytes(out)


@pytest.mark.parametrize("fname,case", [("lane_one_weight.hex", "one"), ("lane_seventeen.hex", "seventeen")])
def test_golden_layouts_decode(fname, case):
    blob = _golden(fname)
    d_blob = torch.from_numpy(np.frombuffer(blob, np.uint8).copy()).cuda()
    info = bs.fw_parse(np.frombuffer(blob, np.uint8)[:96], len(blob))
    (got,), err, _ = _decode([d_blob], [info], [info.n_elems])
    assert err == 0 and np.array_equal(got, _case(case))


def test_empty_tensor():
    fw, info = bs.fw_transcode(torch.zeros(0, dtype=torch.int16, device="cuda"))
    assert fw.cpu().numpy().tobytes() == oracle.fw_encode(np.zeros(0, np.uint16))
    (got,), err, _ = _decode([fw], [info], [0])
    assert err == 0 and got.size == 0


def test_batch_of_workload_tensors():
    specs = [s for s in S.workload("edge_mix") + S.workload("gemma2_layer") if not s.is_raw]
    words = [S.generate(s, "cuda").reshape(-1).contiguous() for s in specs]
    built = [bs.fw_transcode(w) for w in words]
    outs, err, _ = _decode([f for f, _ in built], [i for _, i in built], [w.numel() for w in words], pad=8)
    assert err == 0
    for s, w, o in zip(specs, words, outs):
        assert np.array_equal(o, w.cpu().numpy().view(np.uint16)), s.name


def test_large_tensor_round_trip_on_device():
    # 2^28 + 77 weights: the decode must give the input back; checked on the device
    n = (1 << 28) + 77
    g = torch.Generator(device="cuda").manual_seed(1)
    x = (torch.randn(n, device="cuda", generator=g) * 0.02).to(torch.bfloat16).view(torch.int16)
    fw, info = bs.fw_transcode(x)
    s = (x.view(torch.int16).to(torch.int32) & 0xFFFF) >> 7
    coded = torch.zeros(512, dtype=torch.bool, device="cuda")
    coded[torch.tensor([info.table[k] for k in range(16)], device="cuda")] = True
    hist = torch.bincount(s, minlength=512)
    assert int((hist > 0).sum()) >= 16
    assert info.n_exc == int(hist[~coded].sum())
    out = torch.empty_like(x)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bs.fw_decode([fw], [info], [out], err)
    assert int(err.item()) == 0
    assert torch.equal(out, x)


def _sections(info):
    nt, ne = info.n_tiles, info.n_exc
    te = 96 + 352 * nt
    pos = te + (4 * (nt + 1) + 15) // 16 * 16
    return te, pos


def test_corrupt_tile_exc_is_flagged_and_contained():
    w = _case("wide")[:5000]
    blob = bytearray(oracle.fw_encode(w))
    info = bs.fw_parse(np.frombuffer(bytes(blob), np.uint8)[:96], len(blob))
    te, _ = _sections(info)
    e2 = int.from_bytes(blob[te + 8: te + 12], "little")
    blob[te + 4: te + 8] = (info.n_exc + 5).to_bytes(4, "little")    # tile 0 ends past n_exc
    d = torch.from_numpy(np.frombuffer(bytes(blob), np.uint8).copy()).cuda()
    (got,), err, bigs = _decode([d], [info], [w.size], pad=64)
    assert err & 1
    big = bigs[0].cpu().numpy().view(np.uint16)
    assert (big[:64] == 0x5A5A).all() and (big[-64:] == 0x5A5A).all()
    # the kernel checks tile_exc per group of 4 tiles: tiles 4.. are untouched by the damage
    assert np.array_equal(got[1024:], w[1024:])
    assert e2 >= 0


def test_position_past_tensor_is_flagged_and_contained():
    w = _case("wide")[:256 * 4 + 100]
    blob = bytearray(oracle.fw_encode(w))
    info = bs.fw_parse(np.frombuffer(bytes(blob), np.uint8)[:96], len(blob))
    te, pos = _sections(info)
    last0 = int.from_bytes(blob[te + 4 * (info.n_tiles - 1): te + 4 * info.n_tiles], "little")
    assert last0 < info.n_exc
    blob[pos + info.n_exc - 1] = 250                                  # the last tile holds 100 weights
    d = torch.from_numpy(np.frombuffer(bytes(blob), np.uint8).copy()).cuda()
    (got,), err, bigs = _decode([d], [info], [w.size], pad=64)
    assert err & 1
    big = bigs[0].cpu().numpy().view(np.uint16)
    assert (big[:64] == 0x5A5A).all() and (big[-64:] == 0x5A5A).all()
    assert np.array_equal(got[:256 * 4], w[:256 * 4])


@pytest.mark.parametrize("model", ["factored", "joint"])
def test_layout_from_container_matches_oracle(model):
    # the runtime path: rANS container (kind RANS or JOINT) -> decode on the device -> FW
    # layout on the device
    specs = [s for s in S.workload("edge_mix") if not s.is_raw]
    arrs = [S.words_numpy(S.generate(s, "cpu")) for s in specs]
    c = oracle.encode([(s.name, a, "bf16") for s, a in zip(specs, arrs)], model=model)
    plan = bs.Plan(c, device="cuda:0")
    for k, a in enumerate(arrs):
        fw, info = plan.to_fw(k)
        assert fw.cpu().numpy().tobytes() == oracle.fw_encode(a.reshape(-1)), specs[k].name
