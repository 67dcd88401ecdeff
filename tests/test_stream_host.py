"""CPU checks of the layer streamer's host side: container validation and arena sizing
(bs_streamer_workspace_bytes, bs_streamer_min_arena_bytes). No GPU call is made."""
import numpy as np
import pytest

import oracle

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _container():
    rng = np.random.default_rng(3)
    items = []
    for L in range(3):
        for nm, n in (("q", 70_000), ("k", 5_000), ("norm", 300)):
            x = (rng.standard_normal(n) * 0.02).astype(np.float32)
            items.append((f"layers.{L}.{nm}", (x.view(np.uint32) >> 16).astype(np.uint16), "bf16"))
    items.append(("raw", rng.integers(0, 256, 999, dtype=np.uint8), "raw"))
    items.append(("tiny", np.array([0x3F80], np.uint16), "bf16"))    # stored, not coded
    return items, np.frombuffer(oracle.encode(items), np.uint8)


def _u64(h, off):
    return int(h[off:off + 8].view(np.uint64)[0])


def _coded_range(h, k):
    """[begin, end) of the bytes tensor k's decode reads, from the container directory and
    chunk table: the chunk table or raw data, and every chunk's payload (section 4.5:
    128 bytes of states, 128 bytes of nibble words per 256-weight block when stored, the
    16-bit words, padded to 16 bytes)."""
    e = _u64(h, 24) + 144 * k
    kind, data_off, data_bytes, n_chunks = int(h[e]), _u64(h, e + 48), _u64(h, e + 56), _u64(h, e + 24)
    n, log2c, nib_stored = _u64(h, e + 16), int(h[e + 2]), int(h[e + 7]) == 0
    b, end = data_off, data_off + data_bytes
    if kind == 0:
        for c in range(n_chunks):
            off = _u64(h, data_off + 16 * c)
            nw = int(h[data_off + 16 * c + 8:data_off + 16 * c + 12].view(np.uint32)[0])
            nc = min(1 << log2c, n - (c << log2c))
            size = 128 + (128 * -(-nc // 256) if nib_stored else 0) + 2 * nw
            b, end = min(b, off), max(end, off + (size + 15) // 16 * 16)
    return b & ~15, end


def _up256(v):
    return (v + 255) & ~255


@pytest.mark.parametrize("grouping", ["layers", "each", "one"])
def test_min_arena_bytes(grouping):
    items, h = _container()
    names = [nm for nm, _, _ in items]
    if grouping == "layers":
        key = lambda n: n.split(".")[1] if n.startswith("layers.") else n
    elif grouping == "each":
        key = lambda n: n
    else:
        key = lambda n: 0
    keys = {}
    gid = [keys.setdefault(key(n), len(keys)) for n in names]
    stage, out = {}, {}
    for k, (nm, a, kind) in enumerate(items):
        b, e = _coded_range(h, k)
        lo, hi = stage.get(gid[k], (b, e))
        stage[gid[k]] = (min(lo, b), max(hi, e))
        out[gid[k]] = out.get(gid[k], 0) + _up256(a.size * (1 if kind == "raw" else 2))
    want = 2 * max(_up256(hi - lo) for lo, hi in stage.values()) + max(_up256(v) for v in out.values())
    assert bs.streamer_min_arena_bytes(h, key) == want
    assert bs.streamer_min_arena_bytes(h, gid) == want


def test_invalid_groupings_and_containers():
    items, h = _container()
    n = len(items)
    with pytest.raises(bs.BsError) as e:
        bs.streamer_min_arena_bytes(h, [0] * (n - 1) + [2])   # group 1 unused
    assert e.value.code == bs.E_ARG
    with pytest.raises(bs.BsError) as e:
        bs.streamer_min_arena_bytes(h, [0] * (n - 1) + [-1])
    assert e.value.code == bs.E_ARG
    with pytest.raises(bs.BsError) as e:
        bs.streamer_min_arena_bytes(h, [0] * (n - 1))        # one short
    assert e.value.code == bs.E_ARG
    bad = h.copy()
    bad[0] ^= 1                                               # magic
    with pytest.raises(bs.BsError) as e:
        bs.streamer_min_arena_bytes(bad, [0] * n)
    assert e.value.code == bs.E_FORMAT
    assert bs.lib.bs_streamer_workspace_bytes(bad.ctypes.data, bad.size) == 0
    assert bs.lib.bs_streamer_workspace_bytes(h.ctypes.data, h.size) == bs.workspace_bytes(h)
