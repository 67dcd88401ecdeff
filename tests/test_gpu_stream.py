"""GPU tests of layer streaming (bs_streamer_*): groups decoded on demand from a host
container into a bounded device cache with least-recently-used eviction.

Every group a test acquires is compared bit-exact with its originals, which are
regenerated on the device. The tests also check the cache's bookkeeping (loads, hits,
evictions) and the stream ordering: a block is not reused while queued work still reads it.
"""
import numpy as np
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _layer_key(name: str):
    return name.split(".")[1] if name.startswith("layers.") else "misc"


@pytest.fixture(scope="module", params=["factored", "joint"])
def model(request):
    """Four full-shape Gemma-2-9B layers plus the edge mix, as one host container, in kind
    RANS (the factored model) and in kind JOINT (the bench's default)."""
    specs = S.workload("gemma2_9b", layers=4) + S.workload("edge_mix")
    dev = [(s.name, S.generate(s, "cuda:0")) for s in specs]
    _, h_c = bs.encode(dev, host_copy=True, model=request.param)
    del dev
    torch.cuda.empty_cache()
    return specs, h_c


def _check_group(st, specs, group, outs):
    members = st.members[group]
    assert len(outs) == len(members)
    for k, o in zip(members, outs):
        want = S.generate(specs[k], "cuda:0")
        assert torch.equal(o.reshape(-1), want.reshape(-1)), specs[k].name


def test_min_arena_evicts_every_time(model):
    specs, h_c = model
    st = bs.Streamer(h_c, _layer_key)
    assert st.arena.numel() == st.min_arena_bytes
    order = list(range(st.n_groups)) + list(reversed(range(st.n_groups)))
    for g in order:
        outs = st.acquire(g)
        _check_group(st, specs, g, outs)
        st.release(g)
    st.check()
    stats = st.stats()
    # the last group of the first pass is still resident when the second pass starts
    assert stats["loads"] == len(order) - 1
    assert stats["hits"] == 1
    assert stats["evictions"] == stats["loads"] - 1
    assert stats["h2d_bytes"] > 0 and stats["resident_groups"] == 1


def test_cache_holds_everything(model):
    specs, h_c = model
    total = sum(2 * s.numel if not s.is_raw else s.numel for s in specs)
    st = bs.Streamer(h_c, _layer_key, arena_bytes=total + (1 << 30))
    n_groups = st.n_groups
    for _ in range(2):
        for g in range(n_groups):
            outs = st.acquire(g)
            _check_group(st, specs, g, outs)
            st.release(g)
    st.check()
    stats = st.stats()
    assert stats["loads"] == n_groups and stats["hits"] == n_groups and stats["evictions"] == 0


def test_prefetch_on_a_side_stream(model):
    """The double-buffered pattern: the next group loads on a copy stream while the
    consumer uses the current one."""
    specs, h_c = model
    keys = [_layer_key(s.name) for s in specs]
    biggest = max(sum(2 * s.numel for s, k in zip(specs, keys) if k == key) for key in set(keys))
    arena = bs.streamer_min_arena_bytes(h_c, _layer_key) + biggest + (1 << 20)
    st = bs.Streamer(h_c, _layer_key, arena_bytes=arena)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    st.prefetch(0, stream=side)
    for g in range(st.n_groups):
        if g + 1 < st.n_groups:
            st.prefetch(g + 1, stream=side)
        outs = st.acquire(g, stream=main)
        _check_group(st, specs, g, outs)
        st.release(g, stream=main)
    st.check()
    stats = st.stats()
    assert stats["loads"] == st.n_groups and stats["hits"] == st.n_groups


def test_eviction_waits_for_queued_readers(model):
    """A released group's block is reused only after work queued before the release.
    The consumer queues a long sleep, then a copy of the group. Meanwhile another stream
    loads enough groups to evict it."""
    specs, h_c = model
    st = bs.Streamer(h_c, _layer_key)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    outs = st.acquire(0, stream=main)
    torch.cuda._sleep(200_000_000)  # about 0.1 s at 2 GHz: keeps `main` busy
    copies = [o.clone() for o in outs]
    st.release(0, stream=main)
    for g in range(1, st.n_groups):  # each load evicts the previous group
        st.prefetch(g, stream=side)
    torch.cuda.synchronize()
    _check_group(st, specs, 0, copies)
    assert st.stats()["evictions"] >= 1


def test_pinned_groups_leave_no_room(model):
    _, h_c = model
    st = bs.Streamer(h_c, _layer_key)
    st.acquire(0)
    with pytest.raises(bs.BsError) as e:
        st.prefetch(1)
    assert e.value.code == bs.E_SIZE
    st.release(0)
    st.prefetch(1)
    torch.cuda.synchronize()


def test_bad_arguments(model):
    _, h_c = model
    st = bs.Streamer(h_c, _layer_key)
    n = len(st.names)
    with pytest.raises(bs.BsError) as e:
        bs.Streamer(h_c, _layer_key, arena_bytes=st.min_arena_bytes - 256)
    assert e.value.code == bs.E_SIZE
    with pytest.raises(bs.BsError) as e:
        bs.Streamer(h_c, [0] * (n - 1) + [2])  # group 1 unused
    assert e.value.code == bs.E_ARG
    with pytest.raises(bs.BsError) as e:
        st.release(0)                          # never acquired
    assert e.value.code == bs.E_ARG
    with pytest.raises(bs.BsError):
        st.acquire(st.n_groups)


def _chunk_offset(h: np.ndarray, tensor: int, chunk: int) -> int:
    # header: dir_offset at byte 24; directory entry: data_offset at 48; 16-byte chunk entries
    dir_off = int(h[24:32].view(np.uint64)[0])
    e = dir_off + 144 * tensor
    data_off = int(h[e + 48:e + 56].view(np.uint64)[0])
    return int(h[data_off + 16 * chunk:data_off + 16 * chunk + 8].view(np.uint64)[0])


def test_corrupt_chunk_is_reported(model):
    specs, h_c = model
    st = bs.Streamer(h_c, _layer_key)
    k = next(i for i, s in enumerate(specs) if s.name == "layers.2.down")
    off = _chunk_offset(h_c, k, 3)
    # lane 0's start state below 2^16 is outside the state interval: the chunk must fail
    st.host[off:off + 4] = 0
    g = next(j for j, m in enumerate(st.members) if k in m)
    st.acquire(g)
    st.release(g)
    with pytest.raises(bs.BsError) as e:
        st.check()
    assert e.value.code == bs.E_CORRUPT
    assert e.value.first_bad == (k << 40) | 3
    assert st.check() == -1  # the error word was cleared
