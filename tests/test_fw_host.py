"""CPU checks of the FW layout's host side in libbs (no GPU): bs_fw_parse against the
oracle's layouts and header fields, argument checks of bs_fw_decode, and the refusal of the
device calls without a GPU."""
import ctypes
import struct

import numpy as np
import pytest
import torch

import oracle

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _gauss(n, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    return ((rng.standard_normal(n) * scale).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("n", [0, 1, 17, 256, 1000])
def test_parse_matches_oracle_header(n):
    blob = oracle.fw_encode(_gauss(n, n, scale=1.0))
    want = oracle.fw_info(blob)
    got = bs.fw_parse(np.frombuffer(blob, np.uint8)[:96], len(blob))
    assert (got.n_elems, got.n_tiles, got.n_exc, got.total_bytes) == \
        (want["n_elems"], want["n_tiles"], want["n_exc"], want["total_bytes"])
    assert list(got.table) == want["table"]


def _bad(blob, off, fmt, v):
    b = bytearray(blob[:96])
    struct.pack_into(fmt, b, off, v)
    return np.frombuffer(bytes(b), np.uint8)


def test_parse_refuses_bad_headers():
    blob = oracle.fw_encode(_gauss(700, 1, scale=1.0))
    n = len(blob)
    head = np.frombuffer(blob, np.uint8)[:96]
    with pytest.raises(bs.BsError) as e:
        bs.fw_parse(head, n + 16)                       # size differs from total_bytes
    assert e.value.code == bs.E_FORMAT
    with pytest.raises(bs.BsError) as e:
        bs.fw_parse(head[:80], n)                       # short head
    assert e.value.code == bs.E_FORMAT
    cases = [((0, "<B", 0x41), bs.E_FORMAT), ((8, "<I", 2), bs.E_VERSION), ((12, "<I", 96), bs.E_FORMAT),
             ((24, "<Q", 1), bs.E_FORMAT), ((32, "<Q", 701), bs.E_FORMAT), ((63, "<B", 1), bs.E_FORMAT),
             ((64 + 30, "<H", 600), bs.E_FORMAT)]
    for (off, fmt, v), code in cases:
        with pytest.raises(bs.BsError) as e:
            bs.fw_parse(_bad(blob, off, fmt, v), n)
        assert e.value.code == code, (off, v)


def test_scratch_bytes():
    assert bs.fw_scratch_bytes(0) > 0
    assert bs.fw_scratch_bytes(1 << 20) > bs.fw_scratch_bytes(1 << 10)
    assert bs.fw_scratch_bytes((1 << 40) + 1) == 0


def test_decode_argument_checks_before_any_launch():
    blob = oracle.fw_encode(_gauss(300, 2))
    info = bs.fw_parse(np.frombuffer(blob, np.uint8)[:96], len(blob))
    P = ctypes.c_void_p
    fws = (P * 1)(16)
    outs = (P * 1)(32)
    infos = (bs.FwInfo * 1)(info)
    sizes = (ctypes.c_size_t * 1)(2 * 300 + 2)
    assert bs.lib.bs_fw_decode(1, fws, infos, outs, sizes, 64, None) == bs.E_SIZE
    sizes[0] = 600
    assert bs.lib.bs_fw_decode(1, fws, infos, outs, sizes, None, None) == bs.E_ARG   # no error word
    outs[0] = 34                                                                      # misaligned output
    assert bs.lib.bs_fw_decode(1, fws, infos, outs, sizes, 64, None) == bs.E_ARG
    outs[0] = 32
    bad = bs.FwInfo.from_buffer_copy(info)
    bad.n_exc = bad.n_elems + 1
    infos[0] = bad
    assert bs.lib.bs_fw_decode(1, fws, infos, outs, sizes, 64, None) == bs.E_ARG
    assert bs.lib.bs_fw_decode(0, None, None, None, None, 64, None) == bs.OK       # nothing to do


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_device_calls_fail_loudly_without_gpu():
    info = bs.FwInfo()
    st = bs.lib.bs_fw_measure(256, 1, 256, bs.fw_scratch_bytes(1), None, ctypes.byref(info))
    assert st in (bs.E_CUDA, bs.E_UNSUPPORTED)
