"""CPU checks of the boundary: libbs.so loads and exports every function include/bs.h
declares. No compute call is made (there is no GPU here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bs.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(bs_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("bs_plan", "bs_decode_tensor", "bs_decode_batch", "bs_plan_workspace_bytes", "bs_check"):
        assert want in names


def test_library_exports_every_declared_symbol():
    import lossless_entropy_coding_interleaved_b200 as bs
    lib = ctypes.CDLL(bs.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(bs.EXPORTS) == set(_declared())


def test_status_strings_and_workspace_size_on_host():
    import numpy as np
    import lossless_entropy_coding_interleaved_b200 as bs
    import oracle
    assert bs.lib.bs_status_str(bs.E_CORRUPT).decode().startswith("corrupt")
    w = np.arange(5000, dtype=np.uint16) % 300
    c = oracle.encode([("a", w, "bf16")], force_rans=True)
    n = bs.workspace_bytes(c)
    # the error block, then the s-table (8 B x 2^ns) and the compact fraction rows
    # (4 B x 2^nh per route, plus the UNIFORM row), rounded up to 256 bytes
    ti = oracle.info(c, 0)
    tables = (8 << ti["ns"]) + 4 * (ti["n_routes"] + 1) * (1 << ti["nh"])
    assert n == 256 + (tables + 255) // 256 * 256
    with pytest.raises(bs.BsError):
        bs.workspace_bytes(c[:-16])


def test_plan_without_gpu_fails_loudly():
    import torch
    import lossless_entropy_coding_interleaved_b200 as bs
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(bs.BsError):
        bs.Plan(b"\0" * 64)


def _golden(name):
    hexs = []
    with open(os.path.join(ROOT, "tests", "golden", name)) as fh:
        for line in fh:
            hexs.append(line.split("#", 1)[0])
    return bytes.fromhex("".join("".join(hexs).split()))


def test_library_parses_the_joint_golden_on_host():
    # the two-weight JOINT container derived by hand: the library's parser takes it, and the workspace
    # holds the error block and one JOINT table of 2^13 slots of 8 bytes
    import lossless_entropy_coding_interleaved_b200 as bs
    c = _golden("joint_two_weights.hex")
    assert bs.workspace_bytes(c) == 256 + (8 << 13)


def test_library_refuses_what_the_oracle_refuses():
    # the malformed JOINT containers the oracle's pins refuse (tests/test_oracle_joint.py):
    # the library's own parser must refuse each of them too
    import struct
    import lossless_entropy_coding_interleaved_b200 as bs
    c = _golden("joint_two_weights.hex")
    d, m = 64, 224
    edits = [(d + 4, "<B", 7), (d + 4, "<B", 14), (d + 5, "<B", 3), (d + 6, "<B", 1), (d + 0, "<B", 4),
             (m + 0, "<H", 0), (m + 2, "<H", 1), (m + 8, "<H", 1016), (m + 4, "<H", 4096), (m + 6, "<H", 0),
             (m + 6, "<H", 4095), (d + 40, "<Q", 16)]
    for off, fmt, v in edits:
        b = bytearray(c)
        struct.pack_into(fmt, b, off, v)
        with pytest.raises(bs.BsError):
            bs.workspace_bytes(bytes(b))


def test_library_refuses_nonzero_reserved_fields_and_unaligned_names():
    # the same rules as the oracle's: a nonzero reserved field (the RANS model's second u16,
    # the directory entry's reserved u64, the header's) and a names section off a 16-byte
    # boundary make the container invalid, for the planner and for the no-alloc entry point
    import struct
    import numpy as np
    import lossless_entropy_coding_interleaved_b200 as bs
    import oracle
    w = (np.arange(3000, dtype=np.uint16) % 97) + 0x3C00
    c = oracle.encode([("a", w, "bf16")], force_rans=True)
    ti = oracle.info(c, 0)
    dir_off = int.from_bytes(c[24:32], "little")
    edits = [(ti["model_offset"] + 2, "<H", 1), (dir_off + 72, "<Q", 1), (56, "<Q", 1), (32, "<Q", 208 + 8)]
    for off, fmt, v in edits:
        b = bytearray(c)
        struct.pack_into(fmt, b, off, v)
        with pytest.raises(bs.BsError) as e:
            bs.workspace_bytes(bytes(b))
        assert e.value.code == bs.E_FORMAT
        with pytest.raises(oracle.OracleError):
            oracle.validate(bytes(b))


def test_fw_gemv_refuses_unknown_flags_before_any_launch():
    # argument checks run on the host before any CUDA call, so they work without a GPU
    import lossless_entropy_coding_interleaved_b200 as bs
    item = bs.FwGemvItem()
    err = ctypes.c_uint32(0)
    call = lambda flags: bs.lib.bs_fw_gemv(0, ctypes.byref(item), 1, flags, ctypes.addressof(err), None)
    assert call(2) == bs.E_ARG and call(0x80000000) == bs.E_ARG
    assert bs.lib.bs_fw_gemv(0, ctypes.byref(item), 9, 0, ctypes.addressof(err), None) == bs.E_ARG  # batch 1..8
