"""The oracle: a plain, slow CPU encoder/decoder for the BF16RANS container.

This package is TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it. The GPU library never does, and the
two share no code.

What it computes: the method paragraph of the "Qwen3.8-27B-BF16-NVLC-Lossless" model
card, which splits each BF16 word into sign, exponent and fraction, codes the
sign+exponent symbol with a per-tensor rANS model, and lets that symbol select the
fraction's distribution. The byte layout and every parameter are those of the BF16RANS
(version 2: the fraction's top three bits are coded, its low four bits kept verbatim).
The arithmetic lives in ``bsoracle.c``. This module only marshals arguments through
ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsoracle.c")
_SRCS = (_SRC, os.path.join(_HERE, "fworacle.c"))
_LIB = os.path.join(_HERE, "libbsoracle.so")

OK, E_ARG, E_FORMAT, E_VERSION, E_SIZE, E_CORRUPT, E_NOMEM = 0, 1, 2, 3, 4, 6, 7
KIND_RANS, KIND_STORED, KIND_RAW, KIND_JOINT = 0, 1, 2, 3
_NAMES = {1: "E_ARG", 2: "E_FORMAT", 3: "E_VERSION", 4: "E_SIZE", 6: "E_CORRUPT", 7: "E_NOMEM"}


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what}: status {code} ({_NAMES.get(code, '?')})")
        self.code = code


def build(force: bool = False) -> str:
    """Compile bsoracle.c and fworacle.c into libbsoracle.so next to them (plain gcc, no GPU code)."""
    stale = not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(f) for f in _SRCS)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", *_SRCS, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Item(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_uint32),
        ("ndim", ctypes.c_uint32),
        ("shape", ctypes.c_uint64 * 8),
        ("n_elems", ctypes.c_uint64),
        ("data", ctypes.c_void_p),
        ("name", ctypes.c_char_p),
        ("name_bytes", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
    ]


class _Params(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint32) for k in ("log2_chunk", "ns", "nh", "max_routes", "force_rans", "joint", "nj")]


class _Info(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint32) for k in
                ("kind", "ndim", "log2_chunk", "lanes", "ns", "nh", "n_routes", "name_offset", "name_bytes",
                 "nib_mode")] + \
               [(k, ctypes.c_uint64) for k in
                ("n_elems", "n_chunks", "model_offset", "model_bytes", "data_offset", "data_bytes", "checksum")] + \
               [("shape", ctypes.c_uint64 * 8), ("coded_bytes", ctypes.c_uint64)]


class _FwInfo(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint64) for k in ("n_elems", "n_tiles", "n_exc", "total_bytes")] + \
               [("table", ctypes.c_uint16 * 16)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, u32, u64, i64 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64
        L.bso_encode.argtypes = [ctypes.POINTER(_Item), u32, ctypes.POINTER(_Params), ctypes.POINTER(P),
                                 ctypes.POINTER(u64)]
        L.bso_free.argtypes = [P]
        L.bso_free.restype = None
        L.bso_validate.argtypes = [P, u64, ctypes.POINTER(u32)]
        L.bso_tensor_info_get.argtypes = [P, u64, u32, ctypes.POINTER(_Info)]
        L.bso_decode.argtypes = [P, u64, u32, P, u64, ctypes.POINTER(i64)]
        L.bso_decode_chunks.argtypes = [P, u64, u32, u64, u64, P, u64, ctypes.POINTER(i64)]
        L.bso_quantise.argtypes = [P, u32, u32, P]
        L.bso_choose_routes.argtypes = [P, u32, P, ctypes.POINTER(u32), P]
        L.bso_lane_encode.argtypes = [P, u32, P, P, u32, u32, P, u32, ctypes.POINTER(u32), P, P,
                                      ctypes.POINTER(u32)]
        L.bso_lane_decode.argtypes = [P, u32, P, P, u32, u32, u32, P, u32, P, u32, P, ctypes.POINTER(u32)]
        L.bso_joint_lane_encode.argtypes = [P, u32, P, u32, ctypes.POINTER(u32), P, P, ctypes.POINTER(u32)]
        L.bso_joint_lane_decode.argtypes = [P, u32, u32, P, u32, P, u32, P, ctypes.POINTER(u32)]
        L.bso_fw_bytes.argtypes = [u64, u64]
        L.bso_fw_bytes.restype = u64
        L.bso_fw_table.argtypes = [P, u64, P, ctypes.POINTER(u32)]
        L.bso_fw_encode.argtypes = [P, u64, P, u64, ctypes.POINTER(u64)]
        L.bso_fw_parse.argtypes = [P, u64, ctypes.POINTER(_FwInfo)]
        L.bso_fw_decode.argtypes = [P, u64, P, u64]
        L.bso_mix64.argtypes = [u64]
        L.bso_mix64.restype = u64
        L.bso_checksum.argtypes = [P, u64, u32]
        L.bso_checksum.restype = u64
        for fn in ("bso_encode", "bso_validate", "bso_tensor_info_get", "bso_decode", "bso_decode_chunks",
                   "bso_quantise", "bso_choose_routes", "bso_lane_encode", "bso_lane_decode",
                   "bso_joint_lane_encode", "bso_joint_lane_decode", "bso_fw_table",
                   "bso_fw_encode", "bso_fw_parse", "bso_fw_decode"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data if a.size else 0


def _buf(container) -> tuple[np.ndarray, int]:
    arr = np.frombuffer(container, dtype=np.uint8) if not isinstance(container, np.ndarray) else container
    assert arr.dtype == np.uint8 and arr.flags["C_CONTIGUOUS"]
    return arr, arr.size


def encode(items, log2_chunk: int = 16, ns: int = 11, nh: int = 5, max_routes: int = 15,
           force_rans: bool = False, model: str = "factored", nj: int = 13) -> bytes:
    """items: sequence of (name, array, kind) with kind "bf16" (uint16 words, any shape)
    or "raw" (uint8 bytes). model "factored" codes BF16 tensors as kind RANS (ns, nh, routes),
    "joint" as kind JOINT (one table over (s, h) of precision nj). Returns the container
    bytes (canonical layout: header, directory, names, then each tensor's sections)."""
    assert model in ("factored", "joint")
    keep = []
    arr_items = (_Item * max(1, len(items)))()
    for k, (name, a, kind) in enumerate(items):
        a = np.ascontiguousarray(a)
        if kind == "bf16":
            assert a.dtype == np.uint16
        else:
            assert a.dtype == np.uint8
        nb = name.encode()
        keep += [a, nb]
        it = arr_items[k]
        it.kind = 0 if kind == "bf16" else 2
        shape = a.shape
        it.ndim = len(shape)
        for d, v in enumerate(shape):
            it.shape[d] = v
        it.n_elems = a.size
        it.data = _ptr(a)
        it.name = nb
        it.name_bytes = len(nb)
    p = _Params(log2_chunk, ns, nh, max_routes, 1 if force_rans else 0, 1 if model == "joint" else 0, nj)
    out = ctypes.c_void_p()
    n = ctypes.c_uint64()
    st = lib().bso_encode(arr_items, len(items), ctypes.byref(p), ctypes.byref(out), ctypes.byref(n))
    if st:
        raise OracleError(st, "encode")
    try:
        return ctypes.string_at(out.value, n.value)
    finally:
        lib().bso_free(out)


def validate(container) -> int:
    arr, n = _buf(container)
    nt = ctypes.c_uint32()
    st = lib().bso_validate(_ptr(arr), n, ctypes.byref(nt))
    if st:
        raise OracleError(st, "validate")
    return nt.value


def info(container, idx: int) -> dict:
    arr, n = _buf(container)
    ti = _Info()
    st = lib().bso_tensor_info_get(_ptr(arr), n, idx, ctypes.byref(ti))
    if st:
        raise OracleError(st, "info")
    d = {k: getattr(ti, k) for k, _ in _Info._fields_ if k != "shape"}
    d["shape"] = tuple(ti.shape[i] for i in range(ti.ndim))
    off = int.from_bytes(bytes(arr[32:40]), "little")
    d["name"] = bytes(arr[off + ti.name_offset: off + ti.name_offset + ti.name_bytes]).decode()
    return d


def decode(container, idx: int) -> np.ndarray:
    """Whole tensor: uint16 words (RANS/STORED) or uint8 bytes (RAW)."""
    arr, n = _buf(container)
    ti = info(arr, idx)
    out = np.zeros(ti["n_elems"], dtype=np.uint8 if ti["kind"] == KIND_RAW else np.uint16)
    bad = ctypes.c_int64(-1)
    st = lib().bso_decode(_ptr(arr), n, idx, _ptr(out), out.nbytes, ctypes.byref(bad))
    if st:
        e = OracleError(st, "decode")
        e.bad_chunk = bad.value
        raise e
    return out.reshape(ti["shape"]) if ti["shape"] else out.reshape(())


def decode_chunks(container, idx: int, c0: int, c1: int, out: np.ndarray) -> int:
    """Decode chunks [c0, c1) of a RANS tensor into out (the whole tensor's uint16 array).
    Returns the status (0 or E_CORRUPT...) instead of raising, for fault tests."""
    arr, n = _buf(container)
    bad = ctypes.c_int64(-1)
    st = lib().bso_decode_chunks(_ptr(arr), n, idx, c0, c1, _ptr(out), out.nbytes, ctypes.byref(bad))
    return st


def quantise(counts, M: int) -> np.ndarray:
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    q = np.zeros(c.size, dtype=np.uint32)
    st = lib().bso_quantise(_ptr(c), c.size, M, _ptr(q))
    if st:
        raise OracleError(st, "quantise")
    return q


def choose_routes(ceh, max_routes: int = 15):
    """ceh: 256 x 8 counts of the fraction's top three bits per exponent."""
    c = np.ascontiguousarray(ceh, dtype=np.uint64).reshape(256 * 8)
    route = np.zeros(256, dtype=np.uint8)
    route_e = np.zeros(256, dtype=np.uint32)
    nr = ctypes.c_uint32()
    st = lib().bso_choose_routes(_ptr(c), max_routes, _ptr(route), ctypes.byref(nr), _ptr(route_e))
    if st:
        raise OracleError(st, "choose_routes")
    return route, route_e[: nr.value].copy()


def _tables(Fs, route, Fh):
    Fs = np.ascontiguousarray(Fs, dtype=np.uint32)
    route = np.ascontiguousarray(route, dtype=np.uint8)
    Fh = np.ascontiguousarray(Fh, dtype=np.uint32).reshape(-1)
    assert Fs.size == 512 and route.size == 256 and Fh.size % 8 == 0
    return Fs, route, Fh if Fh.size else np.zeros(8, np.uint32), Fh.size // 8


def lane_encode(Fs, ns, route, Fh, nh, words):
    """One lane of kind RANS: returns (start_state, words, tags). The low
    nibbles of ``words`` do not enter the state; the caller keeps them."""
    Fs, route, Fhb, nr = _tables(Fs, route, Fh)
    w = np.ascontiguousarray(words, dtype=np.uint16)
    S = w.size
    wo = np.zeros(max(S, 1), np.uint16)
    tg = np.zeros(max(S, 1), np.uint32)
    st_out = ctypes.c_uint32()
    nw = ctypes.c_uint32()
    st = lib().bso_lane_encode(_ptr(Fs), ns, _ptr(route), _ptr(Fhb), nr, nh, _ptr(w), S, ctypes.byref(st_out),
                               _ptr(wo), _ptr(tg), ctypes.byref(nw))
    if st:
        raise OracleError(st, "lane_encode")
    return st_out.value, wo[: nw.value].copy(), tg[: nw.value].copy()


def lane_decode(Fs, ns, route, Fh, nh, state, words, nibbles, S):
    """Returns (status, decoded words, final state). ``nibbles[t]`` is weight t's low nibble."""
    Fs, route, Fhb, nr = _tables(Fs, route, Fh)
    wd = np.ascontiguousarray(words, dtype=np.uint16)
    nb = np.ascontiguousarray(nibbles, dtype=np.uint8)
    assert nb.size >= S
    if nb.size == 0:
        nb = np.zeros(1, np.uint8)
    out = np.zeros(max(S, 1), np.uint16)
    fin = ctypes.c_uint32()
    st = lib().bso_lane_decode(_ptr(Fs), ns, _ptr(route), _ptr(Fhb), nr, nh, state, _ptr(wd), wd.size, _ptr(nb), S,
                               _ptr(out), ctypes.byref(fin))
    return st, out[:S].copy(), fin.value


def joint_lane_encode(Fj, nj, words):
    """One lane of the JOINT kind: returns (start_state, words, tags) for the pair table
    Fj[4096] of precision nj. The low nibbles of ``words`` do not enter the state."""
    Fj = np.ascontiguousarray(Fj, dtype=np.uint32)
    assert Fj.size == 4096
    w = np.ascontiguousarray(words, dtype=np.uint16)
    S = w.size
    wo = np.zeros(max(S, 1), np.uint16)
    tg = np.zeros(max(S, 1), np.uint32)
    st_out = ctypes.c_uint32()
    nw = ctypes.c_uint32()
    st = lib().bso_joint_lane_encode(_ptr(Fj), nj, _ptr(w), S, ctypes.byref(st_out), _ptr(wo), _ptr(tg),
                                     ctypes.byref(nw))
    if st:
        raise OracleError(st, "joint_lane_encode")
    return st_out.value, wo[: nw.value].copy(), tg[: nw.value].copy()


def joint_lane_decode(Fj, nj, state, words, nibbles, S):
    """Returns (status, decoded words, final state) of one JOINT lane."""
    Fj = np.ascontiguousarray(Fj, dtype=np.uint32)
    assert Fj.size == 4096
    wd = np.ascontiguousarray(words, dtype=np.uint16)
    nb = np.ascontiguousarray(nibbles, dtype=np.uint8)
    assert nb.size >= S
    if nb.size == 0:
        nb = np.zeros(1, np.uint8)
    out = np.zeros(max(S, 1), np.uint16)
    fin = ctypes.c_uint32()
    st = lib().bso_joint_lane_decode(_ptr(Fj), nj, state, _ptr(wd), wd.size, _ptr(nb), S, _ptr(out),
                                     ctypes.byref(fin))
    return st, out[:S].copy(), fin.value


def mix64(v: int) -> int:
    return int(lib().bso_mix64(v))


def checksum(a: np.ndarray) -> int:
    """The per-tensor checksum, sum of splitmix64 outputs over (i << 16) | w[i] (uint16 words) or
    (i << 8) | b[i] (uint8 bytes), mod 2^64."""
    a = np.ascontiguousarray(a).reshape(-1)
    return int(lib().bso_checksum(_ptr(a), a.size, 2 if a.dtype == np.uint8 else 0))


# ------------------------------------------------------------ fixed-width lane layout
# The fixed-width lane layout; the arithmetic is in fworacle.c.
def fw_bytes(n_elems: int, n_exc: int) -> int:
    """Size of the FW layout of n_elems weights with n_exc escapes."""
    return int(lib().bso_fw_bytes(n_elems, n_exc))


def fw_table(words) -> tuple[list[int], int]:
    """(code table of 16 entries, number of codes used) for uint16 words."""
    w = np.ascontiguousarray(words, dtype=np.uint16).reshape(-1)
    t = np.zeros(16, np.uint16)
    k = ctypes.c_uint32()
    st = lib().bso_fw_table(_ptr(w), w.size, _ptr(t), ctypes.byref(k))
    if st:
        raise OracleError(st, "fw_table")
    return [int(v) for v in t], k.value


def fw_encode(words) -> bytes:
    """The FW layout of uint16 words (any shape, flattened)."""
    w = np.ascontiguousarray(words, dtype=np.uint16).reshape(-1)
    size = ctypes.c_uint64()
    st = lib().bso_fw_encode(_ptr(w), w.size, None, 0, ctypes.byref(size))
    if st:
        raise OracleError(st, "fw_encode")
    out = np.zeros(max(size.value, 1), np.uint8)
    st = lib().bso_fw_encode(_ptr(w), w.size, _ptr(out), out.size, ctypes.byref(size))
    if st:
        raise OracleError(st, "fw_encode")
    return out[: size.value].tobytes()


def fw_info(blob) -> dict:
    """Header fields of an FW layout (validated against its size)."""
    arr, n = _buf(blob)
    info = _FwInfo()
    st = lib().bso_fw_parse(_ptr(arr), n, ctypes.byref(info))
    if st:
        raise OracleError(st, "fw_parse")
    return {"n_elems": info.n_elems, "n_tiles": info.n_tiles, "n_exc": info.n_exc,
            "total_bytes": info.total_bytes, "table": [int(v) for v in info.table]}


def fw_decode(blob) -> np.ndarray:
    """Decode an FW layout into uint16 words; raises OracleError on a malformed one."""
    arr, n = _buf(blob)
    info = _FwInfo()
    st = lib().bso_fw_parse(_ptr(arr), n, ctypes.byref(info))
    if st:
        raise OracleError(st, "fw_parse")
    out = np.zeros(max(info.n_elems, 1), np.uint16)
    st = lib().bso_fw_decode(_ptr(arr), n, _ptr(out), info.n_elems)
    if st:
        raise OracleError(st, "fw_decode")
    return out[: info.n_elems].copy()


def fw_gemv(blob, rows: int, cols: int, x) -> np.ndarray:
    """y = W x in float64, with W (rows x cols, row-major) decoded from an FW layout and x
    BF16 words [batch, cols] (or [cols]). The weights and x are exact in float64; the product
    is numpy's matmul. Returns [batch, rows] (or [rows])."""
    w = fw_decode(blob).reshape(rows, cols)
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    xa = np.ascontiguousarray(x, dtype=np.uint16)
    xf = (xa.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return xf @ wf.T
