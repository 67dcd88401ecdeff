"""Python binding of libbs, the sm_100a decoder for BF16RANS containers.

The binding only marshals arguments. Every step of the decode runs in libbs's CUDA
kernels (csrc/bs_kernels.cu), and its host planner is csrc/bs_plan.cpp. PyTorch
supplies device memory and streams. There is no CPU fallback: importing this module
without a built libbs.so raises, and so does planning without a CUDA device.

The method is the one in the paragraph after the accounting table of the
"Qwen3.8-27B-BF16-NVLC-Lossless" model card:
  - each BF16 word is split into sign, exponent and fraction;
  - the sign+exponent symbol is rANS-decoded with a per-tensor model;
  - that symbol selects the 7-bit fraction's distribution;
  - the fields are recombined bitwise.
The byte layout is the BF16RANS container, version 2.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbs.so")

OK, E_ARG, E_FORMAT, E_VERSION, E_SIZE, E_CUDA, E_CORRUPT, E_NOMEM, E_UNSUPPORTED = range(9)
FW_LAYOUTS_RESIDENT = 1  # bs_fw_gemv flag: no work in flight writes the layouts
KIND_RANS, KIND_STORED, KIND_RAW, KIND_JOINT = 0, 1, 2, 3


class BsError(RuntimeError):
    def __init__(self, code: int, what: str, msg: str = "", first_bad: int = -1):
        super().__init__(f"libbs {what}: {msg or code} (status {code})")
        self.code = code
        self.first_bad = first_bad


class _Range(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_int32), ("reserved", ctypes.c_uint32), ("begin", ctypes.c_uint64),
                ("count", ctypes.c_uint64), ("d_out", ctypes.c_void_p), ("out_bytes", ctypes.c_size_t)]


class _Info(ctypes.Structure):
    _fields_ = [("n_elems", ctypes.c_uint64), ("out_bytes", ctypes.c_uint64), ("coded_bytes", ctypes.c_uint64),
                ("n_chunks", ctypes.c_uint64), ("checksum", ctypes.c_uint64), ("shape", ctypes.c_uint64 * 8),
                ("kind", ctypes.c_uint32), ("ndim", ctypes.c_uint32), ("ns", ctypes.c_uint32),
                ("nh", ctypes.c_uint32), ("n_routes", ctypes.c_uint32), ("log2_chunk", ctypes.c_uint32),
                ("name", ctypes.c_void_p), ("name_bytes", ctypes.c_uint32), ("nib_mode", ctypes.c_uint32)]


class _EncItem(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_uint32), ("ndim", ctypes.c_uint32), ("shape", ctypes.c_uint64 * 8),
                ("n_elems", ctypes.c_uint64), ("d_data", ctypes.c_void_p), ("name", ctypes.c_char_p),
                ("name_bytes", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class _StreamStats(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint64) for k in ("loads", "hits", "evictions", "h2d_bytes", "decoded_bytes",
                                                "resident_groups", "cache_bytes", "cache_bytes_used",
                                                "stage_bytes")]


class _EncParams(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint32) for k in ("log2_chunk", "ns", "nh", "max_routes", "force_rans", "model", "nj")]


class FwInfo(ctypes.Structure):
    """bs_fw_info: the header of a fixed-width lane layout (4-bit codes, 7-bit fractions, exceptions)."""
    _fields_ = [("n_elems", ctypes.c_uint64), ("n_tiles", ctypes.c_uint64), ("n_exc", ctypes.c_uint64),
                ("total_bytes", ctypes.c_uint64), ("table", ctypes.c_uint16 * 16)]

    def __repr__(self):
        return (f"FwInfo(n_elems={self.n_elems}, n_tiles={self.n_tiles}, n_exc={self.n_exc}, "
                f"total_bytes={self.total_bytes}, table={list(self.table)})")


class FwGemvItem(ctypes.Structure):
    """bs_fw_gemv_item: one product y = W x (W in the FW layout)."""
    _fields_ = [("d_fw", ctypes.c_void_p), ("info", FwInfo), ("rows", ctypes.c_uint32), ("cols", ctypes.c_uint32),
                ("d_x", ctypes.c_void_p), ("d_y", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbs.so is not built ({LIB_PATH}); run "
                          f"`python lossless_entropy_coding_interleaved_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
    L.bs_plan_workspace_bytes.argtypes = [P, sz]
    L.bs_plan_workspace_bytes.restype = sz
    L.bs_plan.argtypes = [P, sz, P, P, sz, P, ctypes.POINTER(P)]
    L.bs_plan_destroy.argtypes = [P]
    L.bs_plan_destroy.restype = None
    L.bs_tensor_count.argtypes = [P, ctypes.POINTER(i32)]
    L.bs_tensor_info_get.argtypes = [P, i32, ctypes.POINTER(_Info)]
    L.bs_decode_tensor.argtypes = [P, i32, P, sz, P]
    L.bs_decode_batch.argtypes = [P, P, P, P, i32, P]
    L.bs_decode_ranges.argtypes = [P, ctypes.POINTER(_Range), i32, P]
    L.bs_decode_geometry.argtypes = [P, i32, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
    L.bs_verify_tensor.argtypes = [P, i32, P, sz, P, P, ctypes.POINTER(u64)]
    L.bs_check.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    L.bs_status_str.argtypes = [ctypes.c_int]
    L.bs_status_str.restype = ctypes.c_char_p
    L.bs_last_cuda_error.argtypes = []
    L.bs_decode_tensor_noalloc.argtypes = [P, sz, P, i32, P, sz, P]
    L.bs_decode_tensor_noalloc.restype = ctypes.c_int
    L.bs_launch_counter.argtypes = []
    L.bs_launch_counter.restype = u64
    L.bs_plan_workspace_bytes_device.argtypes = [P, sz, P]
    L.bs_plan_workspace_bytes_device.restype = sz
    L.bs_encoder_create.argtypes = [ctypes.POINTER(_EncItem), i32, ctypes.POINTER(_EncParams), ctypes.POINTER(P)]
    L.bs_encoder_scratch_bytes.argtypes = [P, ctypes.POINTER(sz)]
    L.bs_encoder_run.argtypes = [P, P, sz, P, ctypes.POINTER(sz)]
    L.bs_encoder_emit.argtypes = [P, P, P, sz, P, P]
    L.bs_encoder_destroy.argtypes = [P]
    L.bs_encoder_destroy.restype = None
    L.bs_streamer_workspace_bytes.argtypes = [P, sz]
    L.bs_streamer_workspace_bytes.restype = sz
    L.bs_streamer_min_arena_bytes.argtypes = [P, sz, P]
    L.bs_streamer_min_arena_bytes.restype = sz
    L.bs_streamer_create.argtypes = [P, sz, P, P, sz, P, sz, P, ctypes.POINTER(P)]
    L.bs_streamer_group_count.argtypes = [P, ctypes.POINTER(i32)]
    L.bs_streamer_tensor_info_get.argtypes = [P, i32, ctypes.POINTER(_Info)]
    L.bs_streamer_prefetch.argtypes = [P, i32, P]
    L.bs_streamer_acquire.argtypes = [P, i32, P, i32, P]
    L.bs_streamer_release.argtypes = [P, i32, P]
    L.bs_streamer_get_stats.argtypes = [P, ctypes.POINTER(_StreamStats)]
    L.bs_streamer_check.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    L.bs_streamer_destroy.argtypes = [P]
    L.bs_streamer_destroy.restype = None
    L.bs_fw_scratch_bytes.argtypes = [u64]
    L.bs_fw_scratch_bytes.restype = sz
    L.bs_fw_measure.argtypes = [P, u64, P, sz, P, ctypes.POINTER(FwInfo)]
    L.bs_fw_write.argtypes = [P, u64, P, sz, ctypes.POINTER(FwInfo), P, sz, P]
    L.bs_fw_parse.argtypes = [P, sz, sz, ctypes.POINTER(FwInfo)]
    L.bs_fw_decode.argtypes = [i32, P, P, P, P, P, P]
    L.bs_fw_gemv.argtypes = [i32, ctypes.POINTER(FwGemvItem), ctypes.c_uint32, ctypes.c_uint32, P, P]
    L.bs_fw_gemm.argtypes = [i32, ctypes.POINTER(FwGemvItem), ctypes.c_uint32, P, P]
    for fn in ("bs_fw_measure", "bs_fw_write", "bs_fw_parse", "bs_fw_decode", "bs_fw_gemv", "bs_fw_gemm"):
        getattr(L, fn).restype = ctypes.c_int
    for fn in ("bs_streamer_create", "bs_streamer_group_count", "bs_streamer_tensor_info_get", "bs_streamer_prefetch", "bs_streamer_acquire",
               "bs_streamer_release", "bs_streamer_get_stats", "bs_streamer_check"):
        getattr(L, fn).restype = ctypes.c_int
    for fn in ("bs_plan", "bs_tensor_count", "bs_tensor_info_get", "bs_decode_tensor", "bs_decode_batch",
               "bs_decode_ranges", "bs_decode_geometry", "bs_verify_tensor", "bs_check", "bs_last_cuda_error", "bs_encoder_create", "bs_encoder_scratch_bytes",
               "bs_encoder_run", "bs_encoder_emit"):
        getattr(L, fn).restype = ctypes.c_int
    return L


lib = _load()

#: every symbol include/bs.h declares
EXPORTS = ("bs_plan_workspace_bytes", "bs_plan_workspace_bytes_device", "bs_plan", "bs_plan_destroy",
           "bs_tensor_count", "bs_tensor_info_get", "bs_decode_tensor", "bs_decode_batch", "bs_decode_ranges",
           "bs_decode_geometry",
           "bs_verify_tensor",
           "bs_check", "bs_encoder_create", "bs_encoder_scratch_bytes", "bs_encoder_run", "bs_encoder_emit",
           "bs_encoder_destroy", "bs_status_str", "bs_last_cuda_error", "bs_launch_counter",
           "bs_decode_tensor_noalloc", "bs_streamer_workspace_bytes", "bs_streamer_min_arena_bytes",
           "bs_streamer_create", "bs_streamer_group_count", "bs_streamer_tensor_info_get", "bs_streamer_prefetch",
           "bs_streamer_acquire",
           "bs_streamer_release", "bs_streamer_get_stats", "bs_streamer_check", "bs_streamer_destroy",
           "bs_fw_scratch_bytes", "bs_fw_measure", "bs_fw_write", "bs_fw_parse", "bs_fw_decode", "bs_fw_gemv",
           "bs_fw_gemm")


def decode_noalloc(container, d_container: torch.Tensor, idx: int, out: torch.Tensor, stream=None) -> torch.Tensor:
    """bs_decode_tensor_noalloc: decode tensor idx into out using libbs's static device
    array instead of a workspace. For callers that cannot allocate device memory. It
    synchronises the stream, and calls that overlap on the GPU race on the shared array."""
    h = _host_bytes(container)
    _check(lib.bs_decode_tensor_noalloc(h.ctypes.data, h.size, d_container.data_ptr(), idx, out.data_ptr(),
                                        out.numel() * out.element_size(), _stream(stream)), "decode_tensor_noalloc")
    return out


def launch_counter() -> int:
    """Kernel launches libbs has made in this process."""
    return int(lib.bs_launch_counter())


def _check(st: int, what: str):
    if st != OK:
        msg = lib.bs_status_str(st).decode()
        if st == E_CUDA:
            msg += f" (cudaError {lib.bs_last_cuda_error()})"
        raise BsError(st, what, msg)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _host_bytes(container) -> np.ndarray:
    if isinstance(container, np.ndarray):
        a = np.ascontiguousarray(container.reshape(-1).view(np.uint8))
    else:
        a = np.frombuffer(container, dtype=np.uint8)
    return a


def _info_dict(ti: _Info) -> dict:
    d = {k: getattr(ti, k) for k, _ in _Info._fields_ if k not in ("shape", "name", "name_bytes")}
    d["shape"] = tuple(ti.shape[i] for i in range(ti.ndim))
    d["name"] = ctypes.string_at(ti.name, ti.name_bytes).decode() if ti.name_bytes else ""
    return d


def _container_names(h: np.ndarray) -> list:
    """Tensor names in directory order, read from a container that already passed
    validation (header: n_tensors at byte 16, dir_offset at 24, names_offset at 32; directory:
    144-byte entries with name_offset at 8 and name_bytes at 12)."""
    hdr = h[:64].tobytes()
    nt = int.from_bytes(hdr[16:20], "little")
    d0, n0 = int.from_bytes(hdr[24:32], "little"), int.from_bytes(hdr[32:40], "little")
    names = []
    for k in range(nt):
        e = h[d0 + 144 * k: d0 + 144 * k + 16].tobytes()
        off, nb = int.from_bytes(e[8:12], "little"), int.from_bytes(e[12:16], "little")
        names.append(h[n0 + off: n0 + off + nb].tobytes().decode())
    return names


def workspace_bytes(container) -> int:
    h = _host_bytes(container)
    n = lib.bs_plan_workspace_bytes(h.ctypes.data, h.size)
    if n == 0:
        raise BsError(E_FORMAT, "workspace_bytes", "container fails validation")
    return n


def encode(tensors, log2_chunk: int = 16, ns: int = 11, nh: int = 5, max_routes: int = 15,
           force_rans: bool = False, host_copy: bool = False, stream=None, model: str = "factored", nj: int = 13):
    """Encode device tensors into a container on the device (bs_encoder_*).

    tensors: sequence of (name, tensor) pairs; int16/bfloat16 CUDA tensors are BF16
    words and uint8 CUDA tensors are opaque byte spans. model "factored" codes BF16 tensors
    as kind RANS (ns, nh, routes), "joint" as kind JOINT (one table of precision nj; faster
    to decode). Returns (d_container, h_container),
    a uint8 CUDA tensor and, when host_copy, a uint8 numpy copy (else None).
    """
    keep = []
    items = (_EncItem * max(1, len(tensors)))()
    dev = None
    for k, (name, t) in enumerate(tensors):
        assert t.is_cuda and t.is_contiguous()
        dev = t.device
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        assert t.dtype in (torch.int16, torch.uint8), t.dtype
        nb = name.encode()
        keep += [t, nb]
        it = items[k]
        it.kind = 0 if t.dtype == torch.int16 else 2
        it.ndim = t.dim()
        for d, v in enumerate(t.shape):
            it.shape[d] = v
        it.n_elems = t.numel()
        it.d_data = t.data_ptr() if t.numel() else None
        it.name = nb
        it.name_bytes = len(nb)
    if dev is None:
        dev = torch.device("cuda")
    assert model in ("factored", "joint")
    prm = _EncParams(log2_chunk, ns, nh, max_routes, 1 if force_rans else 0, 1 if model == "joint" else 0, nj)
    enc = ctypes.c_void_p()
    _check(lib.bs_encoder_create(items, len(tensors), ctypes.byref(prm), ctypes.byref(enc)), "encoder_create")
    try:
        sc = ctypes.c_size_t()
        _check(lib.bs_encoder_scratch_bytes(enc, ctypes.byref(sc)), "encoder_scratch_bytes")
        scratch = torch.empty(max(sc.value, 256), dtype=torch.uint8, device=dev)
        total = ctypes.c_size_t()
        st = _stream(stream)
        with torch.cuda.device(dev):
            _check(lib.bs_encoder_run(enc, scratch.data_ptr(), scratch.numel(), st, ctypes.byref(total)),
                   "encoder_run")
            d_container = torch.empty(total.value, dtype=torch.uint8, device=dev)
            h = np.empty(total.value, dtype=np.uint8) if host_copy else None
            _check(lib.bs_encoder_emit(enc, scratch.data_ptr(), d_container.data_ptr(), total.value,
                                       h.ctypes.data if host_copy else None, st), "encoder_emit")
    finally:
        lib.bs_encoder_destroy(enc)
    return d_container, h


class Plan:
    """A validated container resident in device memory, with its decode tables.

    ``container`` holds the container's bytes on the host (bytes or a uint8 numpy
    array), or is None when ``d_container`` is given: the plan then reads the metadata
    from the device. ``d_container`` is an optional uint8 CUDA tensor that already holds
    the container; without it, the host bytes are copied to ``device``.
    """

    def __init__(self, container=None, device="cuda", d_container: torch.Tensor | None = None, stream=None):
        if not torch.cuda.is_available():
            raise BsError(E_UNSUPPORTED, "plan", "no CUDA device")
        if container is None and d_container is None:
            raise BsError(E_ARG, "plan", "no container")
        self.device = torch.device(device) if d_container is None else d_container.device
        h = None if container is None else _host_bytes(container)
        if d_container is None:
            d_container = torch.from_numpy(h.copy()).to(self.device)
        assert d_container.dtype == torch.uint8 and d_container.is_cuda
        assert h is None or d_container.numel() == h.size
        self.d_container = d_container
        self.container_bytes = d_container.numel()
        st = _stream(stream)
        with torch.cuda.device(self.device):
            if h is not None:
                ws = workspace_bytes(h)
            else:
                ws = lib.bs_plan_workspace_bytes_device(d_container.data_ptr(), d_container.numel(), st)
                if ws == 0:
                    raise BsError(E_FORMAT, "workspace_bytes", "container fails validation")
            self.workspace = torch.empty(ws, dtype=torch.uint8, device=self.device)
            self._scratch = torch.zeros(2, dtype=torch.int64, device=self.device)
            ptr = ctypes.c_void_p()
            _check(lib.bs_plan(None if h is None else h.ctypes.data, self.container_bytes, d_container.data_ptr(),
                               self.workspace.data_ptr(), ws, st, ctypes.byref(ptr)), "plan")
        self._p = ptr
        n = ctypes.c_int32()
        _check(lib.bs_tensor_count(self._p, ctypes.byref(n)), "tensor_count")
        self.n_tensors = n.value
        self._info = [self._get_info(k) for k in range(self.n_tensors)]
        self.names = [i["name"] for i in self._info]

    def __del__(self):
        p = getattr(self, "_p", None)
        if p and lib is not None:
            lib.bs_plan_destroy(p)
            self._p = None

    def _get_info(self, idx: int) -> dict:
        ti = _Info()
        _check(lib.bs_tensor_info_get(self._p, idx, ctypes.byref(ti)), "tensor_info")
        return _info_dict(ti)

    def info(self, idx: int) -> dict:
        return dict(self._info[idx])

    def empty_output(self, idx: int) -> torch.Tensor:
        """A device buffer of the right size and dtype for tensor idx: int16 words viewable
        as bfloat16, or uint8 for RAW."""
        i = self._info[idx]
        if i["kind"] == KIND_RAW:
            return torch.empty(i["n_elems"], dtype=torch.uint8, device=self.device)
        return torch.empty(i["shape"] if i["shape"] else (), dtype=torch.int16, device=self.device)

    def decode(self, idx: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if out is None:
            out = self.empty_output(idx)
        _check(lib.bs_decode_tensor(self._p, idx, out.data_ptr(), out.numel() * out.element_size(),
                                    _stream(stream)), "decode_tensor")
        return out

    def decode_batch(self, idxs, outs=None, stream=None):
        idxs = list(idxs)
        if outs is None:
            outs = [self.empty_output(k) for k in idxs]
        n = len(idxs)
        ia = (ctypes.c_int32 * max(n, 1))(*idxs)
        pa = (ctypes.c_void_p * max(n, 1))(*[o.data_ptr() for o in outs])
        ba = (ctypes.c_size_t * max(n, 1))(*[o.numel() * o.element_size() for o in outs])
        _check(lib.bs_decode_batch(self._p, ia, pa, ba, n, _stream(stream)), "decode_batch")
        return outs

    def decode_ranges(self, ranges, stream=None):
        """bs_decode_ranges: ranges is a sequence of (idx, begin, count, out). Elements
        [begin, begin + count) of tensor idx (bytes for RAW) are decoded into out; for coded
        kinds the range covers whole chunks (it may end at the tensor's end)."""
        ranges = list(ranges)
        n = len(ranges)
        ra = (_Range * max(n, 1))()
        for k, (idx, begin, count, out) in enumerate(ranges):
            ra[k].idx, ra[k].reserved, ra[k].begin, ra[k].count = idx, 0, begin, count
            ra[k].d_out = out.data_ptr() if out.numel() else None
            ra[k].out_bytes = out.numel() * out.element_size()
        _check(lib.bs_decode_ranges(self._p, ra, n, _stream(stream)), "decode_ranges")
        return [r[3] for r in ranges]

    def decode_geometry(self, idx: int):
        """bs_decode_geometry: (chunks one CTA of tensor idx's decode takes, CTAs per wave)."""
        cpc, wave = ctypes.c_uint32(), ctypes.c_uint32()
        _check(lib.bs_decode_geometry(self._p, idx, ctypes.byref(cpc), ctypes.byref(wave)), "decode_geometry")
        return cpc.value, wave.value

    def to_fw(self, idx: int, scratch: torch.Tensor | None = None, stream=None):
        """The fixed-width lane layout of BF16 tensor idx, built on the
        device from the container, as the runtime of the NVLC card derives its streams from
        the rANS files at start-up. The tensor is decoded (bs_decode_tensor) into `scratch`
        (or a temporary), checked (bs_check), then transcoded (bs_fw_measure, bs_fw_write).
        Returns (layout, FwInfo). Synchronises the stream."""
        i = self._info[idx]
        if i["kind"] == KIND_RAW:
            raise BsError(E_ARG, "to_fw", "a RAW tensor has no BF16 words")
        n = i["n_elems"]
        if scratch is None or scratch.numel() < n:
            scratch = torch.empty(max(n, 1), dtype=torch.int16, device=self.device)
        words = scratch.view(-1)[:n]
        self.decode(idx, words, stream=stream)
        self.check(stream=stream)
        return fw_transcode(words, stream=stream)

    def verify(self, idx: int, out: torch.Tensor, stream=None) -> int:
        """Checksum of a decoded tensor computed on the device; raises BsError(E_CORRUPT)
        if it differs from the stored one. Synchronises the stream."""
        got = ctypes.c_uint64()
        st = lib.bs_verify_tensor(self._p, idx, out.data_ptr(), out.numel() * out.element_size(),
                                  self._scratch.data_ptr(), _stream(stream), ctypes.byref(got))
        _check(st, "verify_tensor")
        return got.value

    def check(self, stream=None) -> int:
        """Synchronise and read the device error word: -1 if clean, else raises BsError with
        first_bad = (tensor << 40) | chunk."""
        fb = ctypes.c_int64()
        st = lib.bs_check(self._p, _stream(stream), ctypes.byref(fb))
        if st == E_CORRUPT:
            raise BsError(st, "check", "corrupt chunk", first_bad=fb.value)
        _check(st, "check")
        return fb.value


def _group_list(groups, names) -> list:
    if callable(groups):
        keys = {}
        groups = [keys.setdefault(groups(n), len(keys)) for n in names]
    groups = [int(g) for g in groups]
    if len(groups) != len(names):
        raise BsError(E_ARG, "streamer", "one group number per tensor")
    return groups


def streamer_min_arena_bytes(container, groups) -> int:
    """bs_streamer_min_arena_bytes: the smallest device budget for this grouping (two
    staging slots plus the largest decoded group)."""
    h = container.numpy() if isinstance(container, torch.Tensor) else _host_bytes(container)
    if lib.bs_streamer_workspace_bytes(h.ctypes.data, h.size) == 0:
        raise BsError(E_FORMAT, "streamer", "container fails validation")
    g = _group_list(groups, _container_names(h))
    ga = (ctypes.c_int32 * max(1, len(g)))(*g)
    n = lib.bs_streamer_min_arena_bytes(h.ctypes.data, h.size, ga)
    if n == 0:
        raise BsError(E_ARG, "streamer", "invalid grouping")
    return n


class Streamer:
    """Layer streaming (bs_streamer_*): decode groups of tensors on demand from a container
    in host memory into a device cache of ``arena_bytes`` with least-recently-used eviction.

    ``groups`` gives each tensor's group number in directory order: a list of ints, or a
    callable name -> hashable key, whose distinct keys are numbered in order of first use.
    The host bytes are copied once into page-locked memory, so the host-to-device copies
    can overlap other work; a page-locked uint8 CPU tensor is used in place instead. ``arena_bytes`` is the whole device budget: two staging slots
    plus the cache (at least ``min_arena_bytes``).
    """

    def __init__(self, container, groups, arena_bytes: int | None = None, device="cuda", stream=None):
        if not torch.cuda.is_available():
            raise BsError(E_UNSUPPORTED, "streamer", "no CUDA device")
        self.device = torch.device(device)
        if isinstance(container, torch.Tensor) and container.dtype == torch.uint8 and container.is_pinned():
            self.host = container.reshape(-1)          # used in place: it must stay unchanged
        else:
            h = _host_bytes(container)
            self.host = torch.empty(h.size, dtype=torch.uint8, pin_memory=True)
            self.host.numpy()[:] = h
        hp, hn = self.host.data_ptr(), self.host.numel()
        ws = lib.bs_streamer_workspace_bytes(hp, hn)
        if ws == 0:
            raise BsError(E_FORMAT, "streamer", "container fails validation")
        self.names = _container_names(self.host.numpy())
        groups = _group_list(groups, self.names)
        self._groups = (ctypes.c_int32 * max(1, len(groups)))(*groups)
        self.min_arena_bytes = lib.bs_streamer_min_arena_bytes(hp, hn, self._groups)
        if self.min_arena_bytes == 0:
            raise BsError(E_ARG, "streamer", "invalid grouping")
        if arena_bytes is None:
            arena_bytes = self.min_arena_bytes
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(ws, dtype=torch.uint8, device=self.device)
            self.arena = torch.empty(arena_bytes, dtype=torch.uint8, device=self.device)
            ptr = ctypes.c_void_p()
            _check(lib.bs_streamer_create(hp, hn, self._groups, self.workspace.data_ptr(), ws,
                                          self.arena.data_ptr(), arena_bytes, _stream(stream), ctypes.byref(ptr)),
                   "streamer_create")
        self._s = ptr
        n = ctypes.c_int32()
        _check(lib.bs_streamer_group_count(self._s, ctypes.byref(n)), "streamer_group_count")
        self.n_groups = n.value
        self.members = [[k for k, g in enumerate(groups) if g == j] for j in range(self.n_groups)]
        self._info = []
        for k in range(len(self.names)):
            ti = _Info()
            _check(lib.bs_streamer_tensor_info_get(self._s, k, ctypes.byref(ti)), "streamer_tensor_info")
            self._info.append(_info_dict(ti))

    def info(self, idx: int) -> dict:
        return dict(self._info[idx])

    def __del__(self):
        s = getattr(self, "_s", None)
        if s and lib is not None:
            torch.cuda.synchronize(self.device)
            lib.bs_streamer_destroy(s)
            self._s = None

    def prefetch(self, group: int, stream=None):
        _check(lib.bs_streamer_prefetch(self._s, group, _stream(stream)), "streamer_prefetch")

    def acquire(self, group: int, stream=None) -> list:
        """Pin the group and return its tensors as views into the arena (int16 words shaped
        like the originals, uint8 for RAW), valid until release."""
        m = self.members[group] if 0 <= group < self.n_groups else []
        ptrs = (ctypes.c_void_p * max(1, len(m)))()
        _check(lib.bs_streamer_acquire(self._s, group, ptrs, len(m), _stream(stream)), "streamer_acquire")
        base = self.arena.data_ptr()
        out = []
        for k, p in zip(m, ptrs):
            i = self._info[k]
            off = (p or base) - base
            if i["kind"] == KIND_RAW:
                out.append(self.arena[off:off + i["n_elems"]])
            else:
                v = self.arena[off:off + 2 * i["n_elems"]].view(torch.int16)
                out.append(v.view(i["shape"]) if i["shape"] else v.view(()))
        return out

    def release(self, group: int, stream=None):
        _check(lib.bs_streamer_release(self._s, group, _stream(stream)), "streamer_release")

    def stats(self) -> dict:
        st = _StreamStats()
        _check(lib.bs_streamer_get_stats(self._s, ctypes.byref(st)), "streamer_stats")
        return {k: getattr(st, k) for k, _ in _StreamStats._fields_}

    def check(self, stream=None) -> int:
        fb = ctypes.c_int64()
        st = lib.bs_streamer_check(self._s, _stream(stream), ctypes.byref(fb))
        if st == E_CORRUPT:
            raise BsError(st, "streamer_check", "corrupt chunk", first_bad=fb.value)
        _check(st, "streamer_check")
        return fb.value


# ------------------------------------------------------------ fixed-width lane layout
def _words(t: torch.Tensor) -> torch.Tensor:
    assert t.is_cuda and t.is_contiguous() and t.element_size() == 2, "BF16 words: a contiguous 2-byte CUDA tensor"
    return t


def fw_scratch_bytes(n_elems: int) -> int:
    return int(lib.bs_fw_scratch_bytes(n_elems))


def fw_transcode(words: torch.Tensor, stream=None) -> tuple[torch.Tensor, FwInfo]:
    """Build the fixed-width lane layout of BF16 words on their device (bs_fw_measure, then
    bs_fw_write). Returns (layout as a uint8 CUDA tensor, its FwInfo). Synchronises the stream."""
    w = _words(words)
    n = w.numel()
    scratch = torch.empty(max(fw_scratch_bytes(n), 256), dtype=torch.uint8, device=w.device)
    info = FwInfo()
    st = _stream(stream)
    with torch.cuda.device(w.device):
        _check(lib.bs_fw_measure(w.data_ptr() if n else None, n, scratch.data_ptr(), scratch.numel(), st,
                                 ctypes.byref(info)), "fw_measure")
        fw = torch.empty(info.total_bytes, dtype=torch.uint8, device=w.device)
        _check(lib.bs_fw_write(w.data_ptr() if n else None, n, scratch.data_ptr(), scratch.numel(),
                               ctypes.byref(info), fw.data_ptr(), fw.numel(), st), "fw_write")
    return fw, info


def fw_parse(head, fw_bytes: int) -> FwInfo:
    """bs_fw_parse of a host copy of a layout's first 96 bytes (or more)."""
    h = _host_bytes(head)
    info = FwInfo()
    _check(lib.bs_fw_parse(h.ctypes.data, h.size, fw_bytes, ctypes.byref(info)), "fw_parse")
    return info


def fw_decode(fws, infos, outs, err: torch.Tensor, stream=None):
    """bs_fw_decode: decode layouts fws[k] (uint8 CUDA tensors, headers infos[k]) into outs[k]
    (2-byte CUDA tensors of n_elems). err: a zeroed int32 CUDA tensor of one element that
    receives the error flags. Enqueued on the stream."""
    n = len(fws)
    assert len(infos) == n and len(outs) == n
    P = ctypes.c_void_p
    p_fw = (P * max(n, 1))(*[f.data_ptr() for f in fws])
    p_out = (P * max(n, 1))(*[_words(o).data_ptr() if o.numel() else None for o in outs])
    sizes = (ctypes.c_size_t * max(n, 1))(*[o.numel() * 2 for o in outs])
    inf = (FwInfo * max(n, 1))(*infos)
    assert err.is_cuda and err.dtype == torch.int32 and err.numel() >= 1
    with torch.cuda.device(err.device):
        _check(lib.bs_fw_decode(n, p_fw, inf, p_out, sizes, err.data_ptr(), _stream(stream)), "fw_decode")
    return outs


def _fw_products(products, max_batch):
    n = len(products)
    arr = (FwGemvItem * max(n, 1))()
    batch = None
    for k, (fw, info, rows, cols, x, y) in enumerate(products):
        b = 1 if x.dim() == 1 else x.shape[0]
        assert batch in (None, b), "every product of one call has the same batch"
        batch = b
        assert max_batch is None or b <= max_batch
        assert x.is_cuda and x.is_contiguous() and x.element_size() == 2 and x.numel() == b * cols
        assert y.is_cuda and y.is_contiguous() and y.dtype == torch.float32 and y.numel() == b * rows
        arr[k].d_fw = fw.data_ptr()
        arr[k].info = info
        arr[k].rows, arr[k].cols = rows, cols
        arr[k].d_x = x.data_ptr()
        arr[k].d_y = y.data_ptr()
    return n, arr, batch or 1


def fw_gemm(products, err: torch.Tensor, stream=None):
    """bs_fw_gemm: as fw_gemv, on the tensor cores, for any batch (rows a multiple of 128):
    products is a sequence of (fw, info, rows, cols, x [batch, cols] BF16, y [batch, rows] float32).
    err: a zeroed int32 CUDA tensor of one element. Enqueued on the stream."""
    n, arr, batch = _fw_products(products, None)
    assert err.is_cuda and err.dtype == torch.int32 and err.numel() >= 1
    with torch.cuda.device(err.device):
        _check(lib.bs_fw_gemm(n, arr, batch, err.data_ptr(), _stream(stream)), "fw_gemm")
    return [p[5] for p in products]


def fw_gemv(products, err: torch.Tensor, stream=None, layouts_resident: bool = False):
    """bs_fw_gemv: products is a sequence of (fw, info, rows, cols, x, y) with fw the layout of
    W (rows x cols), x a BF16 CUDA tensor [batch, cols] (or [cols]) and y a float32 CUDA
    tensor [batch, rows] (or [rows]); every x has the same batch (1..8). err: a zeroed int32
    CUDA tensor of one element. Enqueued on the stream. layouts_resident: BS_FW_LAYOUTS_RESIDENT,
    a statement that no work in flight on the stream writes the layouts (resident weights), so
    that their copies may start before the preceding kernel has finished."""
    n = len(products)
    arr = (FwGemvItem * max(n, 1))()
    batch = None
    for k, (fw, info, rows, cols, x, y) in enumerate(products):
        b = 1 if x.dim() == 1 else x.shape[0]
        assert batch in (None, b), "every product of one call has the same batch"
        batch = b
        assert x.is_cuda and x.is_contiguous() and x.element_size() == 2 and x.numel() == b * cols
        assert y.is_cuda and y.is_contiguous() and y.dtype == torch.float32 and y.numel() == b * rows
        arr[k].d_fw = fw.data_ptr()
        arr[k].info = info
        arr[k].rows, arr[k].cols = rows, cols
        arr[k].d_x = x.data_ptr()
        arr[k].d_y = y.data_ptr()
    assert err.is_cuda and err.dtype == torch.int32 and err.numel() >= 1
    with torch.cuda.device(err.device):
        _check(lib.bs_fw_gemv(n, arr, batch or 1, FW_LAYOUTS_RESIDENT if layouts_resident else 0, err.data_ptr(),
                              _stream(stream)), "fw_gemv")
    return [p[5] for p in products]
