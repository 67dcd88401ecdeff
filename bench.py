#!/usr/bin/env python
"""Decode benchmark: full-model lossless BF16 decode on B200.

One step decodes the whole 9B-shaped checkpoint, 9,241,702,400 BF16 weights in one
container, with one bs_decode_batch call. The container and the outputs are resident in
HBM. The synthetic weights are drawn on the device from the seeded recipe in
synthetic/, encoded once with the device encoder (untimed), planned, and checked
bit-exact against the originals before timing. The JSON line carries:

* value      decompressed BF16 GB/s over all ranks (replicas: every rank decodes its
             own copy of the checkpoint)
* roofline   (compressed bytes read + BF16 bytes written) per decode step over the step's
             CUDA-event time, against the measured HBM copy bandwidth
* e2e        the same metric with the container copied in from pinned host memory and
             every decoded tensor copied back out, inside the timed region; the copies
             and decodes of successive layer groups overlap on three streams
* cpu_baseline  the oracle decoder on the host cores, on a bounded sample (layer 0)

`--impl reference` times the oracle alone (host cores, rank 0) on the same sample.
"""
from __future__ import annotations

import argparse
import functools
import concurrent.futures as cf
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decompressed BF16 GB/s (full-model decode, 1 B200) and % HBM roofline; bits/weight"
FALLBACK_HBM_GBS = 6650.0


def _args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gemma2_9b", help="a workload of synthetic/ (default: the 9B checkpoint)")
    ap.add_argument("--layers", type=int, default=None, help="truncate a multi-layer workload (smaller cases)")
    ap.add_argument("--verify", choices=["originals", "checksum"], default="originals",
                    help="pre-timing parity: compare with the originals kept on the device, or free the "
                         "originals after encoding and check every tensor's checksum on the device "
                         "(for checkpoints whose originals, container and outputs do not fit together)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-modes", action="store_true",
                    help="model mode on the 9B checkpoint: skip the layer-by-layer and 27B-scale 1 GB-batch "
                         "measurements that the default line carries under 'modes'")
    ap.add_argument("--cpu-threads", type=int, default=0, help="oracle threads (0: all host cores)")
    ap.add_argument("--batch", type=int, default=1,
                    help="gemv mode: tokens per product (1..8 on the CUDA cores, more on the tensor cores)")
    ap.add_argument("--product", choices=["auto", "cuda", "tensor"], default="auto",
                    help="gemv mode: the CUDA-core product (bs_fw_gemv, batch 1..8), the tensor-core one "
                         "(bs_fw_gemm), or auto: tensor cores above batch 4, where they become the faster")
    ap.add_argument("--model", choices=["joint", "factored"], default="joint",
                    help="rANS model of the container: joint (one table over (s, h), kind JOINT; "
                         "the default) or factored (s-model plus exponent routes, kind RANS)")
    ap.add_argument("--mode", choices=["model", "layerwise", "stream", "fw", "gemv"], default="model",
                    help="model: one bs_decode_batch of every tensor per step (the default line); "
                         "layerwise: one bs_decode_batch per layer (group) per step; "
                         "stream: layer streaming from a host container through the LRU device cache; "
                         "fw: one bs_fw_decode of every tensor's fixed-width lane layout per step; "
                         "gemv: y = W x for every weight matrix from its layout (bs_fw_gemv), one "
                         "forward-shaped pass per step, against dense cuBLAS products")
    ap.add_argument("--batch-gb", type=float, default=None,
                    help="model mode: decode in batches of whole chunks of about this many GB of output, "
                         "one bs_decode_ranges call per batch (batches split tensors); default: one "
                         "bs_decode_batch of every tensor")
    ap.add_argument("--batch-streams", type=int, default=1,
                    help="model mode with --batch-gb: streams the batches go to in turn (1: one stream)")
    ap.add_argument("--layer-streams", type=int, default=1,
                    help="layerwise mode: streams consecutive layers go to in turn (1: one stream)")
    ap.add_argument("--log2-chunk", type=int, default=16, help="weights per chunk, as a power of two (8..24)")
    ap.add_argument("--vram-gb", type=float, default=None,
                    help="stream mode: device budget (arena) in GB; default: the smallest arena that "
                         "double-buffers the largest group")
    return ap.parse_args()


def _peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# DRAM traffic per decoded weight of each timed kernel: dram__bytes_read.sum +
# dram__bytes_write.sum of one ncu capture, over the weights that launch decoded. Each entry
# keeps the hash of the kernel's sources at capture time (comments and blank lines removed);
# the figure is reported only while the sources still hash to it, else traffic is null.
_TRAFFIC = {
    # joint4_decode_kernel, first 8 layers of the 9B checkpoint: 2.0910 GB read + 3.1208 GB
    # written for 1,585,561,600 weights
    "joint4_decode_kernel": (("bs_joint4.cu", "bs_device.cuh", "bs_internal.h"), "d8127505dd5bd2be", 3.28706),
    "fw_decode_kernel": (("bs_fw.cu", "bs_fw.cuh"), None, None),
    # fw_gemv_kernel, batch 1, the gate/up call of the 9B checkpoint's layer 0 (two 14336 x
    # 3584 matrices): 148.79 MB read + 3.63 MB written for 102,760,448 weights
    "fw_gemv_kernel": (("bs_fw_gemv.cu", "bs_fw.cuh"), "12b694d32f782e9f", 1.48328),
}


def _source_hash(files):
    """sha256 prefix of the given csrc files with comments and blank lines removed."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "lossless_entropy_coding_interleaved_b200", "csrc")
    text = ""
    for f in files:
        src = open(os.path.join(csrc, f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        text += "\n".join(l.rstrip() for l in src.splitlines() if l.strip()) + "\n"
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def _traffic_per_weight(kernel="joint4_decode_kernel"):
    """DRAM bytes per weight of a kernel from its capture, if its sources are unchanged; else None."""
    files, want, tpw = _TRAFFIC[kernel]
    try:
        return tpw if want is not None and _source_hash(files) == want else None
    except OSError:
        return None


def _workload_desc(name, layers):
    import synthetic as S
    specs = S.workload(name, layers=layers)
    n = sum(s.numel for s in specs if not s.is_raw)
    d = {"gemma2_9b": "42 Gemma-2-9B-shaped decoder layers (q,k,v,o,gate,up,down + 4 RMSNorm vectors) "
                      "+ 256000x3584 embedding",
         "gemma2_layer": "one Gemma-2-9B-shaped decoder layer",
         "qwen_27b_scale": "64 layers of hidden 5120 + 152064x5120 embedding",
         "tensor_1m": "one 1024x1024 tensor", "edge_mix": "edge-case mix"}.get(name, name)
    if layers is not None:
        d += f" (first {layers} layers only)"
    return specs, n, d


def _word_histograms(originals, specs, dev):
    """Per BF16 tensor, the 65536-bin histogram of its words (for the empirical entropy)."""
    import torch
    out = []
    for (nm, t), s in zip(originals, specs):
        if s.is_raw:
            continue
        flat = t.view(-1)
        cnt = torch.zeros(65536, dtype=torch.int64, device=dev)
        for lo in range(0, flat.numel(), 1 << 27):
            cnt += torch.bincount(flat[lo:lo + (1 << 27)].to(torch.int32) & 0xFFFF, minlength=65536)
        out.append((cnt, flat.numel()))
    return out


# ------------------------------------------------------------------ oracle on host cores
def _oracle_sample(workload, threads, model="joint"):
    """The bounded CPU sample: layer 0 of the workload (the whole of a one-tensor or one-layer
    workload), generated and encoded on the host by the oracle, then decoded by the oracle in
    chunk ranges (at most 16 chunks each) spread over `threads` host threads.

    Returns (n, desc, run_once, check). run_once(pool, every=1) decodes every `every`-th
    chunk range (every=1: the whole sample, including its STORED tensors) and returns
    (seconds, weights decoded)."""
    import numpy as np
    import oracle
    import synthetic as S
    specs = [s for s in S.workload(workload, layers=1) if not s.is_raw]
    if workload in ("gemma2_9b", "qwen_27b_scale"):
        specs = [s for s in specs if s.name.startswith("layers.0.")]
    arrs = [S.words_numpy(S.generate(s, "cpu")) for s in specs]
    c = np.frombuffer(oracle.encode([(s.name, a, "bf16") for s, a in zip(specs, arrs)], model=model), np.uint8)
    infos = [oracle.info(c, k) for k in range(len(specs))]
    outs = [np.zeros(i["n_elems"], np.uint16) for i in infos]
    coded = (oracle.KIND_RANS, oracle.KIND_JOINT)
    # ranges of at most 16 chunks, fewer when the sample is small, so that every thread has work
    total = sum(i["n_chunks"] for i in infos if i["kind"] in coded)
    span = max(1, min(16, total // (4 * max(1, threads))))
    tasks = []
    for k, i in enumerate(infos):
        if i["kind"] in coded:
            tasks += [(k, c0, min(c0 + span, i["n_chunks"])) for c0 in range(0, i["n_chunks"], span)]
    n = sum(a.size for a in arrs)
    desc = (f"oracle decode of layer 0 of {workload} ({len(specs)} tensors, {n} weights) in {len(tasks)} "
            f"chunk ranges of at most {span} chunks")

    def weights(k, c0, c1):
        C = 1 << infos[k]["log2_chunk"]
        return min(c1 * C, infos[k]["n_elems"]) - c0 * C

    def run_once(pool, every=1):
        sub = tasks[::every]
        t0 = time.perf_counter()
        futs = [pool.submit(oracle.decode_chunks, c, k, c0, c1, outs[k]) for k, c0, c1 in sub]
        if every == 1:
            for k, i in enumerate(infos):
                if i["kind"] not in coded:
                    outs[k][:] = oracle.decode(c, k).reshape(-1)
        assert all(f.result() == 0 for f in futs)
        sec = time.perf_counter() - t0
        return sec, (n if every == 1 else sum(weights(*t) for t in sub))

    def check():
        for a, o in zip(arrs, outs):
            assert np.array_equal(a.reshape(-1), o), "oracle sample decode mismatch"

    return n, desc, run_once, check


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


CPU_PASSES = 5
CPU_WORKLOADS = ("tensor_1m", "gemma2_layer", "gemma2_9b")


def _cpu_baseline(workload, threads, model, passes=CPU_PASSES):
    """The oracle on the host cores: for each of the three dense workloads' samples (layer 0
    of the checkpoint), the median of `passes` timed decodes on `threads` threads and on one
    thread (one thread decodes every 8th chunk range of the larger samples, which bounds its
    time). The headline value is the all-core figure on `workload`'s sample."""
    per = {}
    head = None
    for wl in dict.fromkeys(CPU_WORKLOADS + (workload,)):
        if wl not in ("tensor_1m", "gemma2_layer", "gemma2_9b", "qwen_27b_scale"):
            continue
        n, desc, run_once, check = _oracle_sample(wl, threads, model)
        every1 = 1 if n <= (1 << 22) else 8
        with cf.ThreadPoolExecutor(threads) as pool:
            run_once(pool)
            check()
            allc = [run_once(pool) for _ in range(passes)]
        with cf.ThreadPoolExecutor(1) as one:
            run_once(one, every1)
            single = [run_once(one, every1) for _ in range(passes)]
        gbs = lambda runs: 2 * statistics.median(w / sec for sec, w in runs) / 1e9
        per[wl] = {"all_cores_gbs": round(gbs(allc), 3), "single_thread_gbs": round(gbs(single), 3),
                   "weights": n, "single_thread_share": f"1/{every1} of the chunk ranges"}
        if wl == workload:
            head = (gbs(allc), desc)
    if head is None:
        return None
    return {"value": round(head[0], 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": head[1] + f"; median of {passes} passes over {threads} host threads",
            "single_thread": per[workload]["single_thread_gbs"], "cpu_model": _cpu_model(),
            "nproc": os.cpu_count(), "passes": passes, "stat": "median", "per_workload": per}


def _cpu_threads(req):
    return req if req > 0 else (os.cpu_count() or 1)


# ------------------------------------------------------------------ clocks during timing
class _Clocks:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 9]
        load = [r for r in rows if r[2].strip().isdigit() and int(r[2]) > 600]
        use = load or rows
        sm = [int(r[2]) for r in use if r[2].strip().isdigit()]
        mx = [int(r[3]) for r in use if r[3].strip().isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if r[6 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max((float(r[4]) for r in use if r[4].replace(".", "", 1).isdigit()), default=None)}


# ------------------------------------------------------------------ ranks (replicas only)
class _Ranks:
    """One process per GPU, launched by torch.distributed.run. The ranks are independent
    replicas: the only collectives are the barriers around the timed region and the max of
    the ranks' times, none of them on the data path."""

    def __init__(self, backend="nccl", device=None, timeout_s=300):
        import datetime
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" and device is not None else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, value: float) -> float:
        """The largest value over all ranks (every rank gets it)."""
        if self.world == 1:
            return float(value)
        import torch
        t = torch.tensor([float(value)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t)

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm
def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    threads = _cpu_threads(a.cpu_threads)
    specs, n_all, desc = _workload_desc(a.workload, a.layers)
    n, sample, run_once, check = _oracle_sample(a.workload, threads, a.model)
    with cf.ThreadPoolExecutor(threads) as pool:
        for _ in range(a.warmup):
            run_once(pool)
        check()
        ts = [run_once(pool)[0] for _ in range(a.steps)]
    # the median step, as the GPU arm's cpu_baseline leg reports it
    med = statistics.median(ts)
    value = 2 * n / med / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * med, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32",
            "data": "synthetic", "config": {"workload": a.workload, "description": desc, "n_weights": n_all,
                                            "step": "one bounded sample per step: " + sample,
                                            "stat": "median step time"},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample + f"; median of {a.steps} passes over {threads} host threads",
                             "cpu_model": _cpu_model(), "nproc": os.cpu_count()},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fw_reference(a):
    """--impl reference --mode fw: the oracle's FW decode alone on the host cores (rank 0)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    threads = _cpu_threads(a.cpu_threads)
    _, n_all, desc = _workload_desc(a.workload, a.layers)
    n, sample, run_once = _fw_oracle_sample(a.workload, threads)
    with cf.ThreadPoolExecutor(threads) as pool:
        for _ in range(a.warmup):
            run_once(pool)
        sec = sum(run_once(pool) for _ in range(a.steps))
    value = 2 * n * a.steps / sec / 1e9
    print(json.dumps({
        "impl": "reference", "metric": FW_METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * sec / a.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
        "config": {"workload": a.workload, "description": desc, "n_weights": n_all,
                   "step": "one bounded sample per step: " + sample},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


# ------------------------------------------------------------------ the other decode modes
def _mode_layerwise(plan, outs, infos, stream, steps, ranks, n_streams=1):
    """The same checkpoint decoded layer by layer: one bs_decode_batch per layer group per
    step, container and outputs in HBM, on one stream or, with n_streams = 2, on two streams
    in turn (as a consumer that double-buffers layers issues them; two layers' CTAs can then
    share the SMs). Returns the measurement as a dict."""
    import torch
    gid = _groups(plan.names)
    members = [[k for k in range(plan.n_tensors) if gid[k] == g] for g in range(max(gid) + 1)]
    coded = sum(i["coded_bytes"] for i in infos)
    out_bytes = sum(i["out_bytes"] for i in infos)
    side = [torch.cuda.Stream(device=stream.device) for _ in range(n_streams)] if n_streams > 1 else []

    def step():
        if not side:
            for m in members:
                plan.decode_batch(m, [outs[k] for k in m], stream=stream)
            return
        start = torch.cuda.Event()
        start.record(stream)
        for s_ in side:
            s_.wait_event(start)
        for i, m in enumerate(members):
            plan.decode_batch(m, [outs[k] for k in m], stream=side[i % len(side)])
        for s_ in side:
            stream.wait_stream(s_)

    for _ in range(3):
        step()
    ms = ranks.max(_timed(stream, steps, step, ranks.barrier))
    plan.check()
    peak, _ = _peak_hbm()
    achieved = (coded + out_bytes) * steps / (ms * 1e-3) / 1e9
    return {"value": round(ranks.world * steps * out_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
            "ms_per_step": round(ms / steps, 4), "steps": steps, "groups": len(members),
            "calls_per_step": len(members), "roofline_frac": round(achieved / peak, 4),
            "how": "one bs_decode_batch per layer group (42 layers + the embedding), "
                   + ("one stream" if not side else f"{n_streams} streams in turn")}


def _mode_batches(workload, batch_gb, model, dev, stream, steps, ranks):
    """A checkpoint decoded in batches of whole chunks holding at most batch_gb GB of output and
    one kernel wave each (bs_decode_ranges), one stream. The originals are freed after the
    histograms, and every tensor's checksum is verified on the device before timing."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    import synthetic as S
    specs, n, _ = _workload_desc(workload, None)
    originals = [(s.name, S.generate(s, dev)) for s in specs]
    d_c, _ = bs.encode(originals, model=model)
    hist = _word_histograms(originals, specs, dev)
    del originals
    torch.cuda.empty_cache()
    plan = bs.Plan(d_container=d_c)
    outs = [plan.empty_output(k) for k in range(plan.n_tensors)]
    infos = [plan.info(k) for k in range(plan.n_tensors)]
    coded = sum(i["coded_bytes"] for i in infos)
    out_bytes = sum(i["out_bytes"] for i in infos)
    bf16_n = sum(i["n_elems"] for i in infos if i["kind"] != bs.KIND_RAW)
    bf16_coded = sum(i["coded_bytes"] for i in infos if i["kind"] != bs.KIND_RAW)
    hbits = 0.0
    for cnt, numel in hist:
        c = cnt[cnt > 0].to(torch.float64)
        hbits += float(-(c * torch.log2(c / numel)).sum())
    batches = _chunk_batches(plan, infos, outs, batch_gb)

    def step():
        for b in batches:
            plan.decode_ranges(b, stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    plan.check()
    for k in range(plan.n_tensors):
        plan.verify(k, outs[k])                  # raises on any mismatch
    ms = ranks.max(_timed(stream, steps, step, ranks.barrier))
    plan.check()
    peak, _ = _peak_hbm()
    achieved = (coded + out_bytes) * steps / (ms * 1e-3) / 1e9
    res = {"value": round(ranks.world * steps * out_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
           "ms_per_step": round(ms / steps, 4), "steps": steps, "workload": workload, "n_weights": n,
           "batches": len(batches), "batch_gb": batch_gb, "roofline_frac": round(achieved / peak, 4),
           "bits_per_weight": round(bf16_coded * 8 / bf16_n, 5),
           "overhead_pct_vs_entropy": round(100 * (bf16_coded * 8 / hbits - 1), 4),
           "parity": "every tensor's checksum verified on the device before timing",
           "how": f"one bs_decode_ranges call per batch of at most {batch_gb} GB of output and one kernel "
                  "wave, in container order, one stream"}
    del plan, outs, d_c
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ our arm
def run_ours(a):
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    import synthetic as S

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = _Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier = ranks.barrier

    specs, n, desc = _workload_desc(a.workload, a.layers)
    t0 = time.time()
    originals = [(s.name, S.generate(s, dev)) for s in specs]
    d_c, _ = bs.encode(originals, model=a.model, log2_chunk=a.log2_chunk)
    torch.cuda.synchronize()
    t_encode = time.time() - t0
    hist_words = None
    if a.verify == "checksum":
        # keep only what the entropy needs, then free the originals before decoding
        hist_words = _word_histograms(originals, specs, dev)
        originals = None
        torch.cuda.empty_cache()
    plan = bs.Plan(d_container=d_c)
    container_bytes = int(d_c.numel())
    outs = [plan.empty_output(k) for k in range(plan.n_tensors)]
    idx = list(range(plan.n_tensors))
    infos = [plan.info(k) for k in idx]
    coded = sum(i["coded_bytes"] for i in infos)
    out_bytes = sum(i["out_bytes"] for i in infos)
    bf16_n = sum(i["n_elems"] for i in infos if i["kind"] != bs.KIND_RAW)
    bf16_coded = sum(i["coded_bytes"] for i in infos if i["kind"] != bs.KIND_RAW)

    # empirical entropy H(s) + H(f|s) = H(w) of the originals, on the device
    if hist_words is None:
        hist_words = _word_histograms(originals, specs, dev)
    hbits = 0.0
    for cnt, numel in hist_words:
        c = cnt[cnt > 0].to(torch.float64)
        hbits += float(-(c * torch.log2(c / numel)).sum())
    h_per_w = hbits / bf16_n

    stream = torch.cuda.current_stream()
    batches = _chunk_batches(plan, infos, outs, a.batch_gb) if a.batch_gb else None
    # with several streams, one batch's last CTAs may overlap the next one's first
    side = [torch.cuda.Stream(device=dev) for _ in range(max(1, a.batch_streams))] if batches else []

    def step():
        if batches is None:
            plan.decode_batch(idx, outs, stream=stream)
            return
        start = torch.cuda.Event()
        start.record(stream)
        for s_ in side:
            s_.wait_event(start)
        for i, b in enumerate(batches):
            plan.decode_ranges(b, stream=side[i % len(side)])
        for s_ in side:
            stream.wait_stream(s_)

    for _ in range(max(1, a.warmup)):
        step()
    torch.cuda.synchronize()
    plan.check()
    if originals is not None:
        parity = all(torch.equal(o.view(-1), t.view(-1)) for o, (_, t) in zip(outs, originals))
        parity_how = "bit-exact vs originals before timing"
    else:
        for k in idx:
            plan.verify(k, outs[k])            # raises on any mismatch
        parity, parity_how = True, "every tensor's checksum verified on the device before timing"
    if not parity:
        raise SystemExit("bench: decoded output differs from the originals")
    del originals
    torch.cuda.empty_cache()

    # timed region: K steps, CUDA events per step on the launching stream
    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    smi_index = phys[local] if local < len(phys) and phys[local].strip().isdigit() else str(local)
    clocks = _Clocks(smi_index)
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    # a container and outputs that fit in L2 (the small workloads) would be timed from the
    # cache: write a buffer of twice the L2 size before each step, outside its events, and
    # time the sum of the steps' events instead of the whole loop
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = (torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)
                 if coded + out_bytes < 2 * l2_bytes else None)
    barrier()
    torch.cuda.synchronize()
    l0 = bs.launch_counter()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for k in range(a.steps):
        if flush_buf is not None:
            flush_buf.fill_(k & 0xFF)
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = bs.launch_counter() - l0
    clk = clocks.stop()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    total_ms = g0.elapsed_time(g1) if flush_buf is None else sum(step_ms)
    plan.check()
    total_ms = ranks.max(total_ms)
    value = world * a.steps * out_bytes / (total_ms * 1e-3) / 1e9
    mean_step = statistics.mean(step_ms)
    peak, peak_kind = _peak_hbm()
    tpw = _traffic_per_weight() if a.model == "joint" else None
    achieved = (coded + out_bytes) / (mean_step * 1e-3) / 1e9

    # end to end: container in from pinned host memory, every tensor back out, per step,
    # pipelined per layer group over three streams (the public Plan.decode_batch per group)
    e2e = None
    if not a.no_e2e and a.e2e_steps > 0:
        h_c = torch.empty(d_c.numel(), dtype=torch.uint8, pin_memory=True)
        h_c.copy_(d_c)
        h_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        ranges, members = _group_ranges(h_c.numpy(), plan.names)
        torch.cuda.synchronize()
        barrier()
        s_in, s_dec, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        n_g = len(members)
        done_out = [None] * n_g     # event: the previous step's copy-out of group g finished
        done_dec = [None] * n_g     # event: the previous step's decode of group g finished
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (s_in, s_dec, s_out):
            st.wait_event(e0)
        for _ in range(a.e2e_steps):
            for g in range(n_g):
                lo, hi = ranges[g]
                if done_dec[g] is not None:   # do not overwrite bytes a decode may still read
                    s_in.wait_event(done_dec[g])
                with torch.cuda.stream(s_in):
                    d_c[lo:hi].copy_(h_c[lo:hi], non_blocking=True)
                    arrived = torch.cuda.Event()
                    arrived.record(s_in)
                s_dec.wait_event(arrived)
                if done_out[g] is not None:
                    s_dec.wait_event(done_out[g])
                plan.decode_batch(members[g], [outs[k] for k in members[g]], stream=s_dec)
                decoded = torch.cuda.Event()
                decoded.record(s_dec)
                done_dec[g] = decoded
                s_out.wait_event(decoded)
                with torch.cuda.stream(s_out):
                    for k in members[g]:
                        h_outs[k].copy_(outs[k], non_blocking=True)
                    done_out[g] = torch.cuda.Event()
                    done_out[g].record(s_out)
        for st in (s_in, s_dec, s_out):
            stream.wait_stream(st)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        plan.check()
        e_ms = ranks.max(e0.elapsed_time(e1))
        e2e = {"value": round(world * a.e2e_steps * out_bytes / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(sum(hi - lo for lo, hi in ranges)), "d2h_bytes_per_step": int(out_bytes),
               "steps": a.e2e_steps, "groups": n_g,
               "path": "per layer group: its container bytes copied in from pinned host memory, "
                       "Plan.decode_batch, its tensors copied back out; three streams overlap the groups"}
        del h_c, h_outs

    # the other two decode modes of the target, beside the whole-model number: the same 9B
    # checkpoint layer by layer, and the 27B-scale checkpoint in 1 GB batches
    modes = None
    if (not a.no_modes and a.workload == "gemma2_9b" and a.layers is None and a.batch_gb is None
            and a.log2_chunk == 16):
        modes = {"layerwise": _mode_layerwise(plan, outs, infos, stream, a.steps, ranks),
                 "layerwise_two_streams": _mode_layerwise(plan, outs, infos, stream, a.steps, ranks, 2)}
        del plan, outs, d_c
        torch.cuda.empty_cache()
        modes["qwen_27b_scale_1gb_batches"] = _mode_batches("qwen_27b_scale", 1.0, a.model, dev, stream,
                                                            max(5, a.steps // 2), ranks)

    cpu = None
    if rank == 0 and not a.no_cpu_baseline:
        cpu = _cpu_baseline(a.workload, _cpu_threads(a.cpu_threads), a.model)

    ranks.close()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(total_ms / a.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32",
        "data": "synthetic (seeded device draws, synthetic/ recipe)",
        "config": {"workload": a.workload, "description": desc, "n_weights": n, "tensors": len(specs),
                   "container_bytes": container_bytes, "coded_bytes": int(coded),
                   "decoded_bytes": int(out_bytes),
                   "bits_per_weight": round(bf16_coded * 8 / bf16_n, 5),
                   "entropy_bits_per_weight": round(h_per_w, 5),
                   "overhead_pct_vs_entropy": round(100 * (bf16_coded * 8 / bf16_n / h_per_w - 1), 4),
                   "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": ("no flush: inputs larger than L2 (container and outputs are GBs)" if flush_buf is None
                          else f"flushed: {2 * l2_bytes >> 20} MiB written before each step, outside its "
                               "events; value from the sum of the step times"),
                   "parity": parity_how, "encode_s": round(t_encode, 2),
                   "log2_chunk": a.log2_chunk,
                   "batches": ("one bs_decode_batch of every tensor" if batches is None else
                               f"{len(batches)} bs_decode_ranges calls of at most {a.batch_gb} GB of output and one "
                               "kernel wave each (whole chunks, in container order; batches split tensors), on "
                               f"{max(1, a.batch_streams)} stream(s) in turn"),
                   "words": "BF16 bit patterns; rANS state arithmetic in u32",
                   "model": ("joint: one rANS table over (sign+exponent, top 3 fraction bits), nj = 13 "
                             "(kind JOINT)" if a.model == "joint" else
                             "factored: s-model (ns = 11) and exponent routes (nh = 5) (kind RANS)")},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": (None if tpw is None else int(tpw * bf16_n)),
                     "traffic_source": "ncu capture of this kernel on the first 8 layers, scaled by weights",
                     "kernel": ("joint4_decode_kernel (with decode_kernel for the JOINT tensors whose "
                                "frequencies exceed 255: the 168 RMSNorm vectors, 0.3% of the step)"
                                if a.model == "joint" else "decode_kernel"),
                     "per_launch_bytes": int(coded + out_bytes),
                     "launch_ms_mean": round(mean_step, 4)},
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if modes is not None:
        line["modes"] = modes
    print(json.dumps(line), flush=True)


def _group_of(name: str):
    """Layer grouping: tensors named layers.<L>.* form group L; every other tensor forms its
    own group."""
    return ("layer", name.split(".")[1]) if name.startswith("layers.") else ("other", name)


def _groups(names):
    keys = {}
    return [keys.setdefault(_group_of(n), len(keys)) for n in names]


def _group_ranges(h: "np.ndarray", names):
    """Per layer group, the contiguous container bytes its tensors use and its member indices.

    The canonical layout writes each tensor's sections (RANS: model,
    chunk table, chunks; else the data) in directory order, each tensor starting at its
    model_offset (RANS) or data_offset. A group's tensors are consecutive, so its bytes run
    from its first tensor's start to the next group's start (or the end of the container)."""
    import numpy as np
    hdr = h[:64].tobytes()
    nt = int.from_bytes(hdr[16:20], "little")
    d0 = int.from_bytes(hdr[24:32], "little")
    total = int.from_bytes(hdr[48:56], "little")
    starts = []
    for k in range(nt):
        e = h[d0 + 144 * k: d0 + 144 * k + 144].tobytes()
        kind = e[0]
        model_off, data_off = int.from_bytes(e[32:40], "little"), int.from_bytes(e[48:56], "little")
        starts.append(model_off if kind == 0 else data_off)
    gid = _groups(names)
    members, ranges = [], []
    for k in range(nt):
        if k == 0 or gid[k] != gid[k - 1]:
            members.append([])
        members[-1].append(k)
    for g, m in enumerate(members):
        lo = starts[m[0]]
        hi = starts[members[g + 1][0]] if g + 1 < len(members) else total
        assert all(starts[k] >= lo for k in m) and hi >= lo
        ranges.append((lo, hi))
    return ranges, members


def _setup(a, dev):
    """Generate the workload on the device, encode it (untimed) and compute its entropy."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    import synthetic as S
    specs, n, desc = _workload_desc(a.workload, a.layers)
    t0 = time.time()
    originals = [(s.name, S.generate(s, dev)) for s in specs]
    d_c, h_c = bs.encode(originals, host_copy=a.mode == "stream", model=a.model)
    torch.cuda.synchronize()
    t_encode = time.time() - t0
    hist = _word_histograms(originals, specs, dev)
    bf16_n = sum(s.numel for s in specs if not s.is_raw)
    hbits = 0.0
    for cnt, numel in hist:
        c = cnt[cnt > 0].to(torch.float64)
        hbits += float(-(c * torch.log2(c / numel)).sum())
    return specs, n, desc, originals, d_c, h_c, t_encode, hbits / bf16_n


def _timed(stream, steps, body, barrier):
    """CUDA-event time (ms) of `steps` calls of body(), bracketed by barrier + synchronize."""
    import torch
    barrier()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(steps):
        body()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return g0.elapsed_time(g1)


def _chunk_batches(plan, infos, outs, batch_gb):
    """The checkpoint's chunks in tensor order, cut into batches of at most batch_gb GB of
    output that each fill at most one wave of the decode kernel (bs_decode_geometry): each
    batch is a list of (idx, begin, count, out view) ranges for Plan.decode_ranges. A
    tensor's ranges are whole CTAs' worth of chunks except its last, so no range leaves a
    part-filled CTA in the middle of a tensor. STORED and RAW tensors go whole into the
    batch that reaches them."""
    import lossless_entropy_coding_interleaved_b200 as bs
    cap = int(batch_gb * 1e9)
    batches, cur = [], []
    room, ctas_free = cap, None

    def close():
        nonlocal cur, room, ctas_free
        if cur:
            batches.append(cur)
        cur, room, ctas_free = [], cap, None

    for k, i in enumerate(infos):
        n = i["n_elems"]
        if i["kind"] not in (bs.KIND_RANS, bs.KIND_JOINT):
            per = 1 if i["kind"] == bs.KIND_RAW else 2
            if n and room < per * n:
                close()
            cur.append((k, 0, n, outs[k].view(-1)))
            room -= per * n
            continue
        cpc, wave = plan.decode_geometry(k)
        C = 1 << i["log2_chunk"]
        n_chunks = -(-n // C)
        c = 0
        while c < n_chunks:
            if ctas_free is None:
                ctas_free = wave
            fit = min(n_chunks - c, ctas_free * cpc, room // (2 * C))
            if fit < n_chunks - c:
                fit -= fit % cpc                          # whole CTAs unless it ends the tensor
            if fit <= 0:
                if not cur:                               # an empty batch takes one CTA's worth
                    fit = min(cpc, n_chunks - c)
                else:
                    close()
                    continue
            b, cnt = c * C, min(fit * C, n - c * C)
            cur.append((k, b, cnt, outs[k].view(-1)[b:b + cnt]))
            c += fit
            room -= 2 * cnt
            ctas_free -= -(-fit // cpc)
            if ctas_free <= 0 or room < 2 * C:
                close()
    close()
    return batches


def run_layerwise(a):
    """One bs_decode_batch per layer group per step, container and outputs in HBM."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = _Ranks("nccl", dev)
    specs, n, desc, originals, d_c, _, t_encode, h_per_w = _setup(a, dev)
    plan = bs.Plan(d_container=d_c)
    outs = [plan.empty_output(k) for k in range(plan.n_tensors)]
    gid = _groups(plan.names)
    members = [[k for k in range(plan.n_tensors) if gid[k] == g] for g in range(max(gid) + 1)]
    infos = [plan.info(k) for k in range(plan.n_tensors)]
    coded = sum(i["coded_bytes"] for i in infos)
    out_bytes = sum(i["out_bytes"] for i in infos)
    stream = torch.cuda.current_stream()
    # with --layer-streams 2, consecutive layers alternate between two streams, as a consumer
    # that double-buffers layers would decode them: two layers' chunks share the SMs
    side = [torch.cuda.Stream(device=dev) for _ in range(max(1, a.layer_streams))]

    def step():
        if len(side) == 1:
            for m in members:
                plan.decode_batch(m, [outs[k] for k in m], stream=stream)
            return
        start = torch.cuda.Event()
        start.record(stream)
        for s_ in side:
            s_.wait_event(start)
        for i, m in enumerate(members):
            plan.decode_batch(m, [outs[k] for k in m], stream=side[i % len(side)])
        for s_ in side:
            stream.wait_stream(s_)

    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize()
    plan.check()
    if not all(torch.equal(o.view(-1), t.view(-1)) for o, (_, t) in zip(outs, originals)):
        raise SystemExit("bench: decoded output differs from the originals")
    del originals
    torch.cuda.empty_cache()
    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    clocks = _Clocks(phys[local] if local < len(phys) and phys[local].strip().isdigit() else str(local))
    time.sleep(0.3)
    l0 = bs.launch_counter()
    ms = ranks.max(_timed(stream, a.steps, step, ranks.barrier))
    launches = bs.launch_counter() - l0
    clk = clocks.stop()
    plan.check()
    peak, peak_kind = _peak_hbm()
    achieved = (coded + out_bytes) * a.steps / (ms * 1e-3) / 1e9
    ranks.close()
    if ranks.rank != 0:
        return
    print(json.dumps({
        "metric": "decompressed BF16 GB/s, layer by layer (one bs_decode_batch per layer)",
        "value": round(ranks.world * a.steps * out_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
        "n_gpus": ranks.world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms / a.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
        "config": {"workload": a.workload, "description": desc, "n_weights": n, "groups": len(members),
                   "layer_streams": len(side),
                   "decoded_bytes": int(out_bytes), "coded_bytes": int(coded),
                   "entropy_bits_per_weight": round(h_per_w, 5), "encode_s": round(t_encode, 2),
                   "l2": "no flush: inputs larger than L2", "parity": "bit-exact vs originals before timing"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "kernel": "decode_kernel (all launches of a step)"},
        "gpu_launches": int(launches), "clocks": clk}), flush=True)


def run_stream(a):
    """Layer streaming: the container stays in pinned host memory, and each pass walks the
    groups in order through bs_streamer. The next group is prefetched on alternating copy
    streams while the current one is acquired on the compute stream. The comparison is
    streaming the same layers dense: their BF16 bytes copied host-to-device in the same
    pattern."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = _Ranks("nccl", dev)
    specs, n, desc, originals, d_c, h_c, t_encode, h_per_w = _setup(a, dev)
    del d_c
    torch.cuda.empty_cache()
    names = [s.name for s in specs]
    gid = _groups(names)
    n_groups = max(gid) + 1
    members = [[k for k in range(len(specs)) if gid[k] == g] for g in range(n_groups)]
    dense = [sum(originals[k][1].numel() * originals[k][1].element_size() for k in m) for m in members]
    h_pinned = torch.empty(h_c.size, dtype=torch.uint8, pin_memory=True)
    h_pinned.numpy()[:] = h_c
    del h_c
    arena = (bs.streamer_min_arena_bytes(h_pinned, gid) + max(dense) + (len(specs) << 8) if a.vram_gb is None
             else int(a.vram_gb * 1e9))
    st = bs.Streamer(h_pinned, gid, arena_bytes=arena, device=dev)
    main = torch.cuda.current_stream()
    side = [torch.cuda.Stream(), torch.cuda.Stream()]
    prefetch_refused = [0]

    def one_pass(check=False):
        try:
            st.prefetch(0, stream=side[0])
        except bs.BsError as e:
            if e.code != bs.E_SIZE:
                raise
        for g in range(n_groups):
            if g + 1 < n_groups:
                try:
                    st.prefetch(g + 1, stream=side[(g + 1) % 2])
                except bs.BsError as e:       # the pinned group leaves no room: acquire loads it
                    if e.code != bs.E_SIZE:
                        raise
                    prefetch_refused[0] += 1
            outs = st.acquire(g, stream=main)
            if check:
                for k, o in zip(members[g], outs):
                    if not torch.equal(o.reshape(-1), originals[k][1].reshape(-1)):
                        raise SystemExit(f"bench: streamed {names[k]} differs from the original")
            st.release(g, stream=main)

    one_pass(check=True)
    torch.cuda.synchronize()
    st.check()
    # dense comparison: the same bytes, per group, host-to-device from pinned memory
    h_dense = [torch.empty(b, dtype=torch.uint8, pin_memory=True) for b in dense]
    for m, h in zip(members, h_dense):
        pos = 0
        for k in m:
            t = originals[k][1].view(-1).view(torch.uint8)
            h[pos:pos + t.numel()].copy_(t)
            pos += t.numel()
    d_dense = [torch.empty(max(dense), dtype=torch.uint8, device=dev) for _ in range(2)]
    del originals
    torch.cuda.empty_cache()

    def dense_pass():
        for g in range(n_groups):
            s = side[g % 2]
            s.wait_stream(main)
            with torch.cuda.stream(s):
                d_dense[g % 2][:dense[g]].copy_(h_dense[g], non_blocking=True)
            main.wait_stream(s)

    for _ in range(max(3, a.warmup)):
        one_pass()
        dense_pass()
    torch.cuda.synchronize()
    s0 = st.stats()
    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    clocks = _Clocks(phys[local] if local < len(phys) and phys[local].strip().isdigit() else str(local))
    time.sleep(0.3)
    l0 = bs.launch_counter()
    ms = ranks.max(_timed(main, a.steps, one_pass, ranks.barrier))
    launches = bs.launch_counter() - l0
    clk = clocks.stop()
    s1 = st.stats()
    st.check()
    ms_dense = ranks.max(_timed(main, a.steps, dense_pass, ranks.barrier))
    out_bytes = sum(dense)
    h2d = (s1["h2d_bytes"] - s0["h2d_bytes"]) / a.steps
    loads = (s1["loads"] - s0["loads"]) / a.steps
    h2d_peak = out_bytes / (ms_dense / a.steps * 1e-3) / 1e9
    achieved = h2d / (ms / a.steps * 1e-3) / 1e9
    ranks.close()
    if ranks.rank != 0:
        return
    print(json.dumps({
        "metric": "streamed decode GB/s: BF16 bytes delivered per second from a host container through the "
                  "LRU device cache",
        "value": round(ranks.world * a.steps * out_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
        "n_gpus": ranks.world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms / a.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
        "config": {"workload": a.workload, "description": desc, "n_weights": n, "groups": n_groups,
                   "arena_bytes": int(arena), "stage_bytes": s1["stage_bytes"],
                   "decoded_bytes_per_pass": int(out_bytes), "h2d_bytes_per_pass": int(h2d),
                   "loads_per_pass": loads, "prefetch_refused": prefetch_refused[0],
                   "vram_saving_x": round(out_bytes / arena, 2), "entropy_bits_per_weight": round(h_per_w, 5),
                   "encode_s": round(t_encode, 2), "parity": "every group bit-exact vs originals on a first pass",
                   "l2": "no flush: every pass moves GBs"},
        "dense_streaming": {"value": round(ranks.world * a.steps * out_bytes / (ms_dense * 1e-3) / 1e9, 3),
                            "unit": "GB/s", "ms_per_step": round(ms_dense / a.steps, 3),
                            "what": "the same layers' BF16 bytes copied host-to-device per group, "
                                    "alternating two copy streams"},
        "speedup_vs_dense_streaming": round(ms_dense / ms, 3),
        "roofline": {"bound": "h2d", "achieved": round(achieved, 2), "peak": round(h2d_peak, 2),
                     "peak_kind": "measured in this run (dense pinned host-to-device copies)", "unit": "GB/s",
                     "frac": round(achieved / h2d_peak, 4), "traffic": None},
        "e2e": {"value": round(ranks.world * a.steps * out_bytes / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 0},
        "gpu_launches": int(launches), "clocks": clk}), flush=True)


# ------------------------------------------------------------------ fixed-width lane layout
FW_METRIC = "decompressed BF16 GB/s from the fixed-width lane layout (full model, 1 B200) and % HBM roofline"


def _fw_oracle_sample(workload, threads):
    """The bounded CPU sample of the FW mode: layer 0 of the workload, laid out and decoded
    by the oracle (one tensor per task on `threads` host threads)."""
    import numpy as np
    import oracle
    import synthetic as S
    specs = [s for s in S.workload(workload, layers=1) if not s.is_raw]
    if workload in ("gemma2_9b", "qwen_27b_scale"):
        specs = [s for s in specs if s.name.startswith("layers.0.")]
    arrs = [S.words_numpy(S.generate(s, "cpu")).reshape(-1) for s in specs]
    with cf.ThreadPoolExecutor(threads) as pool:
        blobs = list(pool.map(oracle.fw_encode, arrs))
    n = sum(a.size for a in arrs)
    desc = f"oracle FW decode of layer 0 of {workload} ({len(specs)} tensors, {n} weights) on {threads} host threads"

    def run_once(pool):
        t0 = time.perf_counter()
        outs = list(pool.map(oracle.fw_decode, blobs))
        sec = time.perf_counter() - t0
        assert all(np.array_equal(a, o) for a, o in zip(arrs, outs)), "oracle FW sample mismatch"
        return sec

    return n, desc, run_once


def run_fw(a):
    """Decode every BF16 tensor of the workload from its fixed-width lane layout (one
    bs_fw_decode per step); layouts and outputs resident in HBM."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    import synthetic as S
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = _Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    specs, _, desc = _workload_desc(a.workload, a.layers)
    specs = [s for s in specs if not s.is_raw]
    originals = [S.generate(s, dev).reshape(-1) for s in specs]
    torch.cuda.synchronize()
    t0 = time.time()
    built = [bs.fw_transcode(w) for w in originals]
    torch.cuda.synchronize()
    t_transcode = time.time() - t0
    fws = [f for f, _ in built]
    infos = [i for _, i in built]
    n = sum(i.n_elems for i in infos)
    n_exc = sum(i.n_exc for i in infos)
    fw_bytes = sum(i.total_bytes for i in infos)
    out_bytes = 2 * n
    outs = [torch.empty_like(w) for w in originals]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(1, a.warmup)):
        bs.fw_decode(fws, infos, outs, err, stream=stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0 or not all(torch.equal(o, w) for o, w in zip(outs, originals)):
        raise SystemExit("bench: FW decode differs from the originals")
    del originals
    torch.cuda.empty_cache()

    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    smi_index = phys[local] if local < len(phys) and phys[local].strip().isdigit() else str(local)
    clocks = _Clocks(smi_index)
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    l0 = bs.launch_counter()
    it = iter(ev)

    def step():
        e0, e1 = next(it)
        e0.record(stream)
        bs.fw_decode(fws, infos, outs, err, stream=stream)
        e1.record(stream)

    total_ms = ranks.max(_timed(stream, a.steps, step, ranks.barrier))
    launches = bs.launch_counter() - l0
    clk = clocks.stop()
    if int(err.item()) != 0:
        raise SystemExit("bench: FW decode raised its error flag")
    mean_step = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    value = world * a.steps * out_bytes / (total_ms * 1e-3) / 1e9
    peak, peak_kind = _peak_hbm()
    achieved = (fw_bytes + out_bytes) / (mean_step * 1e-3) / 1e9
    tpw = _traffic_per_weight("fw_decode_kernel")

    # end to end: every layout copied in from pinned host memory and every output copied back,
    # per layer group on three streams so that the copies of one group overlap the others
    e2e = None
    if not a.no_e2e and a.e2e_steps > 0:
        h_fw = [torch.empty(f.shape, dtype=f.dtype, pin_memory=True) for f in fws]
        for h, f in zip(h_fw, fws):
            h.copy_(f)
        h_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        gid = _groups([s.name for s in specs])
        members = {}
        for k, g in enumerate(gid):
            members.setdefault(g, []).append(k)
        members = list(members.values())
        torch.cuda.synchronize()
        ranks.barrier()
        s_in, s_dec, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        done_dec, done_out = [None] * len(members), [None] * len(members)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (s_in, s_dec, s_out):
            st.wait_event(e0)
        for _ in range(a.e2e_steps):
            for g, m in enumerate(members):
                if done_dec[g] is not None:
                    s_in.wait_event(done_dec[g])
                with torch.cuda.stream(s_in):
                    for k in m:
                        fws[k].copy_(h_fw[k], non_blocking=True)
                    arrived = torch.cuda.Event()
                    arrived.record(s_in)
                s_dec.wait_event(arrived)
                if done_out[g] is not None:
                    s_dec.wait_event(done_out[g])
                bs.fw_decode([fws[k] for k in m], [infos[k] for k in m], [outs[k] for k in m], err, stream=s_dec)
                decoded = torch.cuda.Event()
                decoded.record(s_dec)
                done_dec[g] = decoded
                s_out.wait_event(decoded)
                with torch.cuda.stream(s_out):
                    for k in m:
                        h_out[k].copy_(outs[k], non_blocking=True)
                    done_out[g] = torch.cuda.Event()
                    done_out[g].record(s_out)
        for st in (s_in, s_dec, s_out):
            stream.wait_stream(st)
        e1.record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
        if int(err.item()) != 0:
            raise SystemExit("bench: FW decode raised its error flag (e2e)")
        e_ms = ranks.max(e0.elapsed_time(e1))
        e2e = {"value": round(world * a.e2e_steps * out_bytes / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(fw_bytes), "d2h_bytes_per_step": int(out_bytes), "steps": a.e2e_steps,
               "groups": len(members),
               "path": "per layer group: its layouts copied in from pinned host memory, bs_fw_decode, "
                       "its tensors copied back out; three streams overlap the groups"}
        del h_fw, h_out

    cpu = None
    if rank == 0 and not a.no_cpu_baseline:
        threads = _cpu_threads(a.cpu_threads)
        n_s, sample, run_once = _fw_oracle_sample(a.workload, threads)
        with cf.ThreadPoolExecutor(threads) as pool:
            run_once(pool)
            sec = run_once(pool)
        cpu = {"value": round(2 * n_s / sec / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": sample}
    ranks.close()
    if rank != 0:
        return
    print(json.dumps({
        "metric": FW_METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(total_ms / a.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32",
        "data": "synthetic (seeded device draws, synthetic/ recipe)",
        "config": {"workload": a.workload, "description": desc, "n_weights": n, "tensors": len(specs),
                   "layout": "fixed-width lane layout: 4-bit sign+exponent codes, the 7-bit fraction, exceptions",
                   "fw_bytes": int(fw_bytes), "decoded_bytes": int(out_bytes), "escapes": int(n_exc),
                   "bits_per_weight": round(8 * fw_bytes / n, 5), "transcode_s": round(t_transcode, 3),
                   "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": "no flush: inputs larger than L2 (layouts and outputs are GBs)",
                   "parity": "bit-exact vs originals before timing; error word checked after"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": (None if tpw is None else int(tpw * n)),
                     "traffic_source": "ncu capture of this kernel, scaled by weights",
                     "kernel": "fw_decode_kernel", "per_launch_bytes": int(fw_bytes + out_bytes),
                     "launch_ms_mean": round(mean_step, 4)},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": int(launches), "clocks": clk}), flush=True)


# ------------------------------------------------------------------ fused GEMV on the layout
GEMV_METRIC = "BF16-equivalent weight GB/s of y = W x from the fixed-width lane layout (every matrix, 1 B200)"


def _gemv_calls(specs):
    """The products of one forward-shaped pass, grouped as a decoder step issues them: per layer
    (q, k, v) on one x, o, (gate, up) on one x, down; then the LM head on the embedding.
    The synthetic matrices are iid, so each layer tensor is multiplied as the [out, in] matrix
    of its projection (rows = its second dimension) and the embedding as [vocab, hidden]."""
    by = {s.name: k for k, s in enumerate(specs)}
    calls = []
    layers = sorted({int(s.name.split(".")[1]) for s in specs if s.name.startswith("layers.")})
    for L in layers:
        for grp in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",)):
            ks = [by[f"layers.{L}.{m}"] for m in grp if f"layers.{L}.{m}" in by]
            if ks:
                calls.append([(k, specs[k].shape[1], specs[k].shape[0]) for k in ks])
    if "embed" in by:
        k = by["embed"]
        calls.append([(k, specs[k].shape[0], specs[k].shape[1])])
    return calls


def run_gemv(a):
    """One step = every weight matrix's product y = W x, straight from its FW layout, grouped as
    a decoder pass issues them (169 calls for the 9B checkpoint), captured in a CUDA graph."""
    import torch

    import lossless_entropy_coding_interleaved_b200 as bs
    import synthetic as S
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = _Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    batch = a.batch
    specs_all, _, desc = _workload_desc(a.workload, a.layers)
    specs = [s for s in specs_all if not s.is_raw and len(s.shape) == 2]
    dense = [S.generate(s, dev).reshape(-1) for s in specs]
    built = [bs.fw_transcode(w) for w in dense]
    torch.cuda.synchronize()
    calls = _gemv_calls(specs)
    n_w = sum(rows * cols for c in calls for _, rows, cols in c)
    fw_bytes = sum(built[k][1].total_bytes for c in calls for k, _, _ in c)
    g = torch.Generator(device=dev).manual_seed(1234)
    xs, ys, yd, items = [], [], [], []
    for c in calls:
        cols = c[0][2]
        x = torch.randn(batch, cols, device=dev, generator=g).to(torch.bfloat16)
        xs.append(x)
        y = [torch.empty(batch, rows, dtype=torch.float32, device=dev) for _, rows, _ in c]
        ys.append(y)
        yd.append([torch.empty(batch, rows, dtype=torch.bfloat16, device=dev) for _, rows, _ in c])
        items.append([(built[k][0], built[k][1], rows, cols, x.view(torch.int16), yy) for (k, rows, _), yy in zip(c, y)])
    xy_bytes = sum(2 * batch * c[0][2] + 4 * batch * sum(r for _, r, _ in c) for c in calls)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    # batches 1..4 go to the CUDA cores (bs_fw_gemv), larger ones to the tensor cores
    # (bs_fw_gemm): on the 9B pass the CUDA-core product takes 4.4 / 5.6 / 6.5 / 7.7 ms at
    # batch 1 / 2 / 3 / 4 and 15 ms at 8, the tensor-core one about 8.7 ms at any batch up to 16
    tensor = a.product == "tensor" or (a.product == "auto" and batch > 4)
    if not tensor and batch > 8:
        raise SystemExit("bench: the CUDA-core product takes batches of 1..8")
    # the layouts are written once, before the pass, and stay resident: the CUDA-core product
    # may start copying them while the kernel before it finishes
    product = bs.fw_gemm if tensor else functools.partial(bs.fw_gemv, layouts_resident=True)
    kernel = "fw_gemm_kernel" if tensor else "fw_gemv_kernel"
    if tensor and any(rows % 128 for c in calls for _, rows, _ in c):
        raise SystemExit("bench: the tensor-core product needs rows in multiples of 128")

    def fused_pass():
        for it in items:
            product(it, err, stream=torch.cuda.current_stream())

    def dense_pass():
        for c, x, yy in zip(calls, xs, yd):
            for (k, rows, cols), y in zip(c, yy):
                torch.matmul(x, dense[k].view(torch.bfloat16).view(rows, cols).t(), out=y)

    # parity before timing: every product against a float64 product of the originals on the
    # device, within 2 * K * 2^-24 * (sum |w x| + 64 max|x|) per output (escapes included)
    fused_pass()
    torch.cuda.synchronize()
    worst = 0.0
    for c, x, yy in zip(calls, xs, ys):
        xf = x.double()
        for (k, rows, cols), y in zip(c, yy):
            wf = dense[k].view(torch.bfloat16).view(rows, cols).double()
            ref = xf @ wf.t()
            tol = (4.0 if tensor else 2.0) * cols * 2.0 ** -24 * (xf.abs() @ wf.abs().t() + 64.0 * xf.abs().max())
            worst = max(worst, float(((y.double() - ref).abs() / tol).max()))
    if int(err.item()) != 0 or not worst <= 1.0:
        raise SystemExit(f"bench: fused GEMV out of tolerance (worst {worst:.3g} of the bound) or error flag set")

    def graph_of(fn):
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for _ in range(max(1, a.warmup)):
                fn()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        torch.cuda.synchronize()
        return gr

    l0 = bs.launch_counter()
    g_fused = graph_of(fused_pass)
    launches_per_pass = (bs.launch_counter() - l0) // (max(1, a.warmup) + 1)
    g_dense = graph_of(dense_pass)

    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    smi_index = phys[local] if local < len(phys) and phys[local].strip().isdigit() else str(local)
    clocks = _Clocks(smi_index)
    time.sleep(0.3)
    ms_fused = ranks.max(_timed(stream, a.steps, g_fused.replay, ranks.barrier))
    clk = clocks.stop()
    ms_dense = ranks.max(_timed(stream, a.steps, g_dense.replay, ranks.barrier))
    if int(err.item()) != 0:
        raise SystemExit("bench: fused GEMV raised its error flag")
    step_ms = ms_fused / a.steps
    value = world * a.steps * 2 * n_w / (ms_fused * 1e-3) / 1e9
    peak, peak_kind = _peak_hbm()
    achieved = (fw_bytes + xy_bytes) / (step_ms * 1e-3) / 1e9

    # end to end: x in from pinned host memory and y back out, per call, inside the timed region
    e2e = None
    if not a.no_e2e and a.e2e_steps > 0:
        hx = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True).copy_(x) for x in xs]
        hy = [[torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in yy] for yy in ys]

        def e2e_pass():
            for it, x, h, yy, hh in zip(items, xs, hx, ys, hy):
                x.copy_(h, non_blocking=True)
                product(it, err, stream=torch.cuda.current_stream())
                for y, hy1 in zip(yy, hh):
                    hy1.copy_(y, non_blocking=True)

        e_ms = ranks.max(_timed(stream, a.e2e_steps, e2e_pass, ranks.barrier))
        e2e = {"value": round(world * a.e2e_steps * 2 * n_w / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(sum(x.numel() * 2 for x in xs)),
               "d2h_bytes_per_step": int(sum(y.numel() * 4 for yy in ys for y in yy)), "steps": a.e2e_steps,
               "path": "per call: x copied in from pinned host memory, bs_fw_gemv, y copied back; "
                       "the layouts stay resident (the weights of a served model)"}

    cpu = None
    if rank == 0 and not a.no_cpu_baseline:
        import numpy as np
        import oracle
        c = calls[0]
        k, rows, cols = c[0]
        w = dense[k].cpu().numpy().view(np.uint16)
        blob = oracle.fw_encode(w)
        x = xs[0].view(torch.int16).cpu().numpy().view(np.uint16)
        t0 = time.perf_counter()
        oracle.fw_gemv(blob, rows, cols, x)
        sec = time.perf_counter() - t0
        cpu = {"value": round(2 * rows * cols / sec / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"oracle decode + float64 numpy product of {specs[k].name} ({rows} x {cols}), batch {batch}"}
    ranks.close()
    if rank != 0:
        return
    gemv_tpw = _traffic_per_weight("fw_gemv_kernel") if (not tensor and batch == 1) else None
    print(json.dumps({
        "metric": GEMV_METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded device draws, synthetic/ recipe)",
        "config": {"workload": a.workload, "description": desc, "batch": batch, "matrices": len(specs),
                   "product": ("tensor cores: W decoded tile by tile into shared memory, tcgen05.mma (bs_fw_gemm)"
                               if tensor else "CUDA cores: W decoded in registers, fp32 FMA (bs_fw_gemv)"),
                   "calls_per_step": len(calls), "n_weights": int(n_w), "fw_bytes": int(fw_bytes),
                   "bits_per_weight": round(8 * fw_bytes / n_w, 5),
                   "dense_cublas_ms_per_step": round(ms_dense / a.steps, 4),
                   "speedup_vs_dense": round(ms_dense / ms_fused, 4),
                   "graph": "each step replays one CUDA graph of the pass's calls",
                   "parity": f"every product within its fp32 bound before timing (worst {worst:.3g} of it)",
                   "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": "no flush: the layouts (GBs) are larger than L2"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": (None if gemv_tpw is None else int(gemv_tpw * n_w)),
                     "traffic_source": ("ncu capture of this kernel at batch 1 on one gate/up call, scaled by weights"
                                        if gemv_tpw is not None else None),
                     "kernel": kernel, "per_step_bytes": int(fw_bytes + xy_bytes),
                     "tflops": round(2.0 * n_w * batch / (step_ms * 1e-3) / 1e12, 2),
                     "launches_per_step": int(launches_per_pass)},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": int(launches_per_pass * a.steps), "clocks": clk}),
        flush=True)


def main():
    a = _args()
    if a.impl == "reference" and a.mode == "fw":
        run_fw_reference(a)
    elif a.impl == "reference":
        run_reference(a)
    elif a.mode == "fw":
        run_fw(a)
    elif a.mode == "gemv":
        run_gemv(a)
    elif a.mode == "layerwise":
        run_layerwise(a)
    elif a.mode == "stream":
        run_stream(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
