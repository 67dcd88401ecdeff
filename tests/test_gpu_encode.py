"""GPU encoder parity, and full-size decode parity in the bench's launch configuration.

* The device encoder must write the same bytes as the oracle encoder (the container fixes
  every encoder choice with integer rules), and the oracle must decode them back to the
  originals.
* At full size (the 9B-shaped checkpoint and full-shape 27B-scale layers), every decoded
  tensor is compared bit-exact with its regenerated original on the device. Sampled chunks
  are also decoded by the oracle from a host copy of the same container.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S

pytestmark = pytest.mark.gpu

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


def _gpu_items(specs, device="cuda:0"):
    cpu = [S.generate(s, "cpu") for s in specs]
    return cpu, [(s.name, t.to(device)) for s, t in zip(specs, cpu)]


def _host_items(specs, cpu):
    return [(s.name, S.words_numpy(t), "raw" if s.is_raw else "bf16") for s, t in zip(specs, cpu)]


@pytest.mark.parametrize("name,kw", [("tensor_1m", {}), ("edge_mix", {}), ("edge_mix", {"force_rans": True}),
                                     ("gemma2_layer", {})])
def test_device_encoder_matches_oracle_bytes(name, kw):
    specs = S.workload(name)
    cpu, dev = _gpu_items(specs)
    d_c, h_c = bs.encode(dev, host_copy=True, **kw)
    want = oracle.encode(_host_items(specs, cpu), **kw)
    assert h_c.size == len(want)
    assert bytes(h_c.tobytes()) == want
    assert torch.equal(d_c.cpu(), torch.from_numpy(h_c))


@pytest.mark.parametrize("log2_chunk,ns,nh,max_routes", [(8, 11, 5, 7), (12, 9, 3, 2), (17, 12, 4, 15),
                                                         (16, 12, 4, 0)])
def test_device_encoder_parameters(log2_chunk, ns, nh, max_routes):
    specs = S.workload("edge_mix")[:2] + S.workload("tensor_1m")
    cpu, dev = _gpu_items(specs)
    kw = dict(log2_chunk=log2_chunk, ns=ns, nh=nh, max_routes=max_routes)
    _, h_c = bs.encode(dev, host_copy=True, **kw)
    assert bytes(h_c.tobytes()) == oracle.encode(_host_items(specs, cpu), **kw)
    for k, t in enumerate(cpu):
        assert np.array_equal(oracle.decode(h_c, k), S.words_numpy(t))


def test_device_encoder_sizes():
    rng = np.random.default_rng(5)
    sizes = [0, 1, 2, 7, 8, 255, 256, 257, 1000, 4097, 65535, 65536, 65537]
    arrs = []
    for n in sizes:
        x = (rng.standard_normal(n) * 0.02).astype(np.float32)
        arrs.append((x.view(np.uint32) >> 16).astype(np.uint16))
    dev = [(f"n{n}", torch.from_numpy(a.view(np.int16)).cuda()) for n, a in zip(sizes, arrs)]
    for force in (False, True):
        _, h_c = bs.encode(dev, host_copy=True, force_rans=force)
        assert bytes(h_c.tobytes()) == oracle.encode([(f"n{n}", a, "bf16") for n, a in zip(sizes, arrs)],
                                                     force_rans=force)


def test_plan_from_device_container():
    specs = S.workload("edge_mix")
    cpu, dev = _gpu_items(specs)
    d_c, _ = bs.encode(dev)
    plan = bs.Plan(d_container=d_c)                    # metadata read from the device
    outs = plan.decode_batch(range(len(specs)))
    plan.check()
    for k, (s, t) in enumerate(zip(specs, dev)):
        assert torch.equal(outs[k].view(-1), t[1].reshape(-1)), s.name


def _widest_shape(chunks: int, sms: int, max_warps: int) -> bool:
    """True when a launch of `chunks` chunks takes the largest CTA shape (max_warps warps of two
    chunks each) rather than the per-launch shape read from the parameters: the planner picks
    ceil(ceil(chunks / sms) / 2) warps, capped at max_warps."""
    per_sm = -(-chunks // sms)
    return -(-per_sm // 2) >= max_warps


def _full_size_check(specs, model, sample_chunks=3):
    """Generate on the device, encode with `model`, decode in one batch, compare everything
    bit-exact, then oracle-decode sampled chunks (both coded kinds) from a host copy."""
    dev = [(s.name, S.generate(s, "cuda:0")) for s in specs]
    d_c, h_c = bs.encode(dev, host_copy=True, model=model)
    plan = bs.Plan(d_container=d_c)
    outs = plan.decode_batch(range(len(specs)))
    plan.check()
    n = coded = 0
    coded_chunks = {bs.KIND_RANS: 0, bs.KIND_JOINT: 0}
    for k, (s, (_, t)) in enumerate(zip(specs, dev)):
        assert torch.equal(outs[k].view(-1), t.view(-1)), s.name
        i = plan.info(k)
        n += i["n_elems"]
        coded += i["coded_bytes"]
        if i["kind"] in coded_chunks:
            coded_chunks[i["kind"]] += i["n_chunks"]
    rng = np.random.default_rng(0)
    coded_idx = [k for k in range(len(specs)) if plan.info(k)["kind"] in (bs.KIND_RANS, bs.KIND_JOINT)]
    for k in rng.choice(coded_idx, size=min(4, len(coded_idx)), replace=False):
        i = plan.info(int(k))
        whole = np.zeros(i["n_elems"], np.uint16)
        chunks = rng.choice(i["n_chunks"], size=min(sample_chunks, i["n_chunks"]), replace=False)
        gpu = S.words_numpy(outs[int(k)]).reshape(-1)
        C = 1 << i["log2_chunk"]
        for c in chunks:
            assert oracle.decode_chunks(h_c, int(k), int(c), int(c) + 1, whole) == 0
            lo, hi = int(c) * C, min((int(c) + 1) * C, i["n_elems"])
            assert np.array_equal(whole[lo:hi], gpu[lo:hi])
    del outs, dev, plan, d_c
    torch.cuda.empty_cache()
    return n, coded, coded_chunks


@pytest.mark.parametrize("model", ["factored", "joint"])
def test_full_gemma2_9b_checkpoint(model):
    # the bench's workload and launch: every tensor of the checkpoint in one bs_decode_batch
    n, coded, chunks = _full_size_check(S.workload("gemma2_9b"), model)
    assert n == 9_241_702_400
    assert coded * 8 / n < 10.6
    kind, widest = (bs.KIND_JOINT, 28) if model == "joint" else (bs.KIND_RANS, 24)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # nearly every BF16 tensor is coded with this kind, and the launch takes the widest CTA
    # shape (the compile-time instance the bench times)
    assert chunks[kind] > 0.99 * sum(chunks.values())
    assert _widest_shape(chunks[kind], sms, widest)


@pytest.mark.parametrize("model", ["factored", "joint"])
def test_full_shape_qwen27b_layers(model):
    # two full-shape layers and the full embedding of the 27B-scale checkpoint
    specs = S.workload("qwen_27b_scale", layers=2) + [S.workload("qwen_27b_scale")[-1]]
    _full_size_check(specs, model)


@pytest.mark.parametrize("model", ["factored", "joint"])
def test_every_tensor_of_the_27b_scale_checkpoint(model):
    # all 64 layers and the embedding, each layer encoded and decoded as its own container
    specs = S.workload("qwen_27b_scale")
    layers = {}
    for s in specs:
        layers.setdefault(s.name.split(".")[1] if s.name.startswith("layers.") else "embed", []).append(s)
    n = coded = 0
    for key, group in layers.items():
        dev = [(s.name, S.generate(s, "cuda:0")) for s in group]
        d_c, _ = bs.encode(dev, model=model)
        plan = bs.Plan(d_container=d_c)
        outs = plan.decode_batch(range(len(group)))
        plan.check()
        for k, (s, (_, t)) in enumerate(zip(group, dev)):
            assert torch.equal(outs[k].view(-1), t.view(-1)), s.name
            n += plan.info(k)["n_elems"]
            coded += plan.info(k)["coded_bytes"]
        del dev, outs, plan, d_c
    torch.cuda.empty_cache()
    assert n == 30_642_012_160
    assert coded * 8 / n < 10.7


@pytest.mark.parametrize("model,widest", [("factored", 24), ("joint", 28)])
def test_widest_cta_shape_against_the_oracle(model, widest):
    """The compile-time CTA shape of each coded kind, compared element by element with the
    oracle's decode. Chunks of 1,024 weights make a few million weights enough for the launch
    to take the widest shape: a ragged 8.4M-weight tensor plus small tensors of other
    lengths, all in one bs_decode_batch."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(17)
    sizes = [sms * 56 * 1024 + 777, 1, 255, 1024, 3000, 65537]
    arrs = []
    for k, n in enumerate(sizes):
        x = torch.from_numpy((rng.standard_normal(n) * (0.01 + 0.01 * k)).astype(np.float32))
        arrs.append(x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    c = oracle.encode([(f"t{k}", a, "bf16") for k, a in enumerate(arrs)], log2_chunk=10, model=model)
    kind = bs.KIND_JOINT if model == "joint" else bs.KIND_RANS
    total = sum(oracle.info(c, k)["n_chunks"] for k in range(len(arrs)) if oracle.info(c, k)["kind"] == kind)
    assert oracle.info(c, 0)["kind"] == kind and _widest_shape(total, sms, widest)
    plan = bs.Plan(c, device="cuda:0")
    outs = plan.decode_batch(range(len(arrs)))
    plan.check()
    for k, a in enumerate(arrs):
        got = S.words_numpy(outs[k]).reshape(-1)
        assert np.array_equal(got, a), k
        assert np.array_equal(got, oracle.decode(c, k).reshape(-1)), k
