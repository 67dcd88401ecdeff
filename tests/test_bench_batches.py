"""Host logic of bench.py's batch partition (--batch-gb): the checkpoint's chunks cut into
batches of at most a given output size and one wave of the decode kernel, for
Plan.decode_ranges. Checked on the CPU with the 27B-scale workload's tensor list and a
fake plan that reports a decode geometry:
* every element of every tensor is in exactly one range, and each range's output view is
  the matching slice of the tensor's output;
* coded ranges start on chunk boundaries and, unless they end their tensor, cover a whole
  number of CTAs' worth of chunks;
* no batch exceeds the output cap or one wave of CTAs.
"""
import pytest
import torch

import bench
import synthetic as S

bs = pytest.importorskip("lossless_entropy_coding_interleaved_b200")


class _FakePlan:
    def __init__(self, cpc, wave):
        self.cpc, self.wave = cpc, wave

    def decode_geometry(self, idx):
        return self.cpc, self.wave


def _infos(specs, log2_chunk=16):
    out = []
    for s in specs:
        if s.is_raw:
            out.append(dict(n_elems=s.numel, kind=bs.KIND_RAW, log2_chunk=0))
        elif s.numel <= 4097:
            out.append(dict(n_elems=s.numel, kind=bs.KIND_STORED, log2_chunk=0))
        else:
            out.append(dict(n_elems=s.numel, kind=bs.KIND_JOINT, log2_chunk=log2_chunk))
    return out


@pytest.mark.parametrize("cpc,wave,gb", [(56, 148, 1.0), (48, 148, 1.0), (48, 132, 0.25), (40, 148, 4.0)])
def test_partition_of_a_27b_layer_and_embedding(cpc, wave, gb):
    specs = S.workload("qwen_27b_scale", layers=2)
    specs = specs[:9] + specs[-1:] + [s for s in S.workload("edge_mix") if s.name in ("one", "ragged", "raw_span")]
    infos = _infos(specs)
    outs = [torch.empty(i["n_elems"], dtype=torch.uint8 if i["kind"] == bs.KIND_RAW else torch.int16)
            for i in infos]
    batches = bench._chunk_batches(_FakePlan(cpc, wave), infos, outs, gb)
    seen = {k: [] for k in range(len(infos))}
    for b in batches:
        assert b
        ctas = out_bytes = 0
        for k, beg, cnt, view in b:
            i = infos[k]
            per = 1 if i["kind"] == bs.KIND_RAW else 2
            assert view.numel() == cnt
            assert view.data_ptr() == outs[k].data_ptr() + per * beg
            if i["kind"] == bs.KIND_JOINT:
                C = 1 << i["log2_chunk"]
                chunks = -(-cnt // C)
                assert beg % C == 0
                if beg + cnt != i["n_elems"]:
                    assert cnt % C == 0 and chunks % cpc == 0
                ctas += -(-chunks // cpc)
            out_bytes += per * cnt
            seen[k].append((beg, cnt))
        assert ctas <= wave
        assert out_bytes <= gb * 1e9
    for k, i in enumerate(infos):
        pos = 0
        for beg, cnt in sorted(seen[k]):
            assert beg == pos
            pos += cnt
        assert pos == i["n_elems"], specs[k].name


def test_one_batch_per_wave_when_the_cap_is_loose():
    # tensors of exactly one wave's chunks each: one batch per tensor
    cpc, wave, C = 48, 148, 1 << 16
    infos = [dict(n_elems=cpc * wave * C, kind=bs.KIND_JOINT, log2_chunk=16) for _ in range(3)]
    outs = [torch.empty(1, dtype=torch.int16).expand(i["n_elems"]) for i in infos]
    batches = bench._chunk_batches(_FakePlan(cpc, wave), infos, outs, 100.0)
    assert [[(k, b, c) for k, b, c, _ in bb] for bb in batches] == [[(k, 0, cpc * wave * C)] for k in range(3)]
