"""Host logic of bench.py's product pass (--mode gemv), on the CPU:
* the calls group the projections as a decoder step issues them: per layer (q, k, v) on one
  x, o, (gate, up) on one x, down, then the LM head; every matrix of the pass is in exactly
  one call, and the products of a call share their x (the same number of columns);
* the measured DRAM traffic of a kernel is reported only while its sources hash to the value
  recorded with the capture.
"""
import bench
import synthetic as S


def test_gemv_calls_follow_a_decoder_step():
    specs = [s for s in S.workload("gemma2_9b") if not s.is_raw and len(s.shape) == 2]
    calls = bench._gemv_calls(specs)
    assert len(calls) == 4 * 42 + 1                        # the 169 calls of the 9B pass
    seen = [k for c in calls for k, _, _ in c]
    assert sorted(seen) == list(range(len(specs)))         # every matrix once
    for c in calls:
        assert len({cols for _, _, cols in c}) == 1        # one x per call
        for k, rows, cols in c:
            assert rows * cols == specs[k].numel
    names = [[specs[k].name.split(".")[-1] for k, _, _ in c] for c in calls]
    assert names[:4] == [["q", "k", "v"], ["o"], ["gate", "up"], ["down"]]
    assert names[-1] == ["embed"]
    head = calls[-1][0]
    assert (head[1], head[2]) == (256000, 3584)            # the LM head: [vocab, hidden]


def test_traffic_is_reported_only_for_unchanged_sources(monkeypatch):
    files, _, tpw = bench._TRAFFIC["fw_gemv_kernel"]
    now = bench._source_hash(files)
    assert len(now) == 16
    monkeypatch.setitem(bench._TRAFFIC, "fw_gemv_kernel", (files, now, tpw))
    assert bench._traffic_per_weight("fw_gemv_kernel") == tpw
    monkeypatch.setitem(bench._TRAFFIC, "fw_gemv_kernel", (files, "0" * 16, tpw))
    assert bench._traffic_per_weight("fw_gemv_kernel") is None
    monkeypatch.setitem(bench._TRAFFIC, "fw_gemv_kernel", (files, None, None))
    assert bench._traffic_per_weight("fw_gemv_kernel") is None
