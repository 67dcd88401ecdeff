"""The multi-rank side of bench.py, on CPU: two gloo ranks exercise the barrier and the max of
the ranks' times. The bench runs N independent replicas (one per GPU). The decode has no
exchange step, so these are its only collectives. Also checks that the reference arm
leaves all work to rank 0."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json
sys.path.insert(0, {root!r})
import bench
r = bench._Ranks("gloo", None, timeout_s=60)
r.barrier()
m = r.max(10.0 * r.rank + 5.0)
r.barrier()
print(json.dumps({{"rank": r.rank, "world": r.world, "max": m}}))
r.close()
'''


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_and_barrier():
    port = _free_port()
    code = WORKER.format(root=ROOT)
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                   LOCAL_RANK=str(rank))
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(out.strip().splitlines()[-1])
    import json
    got = sorted((json.loads(o) for o in outs), key=lambda d: d["rank"])
    assert [d["rank"] for d in got] == [0, 1]
    assert all(d["world"] == 2 and d["max"] == 15.0 for d in got)


def test_single_rank_is_a_no_op(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    r = bench._Ranks("gloo")
    r.barrier()
    assert (r.world, r.rank, r.max(3.5)) == (1, 0, 3.5)
    r.close()


def test_reference_arm_leaves_other_ranks_idle(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "_oracle_sample", lambda *a, **k: called.append(1))
    args = type("A", (), dict(cpu_threads=1, workload="tensor_1m", layers=None, warmup=1, steps=1, gpus=2))()
    bench.run_reference(args)
    assert called == [] and capsys.readouterr().out == ""
