"""The multi-process side of bench.py on CPU (gloo, two ranks): every rank gets the max
of the per-rank timers, only rank 0 reports, the whole-job value counts every rank's
tokens over the slowest rank's time, a timed region slowed on one rank is timed once
more on every rank, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    r = bench.Ranks("gloo", device="cpu", timeout_s=60)
    got = r.max(10.0 * (rank + 1) + 0.25)
    r.barrier()
    q.put((rank, r.is_root, r.world, got, bench.job_value(r.world, 256, 100, got)))
    r.close()


def test_two_gloo_ranks_share_the_max_timer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    for rank, root, world, got, value in results:
        assert world == 2 and root == (rank == 0)
        assert got == 20.25
        assert value == pytest.approx(2 * 256 * 100 / 20.25e-3)


class _ScriptedSampler:
    """bench.Clocks stand-in: rank 1's first region saw a thermal slowdown."""
    calls = 0

    def __init__(self, dev):
        pass

    def start(self):
        pass

    def stop(self):
        _ScriptedSampler.calls += 1
        slowed = os.environ["RANK"] == "1" and _ScriptedSampler.calls == 1
        return {"reasons": ["hw_thermal_slowdown"] if slowed else []}


def _remeasure_worker(rank, world, port, q):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    r = bench.Ranks("gloo", device="cpu", timeout_s=60)
    runs = []
    out, clocks = bench.clocked(r, "cpu", lambda: runs.append(1) or len(runs), sampler=_ScriptedSampler)
    got = r.max(float(out))          # the ranks' collectives still pair up afterwards
    q.put((rank, len(runs), out, clocks.get("remeasured_after"), got))
    r.close()


def test_a_region_slowed_on_one_rank_is_timed_again_on_all():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_remeasure_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == [(0, 2, 2, [], 2.0), (1, 2, 2, ["hw_thermal_slowdown"], 2.0)]


def test_single_rank_is_a_no_op(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    r = bench.Ranks("gloo", device="cpu")
    assert r.world == 1 and r.is_root and r.max(3.5) == 3.5
    r.barrier()
    r.close()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import argparse
    import bench
    from block_diffusion_lm_masked_b200 import configs as CF
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=3, warmup=1, gpus=2)
    assert bench.run_reference(args, CF.CONFIGS["layer1_bf16"], "layer1_bf16") == 0
    assert capsys.readouterr().out == ""
