"""The benchmark's multi-rank path on CPU with two gloo ranks.

The layer forward does not exchange data between GPUs: every rank runs its own
replica on its own tokens (weak scaling).  What is shared is the timing: the
job's step time is the max over ranks and the value counts every rank's tokens.
"""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(10.0 + 3.0 * rank, dist, "cpu")
    dist.barrier()
    q.put((rank, ms, bench.weak_value(4096, world, ms)))
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [13.0, 13.0]
    assert got[0][2] == pytest.approx(2 * 4096 / 13e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.weak_value(32, 1, 2.0) == pytest.approx(16000.0)


def test_reference_arm_on_a_nonzero_rank_exits_without_work(monkeypatch, capsys):
    import bench
    import synth
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup = 5, 3
    assert bench.run_reference(A, synth.MIXTRAL) == 0
    assert capsys.readouterr().out == ""


def test_algorithmic_bytes_count_the_fallback_expert():
    # the fallback expert's rows and weights enter the roofline like any expert's
    import numpy as np

    import bench
    import synth
    wl = synth.SWITCH_FALLBACK.with_(T=64, N=4, d=32, H=48)
    kept = np.array([16, 16, 0, 10])
    plain = bench.algorithmic(wl, kept)
    fb = bench.algorithmic(wl, np.append(kept, 22))     # 22 pairs over capacity
    es = 2
    assert fb["touched"] == plain["touched"] + 1 and fb["R"] == plain["R"] + 22
    assert fb["bytes"] - plain["bytes"] == 2 * wl.d * wl.H * es     # W1 and W2 (ReLU)
    assert fb["flops"] - plain["flops"] == 22 * 2.0 * 2 * wl.d * wl.H
