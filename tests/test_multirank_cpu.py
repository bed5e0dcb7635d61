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


def test_clock_summary_keeps_the_timed_region_and_every_reason():
    # host-only: samples stamped outside [t0 - 0.06, t1 + 0.06] are dropped, every
    # reason seen active inside is reported with the raw masks, and the bench's
    # up_kernel names the kernel each workload's up-projection runs on
    import datetime
    import bench
    import synth
    c = bench.Clocks.__new__(bench.Clocks)
    c.names = list(bench.Clocks.NAMES)
    t0 = 1.0e9
    def line(t, mhz, mask, active):
        ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        flags = ["Active" if n in active else "Not Active" for n in c.names]
        return ", ".join([ts, str(mhz), "1965", "500.0", mask] + flags)
    c.out = "\n".join([line(t0 - 1.0, 900, "0x8", {"hw_slowdown"}),        # before: dropped
                       line(t0 + 0.1, 1500, "0x4", {"sw_power_cap"}),
                       line(t0 + 0.2, 1700, "0x0", set()),
                       line(t0 + 5.0, 800, "0x40", {"sw_thermal_slowdown"})])  # after: dropped
    s = c.summary(t0, t0 + 0.3)
    assert s["samples"] == 2 and s["sm_min_mhz"] == 1500 and s["sm_mhz"] == 1600
    assert s["reasons"] == ["sw_power_cap"] and s["active_masks"] == ["0x0", "0x4"]
    assert c.summary()["samples"] == 4
    assert bench.up_kernel(synth.DEEPSEEK)[0] == "grouped_gemm_tc_pairt"
    assert bench.up_kernel(synth.MIXTRAL)[0] == "grouped_gemm_tc_pair"
    assert bench.up_kernel(synth.SWITCH_FALLBACK)[0] == "grouped_gemm_tc"
    assert bench.up_kernel(synth.TINY_F32)[0] == "layer_small_f32"
