"""Expert-parallel exchange on CPU with gloo ranks ("MoE: what it costs to
train and serve", Expert parallelism and two all-to-alls).

Each rank routes its own tokens (oracle), sends its expert-ordered rows to the
ranks owning the experts through the library's planner and all-to-alls, the
owners run their experts on what they received (oracle FFN, weight block =
local expert of the group), the outputs go back and are combined.  The result
must equal the single-process oracle layer on every rank's tokens, for
2 and 4 ranks, with and without capacity dropping.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, cf, q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from top_routing_expert_warp_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, k, d, H = 8, 2, 16, 24
        base = synth.Workload("ep", T=40 + 7 * rank, d=d, N=N, k=k, H=H, act="swiglu",
                              dtype="f32", gate_mode="R", capacity_factor=cf, seed=60)
        wl = base.with_(seed=60)                       # same weights on every rank
        host = synth.make_host(wl)
        # this rank's tokens: a seed of its own
        x = synth.normal(100 + rank, 0, wl.T * d, 1.0, "f32").reshape(wl.T, d)
        host = dict(host, x=x)
        ref = oracle.route(wl, x, host["Wg"])
        R = ref["R"]
        x_perm = oracle.decode(x)[ref["perm"] // k]            # [R, d] expert-ordered rows
        plan = ep.exchange_counts(ep.send_counts_of(ref["offsets"], world))
        recv = ep.exchange_rows(torch.from_numpy(x_perm), plan).numpy()
        # the experts this rank owns, on the rows every rank sent it
        E = N // world
        off = plan.recv_offsets()
        y_recv = np.zeros_like(recv)
        for g in range(world * E):
            e = rank * E + g % E
            for r in range(off[g], off[g + 1]):
                y_recv[r] = oracle.ffn_row(recv[r], host["W1"][e], host["W3"][e], host["W2"][e],
                                           "swiglu")
        y_back = ep.return_rows(torch.from_numpy(y_recv), plan).numpy()
        assert y_back.shape[0] == R
        y = oracle.combine(y_back, ref["inv_row"], ref["gate"])
        want = oracle.forward_rows(wl, host, ref, np.arange(wl.T))
        err = float(np.abs(y - want).max())
        q.put((rank, err, plan.send_rows, plan.recv_rows, int(ref["drop"].sum())))
    except Exception as e:               # report, so the parent does not wait for good
        q.put((rank, repr(e), None, None, None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cf", [(2, 0.0), (2, 0.6), (4, 0.0), (4, 0.7)])
def test_expert_parallel_exchange_matches_single_process(world, cf):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cf, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, sent, recv, dropped in got:
        assert not isinstance(err, str), err
        assert err < 1e-12, (rank, err)
    # every row sent is received once: the matrix of sends is the transpose of receives
    sends = np.array([g[2] for g in got])
    recvs = np.array([g[3] for g in got])
    assert np.array_equal(sends, recvs.T)
    if cf > 0:
        assert sum(g[4] for g in got) > 0      # capacity dropped some pairs


def test_send_plan_from_expert_offsets():
    from top_routing_expert_warp_b200 import ep
    # 6 experts on 3 ranks (2 each); expert e has e + 1 rows, except expert 4 (none)
    rows = np.array([1, 2, 3, 4, 0, 6])
    offsets = np.concatenate([[0], np.cumsum(rows)])
    sc = ep.send_counts_of(offsets, 3)
    assert sc.tolist() == [[1, 2], [3, 4], [0, 6]]
    with pytest.raises(ValueError):
        ep.send_counts_of(offsets, 4)            # 6 experts do not split over 4 ranks
    # what rank r receives: row r of every source's send counts
    recv = np.array([[5, 0], [1, 1], [2, 7]])
    plan = ep.SendPlan(send_counts=sc, recv_counts=recv)
    assert plan.send_rows == [3, 7, 6] and plan.recv_rows == [5, 2, 9]
    # received rows: source-major, then by local expert
    assert plan.recv_offsets().tolist() == [0, 5, 5, 6, 7, 9, 16]


def test_expert_parallel_rejects_fallback_expert():
    """The exchange covers offsets[0..N]; a fallback expert's rows would be
    lost, so the layer refuses such a configuration before any launch."""
    import top_routing_expert_warp_b200 as moe
    from top_routing_expert_warp_b200 import ep
    cfg = moe.make_config(64, 64, 8, 2, 128, capacity_factor=1.0, overflow="fallback")
    with pytest.raises(ValueError, match="fallback"):
        ep.ep_layer_forward(cfg, None, None, None, None, None, None)
