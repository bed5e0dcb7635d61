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


def _layer_worker(rank, world, port, cap_rank0, q):
    """ExpertParallelLayer end to end on gloo ranks, its kernels replaced by
    oracle computations on CPU tensors (the planning, the agreement on the
    receive capacity, the exchanges into the preallocated buffers and their
    reuse are the layer's own)."""
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    import top_routing_expert_warp_b200 as moe
    from top_routing_expert_warp_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, k, d, H, T = 8, 2, 16, 24, 30 + 5 * rank
        wl = synth.Workload("ep-layer", T=T, d=d, N=N, k=k, H=H, act="swiglu", dtype="f32",
                            gate_mode="R", capacity_factor=0.8, seed=61)
        host = synth.make_host(wl)
        E = N // world

        def router(cfg, x, Wg, bias, logits, idx, gw, pm, ws, s):
            r = oracle.route(wl.with_(T=cfg.T), x.numpy(), Wg.numpy())
            idx.copy_(torch.from_numpy(r["idx"]))
            gw.copy_(torch.from_numpy(r["gate"].astype(np.float32)))

        def dispatch(cfg, x, idx, counts, offsets, perm, inv_row, drop, x_perm, xs, pm, f, aux,
                     ws, s):
            r = oracle.dispatch(idx.numpy(), cfg.N, cfg.capacity_factor)
            counts.copy_(torch.from_numpy(r["counts"]))
            offsets[:N + 1].copy_(torch.from_numpy(r["offsets"]))
            perm[:r["R"]].copy_(torch.from_numpy(r["perm"]))
            inv_row.copy_(torch.from_numpy(r["inv_row"]))
            drop.copy_(torch.from_numpy(r["drop"]))
            x_perm[:r["R"]].copy_(x[torch.from_numpy(r["perm"] // cfg.k).long()])

        def ffn_multi(cfg_e, P, cap, x_rows, s_rows, off, W1, W3, W2, y_rows, ws, s):
            o = off.numpy()
            for g in range(P * cfg_e.N):
                e = g % cfg_e.N
                for r in range(o[g], o[g + 1]):
                    y_rows[r] = torch.from_numpy(oracle.ffn_row(
                        x_rows[r].double().numpy(), W1[e].numpy(), W3[e].numpy(), W2[e].numpy(),
                        "swiglu").astype(np.float32))

        def combine(cfg, y_perm, inv_row, gw, ysh, y, ws, s):
            y.copy_(torch.from_numpy(oracle.combine(y_perm.double().numpy(), inv_row.numpy(),
                                                    gw.double().numpy()).astype(np.float32)))

        ep.moe_router, ep.moe_dispatch = router, dispatch
        ep.moe_expert_ffn_multi, ep.moe_combine = ffn_multi, combine
        cfg = moe.config_from(wl.with_(T=T))
        mine = slice(rank * E, (rank + 1) * E)
        W = [torch.from_numpy(host[n][mine].copy()) for n in ("W1", "W3", "W2")]
        Wg = torch.from_numpy(host["Wg"])
        cap = cap_rank0 if rank == 0 else None
        layer = ep.ExpertParallelLayer(cfg, recv_capacity=cap, device="cpu")
        errs, ptrs = [], []
        for call in range(2):
            x = synth.normal(200 + 10 * rank + call, 0, T * d, 1.0, "f32").reshape(T, d)
            try:
                y, idx, gw = layer.forward(torch.from_numpy(x), Wg, None, *W)
            except ValueError as e:
                q.put((rank, "overflow", str(e)))
                return
            ref = oracle.route(wl.with_(T=T), x, host["Wg"])
            want = oracle.forward_rows(wl.with_(T=T), dict(host, x=x), ref, np.arange(T))
            errs.append(float(np.abs(y.double().numpy() - want).max() / np.abs(want).max()))
            ptrs.append((y.data_ptr(), layer.x_rows.data_ptr(), layer.y_perm.data_ptr()))
        q.put((rank, "ok", (max(errs), ptrs[0] == ptrs[1])))
    except Exception as e:               # report, so the parent does not wait for good
        q.put((rank, "error", repr(e)))
    finally:
        dist.destroy_process_group()


def _run_layer_ranks(world, cap_rank0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_layer_worker, args=(r, world, port, cap_rank0, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


def test_expert_parallel_layer_object_two_ranks_reuses_buffers():
    got = _run_layer_ranks(2, None)
    for rank, what, detail in got:
        assert what == "ok", (rank, what, detail)
        err, same_buffers = detail
        assert err < 1e-5, (rank, err)          # fp32 rows through the exchange
        assert same_buffers, rank               # the second call reused every buffer


def test_expert_parallel_receive_overflow_raises_on_every_rank():
    # rank 0 can hold 3 received rows: every rank learns it before any row moves
    got = _run_layer_ranks(2, 3)
    assert [w for _, w, _ in got] == ["overflow", "overflow"], got
