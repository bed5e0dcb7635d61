"""Expert-parallel pieces on one GPU ("MoE: what it costs to train and serve",
Expert parallelism and two all-to-alls, step 2).

moe_expert_ffn_multi runs a rank's N local experts on rows received from
n_src ranks, grouped source-major then by expert; group (s, e) uses weight
block e.  Checked against the oracle on synthetic groups (empty ones
included, on the one-CTA and the CTA-pair GEMM), and the whole expert-parallel
layer forward on a one-rank NCCL group against the oracle layer.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_warp_b200 as moe
from gpu_util import cfg_of, rel_l2, route_near_ties, to_f64, upload_inputs, y_tol

pytestmark = pytest.mark.gpu

MULTI = {
    # (workload of the local experts, n_src, rows per (source, expert))
    "bf16-swiglu-3src": (synth.Workload("m", T=1, d=128, N=4, k=1, H=192, act="swiglu",
                                        dtype="bf16", gate_mode="R", seed=70), 3,
                         [5, 0, 33, 129, 0, 17, 250, 1, 64, 0, 48, 140]),
    "f32-relu-2src": (synth.Workload("m", T=1, d=64, N=3, k=1, H=96, act="relu", dtype="f32",
                                     gate_mode="R", seed=71), 2, [7, 0, 30, 12, 41, 3]),
    "fp8-swiglu-2src": (synth.Workload("m", T=1, d=128, N=4, k=1, H=128, act="swiglu",
                                       dtype="bf16", gate_mode="R", dispatch="fp8", seed=72), 2,
                        [20, 90, 0, 150, 33, 0, 75, 10]),
    # >= 512 rows per group on average: the CTA-pair GEMM
    "bf16-pair-2src": (synth.Workload("m", T=1, d=128, N=2, k=1, H=256, act="swiglu",
                                      dtype="bf16", gate_mode="R", seed=73), 2,
                       [600, 530, 700, 290]),
}


@pytest.mark.parametrize("name", list(MULTI))
def test_expert_ffn_multi_source(name):
    base, n_src, counts = MULTI[name]
    counts = np.array(counts)
    R = int(counts.sum())
    wl = base.with_(T=R)                     # cfg.T * k bounds the rows (R here)
    host = synth.make_host(wl)
    dev, _ = upload_inputs(wl)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    fp8 = wl.dispatch == "fp8"
    if fp8:
        q, sc = oracle.quantize_rows(host["x"])
        xr, xs = torch.from_numpy(q).cuda(), torch.from_numpy(sc).cuda()
        xin = oracle.dequantize_rows(q, sc)
    else:
        xr, xs = dev["x"], None
        xin = oracle.decode(host["x"])
    y = torch.zeros((R, wl.d), dtype=dev["x"].dtype, device="cuda")
    moe.moe_expert_ffn_multi(cfg, n_src, R, xr, xs, torch.from_numpy(offsets).cuda(), dev["W1"],
                             dev.get("W3"), dev["W2"], y, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    got = to_f64(y)
    group = np.repeat(np.arange(n_src * wl.N), counts)
    want = np.empty((R, wl.d))
    for r in range(R):
        e = group[r] % wl.N
        want[r] = oracle.ffn_row(xin[r], host["W1"][e], host["W3"][e] if wl.act == "swiglu" else None,
                                 host["W2"][e], wl.act)
    tol = 1e-5 if wl.dtype == "f32" else 5e-3
    for g in range(n_src * wl.N):
        lo, hi = offsets[g], offsets[g + 1]
        if hi > lo:
            assert rel_l2(got[lo:hi], want[lo:hi]) <= tol, (g, "source", g // wl.N)


def test_expert_ffn_multi_rejects_bad_arguments():
    wl = synth.Workload("m", T=64, d=64, N=4, k=1, H=64, act="relu", dtype="bf16", gate_mode="R")
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    z = torch.zeros(8, dtype=torch.int32, device="cuda")
    for n_src, cap in [(0, 64), (257, 64), (2, 65)]:          # no source, > 1024 groups, > T*k rows
        with pytest.raises(moe.MoeError) as e:
            moe.moe_expert_ffn_multi(cfg, n_src, cap, z, None, z, z, None, z, z, ws)
        assert e.value.status == moe.MOE_ERR_INVALID_ARG
    fb = cfg_of(wl.with_(overflow="fallback", capacity_factor=1.0))
    with pytest.raises(moe.MoeError) as e:
        moe.moe_expert_ffn_multi(fb, 1, 0, None, None, None, None, None, None, None,
                                 moe.workspace(fb))
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_expert_parallel_layer_one_rank():
    import torch.distributed as dist
    from top_routing_expert_warp_b200 import ep
    wl = synth.MIXTRAL.with_(T=300, d=256, H=384, capacity_factor=0.9)
    dev, host = upload_inputs(wl)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        y, idx, gw = ep.ep_layer_forward(cfg_of(wl), dev["x"], dev["Wg"], None, dev["W1"],
                                         dev["W3"], dev["W2"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.route(wl, host["x"], host["Wg"])
    tie = route_near_ties(wl, ref)
    ok = np.all(idx.cpu().numpy() == ref["idx"], axis=1)
    assert np.all(ok | tie)
    flipped = set(ref["idx"][~ok].ravel().tolist())
    toks = np.where(~np.isin(ref["idx"], list(flipped)).any(axis=1))[0] if flipped else \
        np.arange(wl.T)
    want = oracle.forward_rows(wl, host, ref, toks)
    assert rel_l2(to_f64(y)[toks], want) <= y_tol(wl)
