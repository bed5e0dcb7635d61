"""Node-limited routing on the GPU against the oracle.

"MoE: what it costs to train and serve", Limit how many machines a token
touches: a token may use at most topk_groups of n_groups nodes (blocks of
N / n_groups consecutive experts), chosen by the sum of each node's
ceil(k / topk_groups) highest router probabilities; the top-k is taken among
the chosen nodes' experts.  Routing is compared exactly except on tokens whose
choice is a near-tie, either between nodes (the topk_groups-th and next node
scores) or between experts of the chosen nodes (the k-th and next logits).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_warp_b200 as moe
from gpu_util import LayerRun, cfg_of, rel_l2, route_near_ties, to_f64, upload_inputs, y_tol

pytestmark = pytest.mark.gpu

BASE = synth.Workload("nl", T=300, d=256, N=256, k=8, H=128, act="swiglu", dtype="bf16",
                      gate_mode="F", renormalize=True, n_groups=8, topk_groups=4, seed=40)
CASES = {
    # DeepSeek-V3-like: 8 nodes of 32 experts, at most 4 per token, top-8
    "n256-g8-m4-k8-renormF": BASE,
    # nodes smaller than a warp's lane row (8 experts per node), mode R
    "n64-g8-m3-k4-R": BASE.with_(N=64, k=4, d=128, gate_mode="R", renormalize=False,
                                 topk_groups=3, seed=41),
    # one node of three allowed, 32 experts per node
    "n96-g3-m1-k2-renormF": BASE.with_(N=96, k=2, n_groups=3, topk_groups=1, seed=42),
    # fp32 layer (CUDA-core router, N <= 16)
    "f32-n16-g4-m2-k4-R": BASE.with_(N=16, k=4, d=64, dtype="f32", gate_mode="R",
                                     renormalize=False, n_groups=4, topk_groups=2, seed=43),
}


@pytest.mark.parametrize("name", list(CASES))
def test_node_limited_router_parity(name):
    wl = CASES[name]
    dev, host = upload_inputs(wl)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    T, k, N = wl.T, wl.k, wl.N
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    pm = torch.empty(N, dtype=torch.float32, device="cuda")
    moe.moe_router(cfg, dev["x"], dev["Wg"], dev.get("bias"), None, idx, w, pm, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    ref = oracle.route(wl, host["x"], host["Wg"], host.get("bias"))
    # the limit binds: the plain top-k would span more nodes for some tokens
    plain, _, _ = oracle.topk_gate(ref["logits"], k, wl.gate_mode, wl.renormalize)
    S = N // wl.n_groups
    assert np.mean([len(set(r)) > wl.topk_groups for r in (plain // S).tolist()]) > 0.05
    tie = route_near_ties(wl, ref)
    ok = ~tie
    assert ok.mean() > 0.9
    gi = idx.cpu().numpy()
    assert np.array_equal(gi[ok], ref["idx"][ok]), "expert indices differ off near-ties"
    assert all(len(set(r)) <= wl.topk_groups for r in (gi // S).tolist())
    gw = w.cpu().numpy().astype(np.float64)
    relw = np.abs(gw[ok] - ref["gate"][ok]) / np.abs(ref["gate"][ok])
    assert relw.max() <= 1e-6, f"gate rel err {relw.max():.3g}"
    np.testing.assert_allclose(pm.cpu().numpy(), ref["p_mean"], rtol=1e-5, atol=1e-9)


def test_node_limited_layer_parity():
    wl = synth.DEEPSEEK_NODE_LIMITED.with_(T=200, d=256, H=128, H_shared=128)
    dev, host = upload_inputs(wl)
    run = LayerRun(wl, dev)
    run()
    assert run.check_status()[0] == moe.MOE_OK
    ref = oracle.route(wl, host["x"], host["Wg"], host.get("bias"))
    tie = route_near_ties(wl, ref)
    toks = np.where(~tie)[0]
    assert np.array_equal(run.topk_idx.cpu().numpy()[toks], ref["idx"][toks])
    want = oracle.forward_rows(wl, host, ref, toks)
    assert rel_l2(to_f64(run.y)[toks], want) <= y_tol(wl)


def test_node_limited_config_checks():
    ok = dict(T=64, d=128, N=64, k=4, H=128, dtype="bf16", gate_mode="R", n_groups=8, topk_groups=2)
    assert moe.moe_workspace_bytes(moe.make_config(**{**ok, "T": ok["T"]})) > 0
    # N not a multiple of the node count, more than 32 nodes, too few experts allowed
    for bad in ({"n_groups": 7}, {"N": 128, "n_groups": 64}, {"k": 8, "topk_groups": 1, "n_groups": 16}):
        cfg = moe.make_config(**{**ok, **bad})
        assert moe.moe_workspace_bytes(cfg) == 0, bad
    # plain mode F with nodes is refused by the router (renormalised mode F is fine)
    cfg = moe.make_config(**{**ok, "gate_mode": "F"})
    ws = moe.workspace(cfg)
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((64, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((64, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_router(cfg, x, wg, None, None, idx, w, None, ws)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
