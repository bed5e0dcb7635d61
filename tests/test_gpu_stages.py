"""GPU parity of each C-ABI stage against the oracle, on the same seeded inputs.

Sizes are small enough for the oracle to finish in seconds but span several
tiles and ragged tails.  Integer outputs are compared bit for bit; floating
point outputs within the bounds the layer's precision allows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_warp_b200 as moe
from gpu_util import (cfg_of, near_tie_tokens, rel_l2, tdtype, to_dev, to_f64, to_host_bits,
                      upload_inputs, y_tol)

pytestmark = pytest.mark.gpu

# Small workloads with the structure of the five layers (dtype, routing mode,
# activation, capacity, bias skew, FP8 dispatch, shared expert).
SMALL = {
    "tiny": synth.TINY_F32,
    "mixtral": synth.MIXTRAL.with_(T=300, d=256, H=384),
    "switch": synth.SWITCH.with_(T=1000, d=128, H=256),
    "deepseek": synth.DEEPSEEK.with_(T=200, d=256, H=128, H_shared=128),
    # FP8 dispatch with a partial last K step in every d-wide GEMM (d = 272
    # and 264: not multiples of 64; 264 not of 16 either)
    "deepseek-d272": synth.DEEPSEEK.with_(T=300, d=272, H=192, H_shared=0, seed=31),
    "deepseek-d264": synth.DEEPSEEK.with_(T=150, d=264, H=128, H_shared=64, seed=32),
    "grok": synth.GROK.with_(d=512, H=1024),
}


@pytest.fixture(params=list(SMALL))
def small(request):
    wl = SMALL[request.param]
    dev, host = upload_inputs(wl)
    return wl, dev, host


def test_router_parity(small):
    wl, dev, host = small
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    T, k, N = wl.T, wl.k, wl.N
    logits = torch.empty((T, N), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    pm = torch.empty(N, dtype=torch.float32, device="cuda")
    moe.moe_router(cfg, dev["x"], dev["Wg"], dev.get("bias"), logits, idx, w, pm, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    ref = oracle.route(wl, host["x"], host["Wg"], host.get("bias"))
    tie = near_tie_tokens(ref["logits"], ref["idx"], k)
    gi = idx.cpu().numpy()
    ok = ~tie
    assert np.array_equal(gi[ok], ref["idx"][ok]), "expert indices differ off near-ties"
    gw = w.cpu().numpy().astype(np.float64)
    relw = np.abs(gw[ok] - ref["gate"][ok]) / np.abs(ref["gate"][ok])
    assert relw.max() <= 1e-6, f"gate rel err {relw.max():.3g}"
    np.testing.assert_allclose(pm.cpu().numpy(), ref["p_mean"], rtol=1e-5, atol=1e-9)
    # logits: fp32 accumulation of bf16 products (large N) or rounded fp64 (small N)
    np.testing.assert_allclose(logits.cpu().numpy(), ref["logits"], rtol=0,
                               atol=2e-5 * max(1.0, np.abs(ref["logits"]).max()))


@pytest.mark.parametrize("skew", [0.0, 0.7])
def test_dispatch_parity(small, skew):
    wl, dev, host = small
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    T, k, N, d = wl.T, wl.k, wl.N, wl.d
    idx_h = synth.synthetic_topk(wl.seed + 50, T, N, k, skew=skew)
    idx = torch.from_numpy(idx_h).cuda()
    rows = T * k
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    offs = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv = torch.empty(rows, dtype=torch.int32, device="cuda")
    drop = torch.empty(rows, dtype=torch.uint8, device="cuda")
    fp8 = wl.dispatch == "fp8"
    xp = torch.zeros((rows, d), dtype=torch.uint8 if fp8 else tdtype(wl), device="cuda")
    xs = torch.zeros(rows, dtype=torch.float32, device="cuda") if fp8 else None
    pm = torch.full((N,), 1.0 / N, dtype=torch.float32, device="cuda")
    f = torch.empty(N, dtype=torch.float32, device="cuda")
    aux = torch.empty(1, dtype=torch.float32, device="cuda")
    moe.moe_dispatch(cfg, dev["x"], idx, counts, offs, perm, inv, drop, xp, xs, pm, f, aux, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    ref = oracle.dispatch(idx_h, N, wl.capacity_factor)
    R = ref["R"]
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(offs.cpu().numpy(), ref["offsets"])
    assert np.array_equal(perm.cpu().numpy()[:R], ref["perm"])
    assert np.array_equal(inv.cpu().numpy(), ref["inv_row"])
    assert np.array_equal(drop.cpu().numpy(), ref["drop"])
    # f and L_aux (with p_i = 1/N, L_aux = alpha * sum f_i = alpha)
    np.testing.assert_allclose(f.cpu().numpy(), ref["counts"] / (T * k), rtol=1e-7)
    _, _, laux = oracle.aux(ref["counts"], np.full((T, N), 1.0 / N), k, wl.aux_alpha)
    np.testing.assert_allclose(aux.item(), laux, rtol=1e-5)
    # payload rows
    tok = ref["perm"] // k
    if fp8:
        q, s = oracle.quantize_rows(host["x"][tok])
        assert np.array_equal(xp.cpu().numpy()[:R], q)
        assert np.array_equal(xs.cpu().numpy()[:R], s)
    else:
        assert np.array_equal(to_host_bits(xp)[:R], host["x"][tok])


def test_expert_ffn_parity(small):
    wl, dev, host = small
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    T, k, N, d = wl.T, wl.k, wl.N, wl.d
    idx_h = synth.synthetic_topk(wl.seed + 60, T, N, k, skew=0.3)
    ref = oracle.dispatch(idx_h, N, wl.capacity_factor)
    R = ref["R"]
    rows = T * k
    fp8 = wl.dispatch == "fp8"
    tok = ref["perm"] // k
    # payload rows as the oracle defines them
    if fp8:
        q, s = oracle.quantize_rows(host["x"][tok])
        xp_h = np.zeros((rows, d), np.uint8)
        xp_h[:R] = q
        xs = torch.zeros(rows, dtype=torch.float32, device="cuda")
        xs[:R] = torch.from_numpy(s).cuda()
        xp = torch.from_numpy(xp_h).cuda()
        xin = oracle.dequantize_rows(q, s)
    else:
        xp_h = np.zeros((rows, d), host["x"].dtype)
        xp_h[:R] = host["x"][tok]
        xp = to_dev(xp_h)
        xs = None
        xin = oracle.decode(host["x"][tok])
    offs = torch.from_numpy(ref["offsets"]).cuda()
    yp = torch.zeros((rows, d), dtype=tdtype(wl), device="cuda")
    moe.moe_expert_ffn(cfg, xp, xs, offs, dev["W1"], dev.get("W3"), dev["W2"], yp, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    got = to_f64(yp)[:R]
    exp_of_row = np.repeat(np.arange(N), ref["kept"])
    want = np.empty((R, d))
    for r in range(R):
        e = exp_of_row[r]
        want[r] = oracle.ffn_row(xin[r], host["W1"][e], host["W3"][e] if wl.act == "swiglu" else None,
                                 host["W2"][e], wl.act)
    err = rel_l2(got, want)
    tol = 1e-5 if wl.dtype == "f32" else 5e-3
    assert err <= tol, f"y_perm rel-L2 {err:.3g}"
    # rows past R stay untouched
    assert torch.all(yp[R:].float() == 0)


def test_combine_parity(small):
    wl, dev, host = small
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    T, k, N, d = wl.T, wl.k, wl.N, wl.d
    idx_h = synth.synthetic_topk(wl.seed + 70, T, N, k, skew=0.8)
    ref = oracle.dispatch(idx_h, N, wl.capacity_factor if wl.capacity_factor > 0 else 0.9)
    rows = T * k
    yrows_h = synth.normal(wl.seed, 60, rows * d, 1.0, wl.dtype).reshape(rows, d)
    gate_h = np.abs(synth.normal(wl.seed, 61, T * k, 0.5, "f32")).reshape(T, k)
    ysh_h = synth.normal(wl.seed, 62, T * d, 1.0, wl.dtype).reshape(T, d)
    y = torch.empty((T, d), dtype=tdtype(wl), device="cuda")
    moe.moe_combine(cfg, to_dev(yrows_h), torch.from_numpy(ref["inv_row"]).cuda(),
                    torch.from_numpy(gate_h).cuda(), to_dev(ysh_h), y, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    want = oracle.combine(oracle.decode(yrows_h), ref["inv_row"], gate_h.astype(np.float64),
                          oracle.decode(ysh_h))
    got = to_f64(y)
    # one rounding of the fp32 sum to the output type
    tol = 2.0 ** -8 if wl.dtype == "bf16" else 1e-6
    np.testing.assert_allclose(got, want, rtol=tol, atol=tol * np.abs(want).max() * 1e-2)
