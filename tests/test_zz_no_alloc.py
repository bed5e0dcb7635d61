"""moe_dispatch_noalloc against moe_dispatch.

moe_dispatch_noalloc is the dispatch entry point for callers that cannot give
the library a workspace allocated with cudaMalloc: a host framework that owns
all device memory through its own pool, a runtime whose memory budget is
fixed up front, or a call path where cudaMalloc/cudaFree may not be used
because they can synchronise the device.  It keeps its scratch in an array
built into the library instead.  This file is collected last so that a run
that stops at the first failure has run every other test before it.

Each case calls the no-allocation entry point twice in a row (the second time
on different routing, so leftovers in the shared array would show) and
compares both results with moe_dispatch given a workspace, bit for bit as the
other dispatch tests do.  Batches of more than 8192 (token, slot) pairs take
the multi-block sort, the path that keeps per-block expert counts and
fallback bases in the built-in array between its launches: those cases run
two calls of different block counts (different batch sizes) and are also
compared with the oracle's dispatch, up to the 262,144-pair limit.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_warp_b200 as moe
from gpu_util import cfg_of, tdtype, upload_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "capacity-bf16": synth.SWITCH.with_(T=1000, d=128, H=256),
    "fp8-k8": synth.DEEPSEEK.with_(T=200, d=256, H=128, H_shared=128),
    "fp32": synth.TINY_F32,
    "fallback-slot": synth.MIXTRAL.with_(T=600, d=128, N=8, H=256, capacity_factor=0.7,
                                         overflow="fallback", slot_priority=True),
}


def _buffers(wl):
    rows = wl.T * wl.k
    fp8 = wl.dispatch == "fp8"
    return dict(
        counts=torch.empty(wl.N, dtype=torch.int32, device="cuda"),
        offs=torch.empty(wl.N + 2, dtype=torch.int32, device="cuda"),
        perm=torch.full((rows,), -1, dtype=torch.int32, device="cuda"),
        inv=torch.empty(rows, dtype=torch.int32, device="cuda"),
        drop=torch.empty(rows, dtype=torch.uint8, device="cuda"),
        xp=torch.zeros((rows, wl.d), dtype=torch.uint8 if fp8 else tdtype(wl), device="cuda"),
        xs=torch.zeros(rows, dtype=torch.float32, device="cuda") if fp8 else None,
        f=torch.empty(wl.N, dtype=torch.float32, device="cuda"),
        aux=torch.empty(1, dtype=torch.float32, device="cuda"),
        n_off=wl.N + (2 if wl.overflow == "fallback" else 1),
    )


def _same(a, b, R):
    assert torch.equal(a["counts"], b["counts"])
    n = a["n_off"]
    assert torch.equal(a["offs"][:n], b["offs"][:n])
    assert torch.equal(a["perm"][:R], b["perm"][:R])
    assert torch.equal(a["inv"], b["inv"])
    assert torch.equal(a["drop"], b["drop"])
    assert torch.equal(a["xp"][:R].view(torch.uint8), b["xp"][:R].view(torch.uint8))
    if a["xs"] is not None:
        assert torch.equal(a["xs"][:R], b["xs"][:R])
    assert torch.equal(a["f"], b["f"])
    assert torch.equal(a["aux"], b["aux"])


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_dispatch_matches_workspace_dispatch(name):
    wl = CASES[name]
    cfg = cfg_of(wl)
    dev, _ = upload_inputs(wl)
    pm = torch.full((wl.N,), 1.0 / wl.N, dtype=torch.float32, device="cuda")
    ws = moe.workspace(cfg)
    for call, skew in enumerate((0.6, 0.1)):
        idx = torch.from_numpy(synth.synthetic_topk(wl.seed + 90 + call, wl.T, wl.N, wl.k,
                                                    skew=skew)).cuda()
        ref, got = _buffers(wl), _buffers(wl)
        moe.moe_dispatch(cfg, dev["x"], idx, ref["counts"], ref["offs"], ref["perm"], ref["inv"],
                         ref["drop"], ref["xp"], ref["xs"], pm, ref["f"], ref["aux"], ws)
        moe.moe_dispatch_noalloc(cfg, dev["x"], idx, got["counts"], got["offs"], got["perm"],
                                 got["inv"], got["drop"], got["xp"], got["xs"], pm, got["f"],
                                 got["aux"])
        torch.cuda.synchronize()
        assert moe.moe_check_status(ws)[0] == moe.MOE_OK
        R = int(ref["offs"][ref["n_off"] - 1].item())
        _same(ref, got, R)


# batches above 8192 pairs (multi-block sort): (workload, second call's T)
MULTI = {
    "n256-fp8-20k": (synth.DEEPSEEK.with_(T=2500, d=128, H=128, H_shared=0), 1100),
    "fallback-50k": (synth.SWITCH.with_(T=50000, d=64, H=64, overflow="fallback"), 30000),
    "slot-drop-40k": (synth.MIXTRAL.with_(T=20000, d=64, N=16, H=64, capacity_factor=0.9,
                                          slot_priority=True), 9000),
    "limit-262144": (synth.MIXTRAL.with_(T=131072, d=64, N=8, H=64, capacity_factor=1.1), 70000),
}


def _oracle_check(wl, x_bits, idx, got):
    ref = oracle.dispatch(idx, wl.N, wl.capacity_factor, wl.overflow == "fallback",
                          wl.slot_priority)
    n = got["n_off"]
    assert np.array_equal(got["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(got["offs"][:n].cpu().numpy(), ref["offsets"])
    R = ref["R"]
    assert np.array_equal(got["perm"][:R].cpu().numpy(), ref["perm"])
    assert np.array_equal(got["inv"].cpu().numpy(), ref["inv_row"])
    assert np.array_equal(got["drop"].cpu().numpy(), ref["drop"])
    rows = x_bits[ref["perm"] // wl.k]
    if wl.dispatch == "fp8":
        q, sc = oracle.quantize_rows(rows)
        assert np.array_equal(got["xp"][:R].cpu().numpy(), q)
        assert np.array_equal(got["xs"][:R].cpu().numpy(), sc)
    else:
        assert np.array_equal(got["xp"][:R].view(torch.int16).cpu().numpy().view(np.uint16), rows)
    f, _, _ = oracle.aux(ref["counts"], np.full((wl.T, wl.N), 1.0 / wl.N), wl.k, wl.aux_alpha)
    np.testing.assert_allclose(got["f"].cpu().numpy(), f, rtol=1e-6)


@pytest.mark.parametrize("name", list(MULTI))
def test_noalloc_multiblock_matches_workspace_dispatch_and_oracle(name):
    wl0, T2 = MULTI[name]
    assert wl0.T * wl0.k > 8192 and T2 * wl0.k > 8192
    assert (wl0.T * wl0.k + 2047) // 2048 != (T2 * wl0.k + 2047) // 2048   # different block counts
    x_bits = synth.normal(wl0.seed, synth.TENSOR_IDS["x"], wl0.T * wl0.d, 1.0,
                          wl0.dtype).reshape(wl0.T, wl0.d)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    pm = torch.full((wl0.N,), 1.0 / wl0.N, dtype=torch.float32, device="cuda")
    for call, (T, skew) in enumerate(((wl0.T, 0.5), (T2, 0.05))):
        wl = wl0.with_(T=T)
        cfg = cfg_of(wl)
        ws = moe.workspace(cfg)
        idx_np = synth.synthetic_topk(wl.seed + 200 + call, T, wl.N, wl.k, skew=skew)
        idx = torch.from_numpy(idx_np).cuda()
        ref, got = _buffers(wl), _buffers(wl)
        moe.moe_dispatch(cfg, x[:T], idx, ref["counts"], ref["offs"], ref["perm"], ref["inv"],
                         ref["drop"], ref["xp"], ref["xs"], pm, ref["f"], ref["aux"], ws)
        moe.moe_dispatch_noalloc(cfg, x[:T], idx, got["counts"], got["offs"], got["perm"],
                                 got["inv"], got["drop"], got["xp"], got["xs"], pm, got["f"],
                                 got["aux"])
        torch.cuda.synchronize()
        assert moe.moe_check_status(ws)[0] == moe.MOE_OK
        R = int(ref["offs"][ref["n_off"] - 1].item())
        _same(ref, got, R)
        _oracle_check(wl, x_bits[:T], idx_np, got)
        del ws


def test_noalloc_rejects_batches_beyond_its_scratch():
    # 262145 (token, slot) pairs: one more than the built-in array holds
    cfg = moe.make_config(262145, 128, 8, 1, 128)
    fake = ctypes.c_void_p(1 << 40)          # never dereferenced: rejected on the host
    r = moe.lib().moe_dispatch_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake,
                                       fake, fake, None, None, None, None, None)
    assert r == moe.MOE_ERR_WORKSPACE
    ok = moe.make_config(131072, 128, 8, 2, 128)   # exactly at the limit: accepted sizes
    assert ok.T * ok.k == 262144
