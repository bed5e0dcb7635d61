"""Edge cases on the GPU: degenerate shapes, empty experts, full drops, T = 0,
ragged tiles, and the device status word."""
import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_warp_b200 as moe
from gpu_util import LayerRun, cfg_of, rel_l2, to_f64, upload_inputs, y_tol

pytestmark = pytest.mark.gpu


def _layer_vs_oracle(wl, tokens=None):
    dev, host = upload_inputs(wl)
    run = LayerRun(wl, dev)
    run()
    st = run.check_status()
    assert st[0] == moe.MOE_OK, st
    ref = oracle.route(wl, host["x"], host["Wg"], host.get("bias"))
    assert np.array_equal(run.topk_idx.cpu().numpy(), ref["idx"])
    tokens = np.arange(wl.T) if tokens is None else tokens
    want = oracle.forward_rows(wl, host, ref, tokens)
    got = to_f64(run.y)[tokens]
    if np.abs(want).max() == 0:
        assert np.all(got == 0)
    else:
        assert rel_l2(got, want) <= y_tol(wl)
    return run, ref


@pytest.mark.parametrize("base", [synth.TINY_F32, synth.MIXTRAL.with_(d=128, H=256),
                                  synth.SWITCH.with_(d=128, H=256),
                                  synth.DEEPSEEK.with_(d=128, H=128, H_shared=64)])
def test_single_token(base):
    _layer_vs_oracle(base.with_(T=1))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_one_expert_k1_is_dense_ffn(dtype):
    wl = synth.Workload("n1k1", T=129, d=64, N=1, k=1, H=256, act="swiglu", dtype=dtype,
                        gate_mode="R", seed=21)
    run, ref = _layer_vs_oracle(wl)
    assert np.all(run.topk_w.cpu().numpy() == 1.0)


def test_k_equals_n_full_softmax():
    wl = synth.Workload("k=N", T=77, d=64, N=4, k=4, H=128, act="relu", dtype="bf16",
                        gate_mode="R", seed=22)
    _layer_vs_oracle(wl)


def test_capacity_zero_drops_everything():
    wl = synth.Workload("C=0", T=64, d=64, N=8, k=2, H=128, act="relu", dtype="bf16",
                        gate_mode="F", capacity_factor=0.01, seed=23)
    run, ref = _layer_vs_oracle(wl)
    assert ref["R"] == 0
    assert torch.all(run.y == 0)


def test_empty_experts_large_n():
    # a strong negative bias on half the experts leaves them without tokens
    wl = synth.Workload("empty", T=300, d=128, N=64, k=2, H=128, act="swiglu", dtype="bf16",
                        gate_mode="F", renormalize=True, bias_std=1.0, seed=24)
    dev, host = upload_inputs(wl)
    bias = host["bias"].copy()
    bias[::2] = -100.0
    dev["bias"] = torch.from_numpy(bias).cuda()
    host["bias"] = bias
    run = LayerRun(wl, dev)
    run()
    assert run.check_status()[0] == moe.MOE_OK
    ref = oracle.route(wl, host["x"], host["Wg"], bias)
    assert np.all(ref["counts"][::2] == 0)
    assert np.array_equal(run.topk_idx.cpu().numpy(), ref["idx"])
    want = oracle.forward_rows(wl, host, ref, np.arange(wl.T))
    assert rel_l2(to_f64(run.y), want) <= y_tol(wl)


def test_zero_tokens():
    wl = synth.MIXTRAL.with_(T=0, d=128, H=128)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    dev, _ = upload_inputs(wl.with_(T=1))
    y = torch.empty((0, wl.d), dtype=torch.bfloat16, device="cuda")
    aux = torch.full((1,), 7.0, device="cuda")
    pm = torch.full((wl.N,), 7.0, device="cuda")
    moe.moe_layer_forward(cfg, dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"],
                          None, None, None, y, None, None, None, None, pm, aux, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    assert aux.item() == 0.0 and torch.all(pm == 0)


def test_bad_expert_index_sets_status_word():
    wl = synth.MIXTRAL.with_(T=64, d=128, H=128)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    dev, _ = upload_inputs(wl)
    idx = torch.from_numpy(synth.synthetic_topk(1, wl.T, wl.N, wl.k)).cuda()
    idx[5, 1] = wl.N          # out of range
    rows = wl.T * wl.k
    counts = torch.empty(wl.N, dtype=torch.int32, device="cuda")
    offs = torch.empty(wl.N + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(rows, dtype=torch.int32, device="cuda")
    inv = torch.empty(rows, dtype=torch.int32, device="cuda")
    drop = torch.empty(rows, dtype=torch.uint8, device="cuda")
    xp = torch.empty((rows, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(cfg, dev["x"], idx, counts, offs, perm, inv, drop, xp, None, None, None,
                     None, ws)
    st, word = moe.moe_check_status(ws)
    assert st == moe.MOE_ERR_DEVICE_STATUS and (word & 1)
    assert drop[5 * wl.k + 1].item() == 1 and inv[5 * wl.k + 1].item() == -1
    assert counts.sum().item() == rows - 1
    # the word was cleared by the read
    assert moe.moe_check_status(ws) == (moe.MOE_OK, 0)


def test_ragged_rows_many_tiles():
    # 1 expert, 3 m-tiles with a ragged tail, two SwiGLU n-tiles
    wl = synth.Workload("ragged", T=300, d=192, N=1, k=1, H=256, act="swiglu", dtype="bf16",
                        gate_mode="R", seed=25)
    _layer_vs_oracle(wl)


@pytest.mark.parametrize("act", ["swiglu", "relu"])
def test_pair_tiles_ragged(act):
    # >= 512 rows per expert selects the CTA-pair GEMM (256-row tiles); segments
    # of ~550 rows end in partial pair tiles and H = 384 masks output columns
    wl = synth.Workload("pair", T=1100, d=256, N=2, k=1, H=384, act=act, dtype="bf16",
                        gate_mode="R", seed=26)
    run, ref = _layer_vs_oracle(wl)
    assert ref["R"] >= 512 * wl.N // 2 and np.all(ref["kept"] > 256)


def test_pair_tiles_shared_expert():
    # the shared expert runs every token (1100 rows, one group) on CTA pairs
    wl = synth.Workload("pair-shared", T=1100, d=256, N=4, k=1, H=128, act="swiglu",
                        dtype="bf16", gate_mode="F", renormalize=True, H_shared=256, seed=27)
    _layer_vs_oracle(wl)


@pytest.mark.parametrize("act", ["swiglu", "relu"])
def test_pair_tile_remainders(act):
    # CTA-pair GEMM (>= 512 rows per expert on average) with each expert's
    # last 256-row tile holding 1, 32, 33, 224 or 225 rows, or none (rows past
    # the expert's segment belong to the next expert or lie past the array and
    # must not reach the output); H = 384 leaves a partial column tile for ReLU
    counts = np.array([513, 544, 545, 736, 737, 512])
    wl = synth.Workload("pair-rem", T=int(counts.sum()), d=256, N=len(counts), k=1, H=384,
                        act=act, dtype="bf16", gate_mode="R", seed=28)
    assert wl.T >= 512 * wl.N
    dev, host = upload_inputs(wl)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    yp = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, dev["x"], None, torch.from_numpy(offsets).cuda(), dev["W1"],
                       dev.get("W3"), dev["W2"], yp, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    got = to_f64(yp)
    xin = oracle.decode(host["x"])
    exp_of_row = np.repeat(np.arange(wl.N), counts)
    want = np.empty((wl.T, wl.d))
    for r in range(wl.T):
        e = exp_of_row[r]
        want[r] = oracle.ffn_row(xin[r], host["W1"][e], host["W3"][e] if act == "swiglu" else None,
                                 host["W2"][e], act)
    # every expert's rows, the last tile's in particular, on their own
    for e in range(wl.N):
        lo, hi = offsets[e], offsets[e + 1]
        tail = lo + (counts[e] // 256) * 256
        assert rel_l2(got[lo:hi], want[lo:hi]) <= 5e-3, (e, "all rows")
        if hi > tail:
            assert rel_l2(got[tail:hi], want[tail:hi]) <= 5e-3, (e, "last tile")


@pytest.mark.parametrize("act,fp8,d", [("swiglu", False, 256), ("relu", False, 256),
                                        ("swiglu", True, 256), ("relu", True, 272),
                                        ("swiglu", True, 264)])
def test_gemm_combined_tiles(act, fp8, d):
    # one-CTA GEMM (< 512 rows per expert on average): experts a few rows past
    # 128 or 256 (129, 150, 176, 304) put those rows in a combined tile with
    # the last 128; 177 and 200 leave a separate transposed tile, 100 and 20 a
    # transposed tile alone, 128 a plain one.  FP8: per-row scales in the
    # epilogue.  d = 272 and 264 end in a partial K step (zero-filled by TMA).
    counts = np.array([129, 150, 176, 177, 128, 100, 304, 20, 200])
    wl = synth.Workload("combo", T=int(counts.sum()), d=d, N=len(counts), k=1, H=384, act=act,
                        dtype="bf16", gate_mode="R", dispatch="fp8" if fp8 else "", seed=29)
    assert wl.T < 512 * wl.N
    dev, host = upload_inputs(wl)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    if fp8:
        q, sc = oracle.quantize_rows(host["x"])
        xp = torch.from_numpy(q).cuda()
        xs = torch.from_numpy(sc).cuda()
        xin = oracle.dequantize_rows(q, sc)
    else:
        xp, xs = dev["x"], None
        xin = oracle.decode(host["x"])
    yp = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, xp, xs, torch.from_numpy(offsets).cuda(), dev["W1"], dev.get("W3"),
                       dev["W2"], yp, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    got = to_f64(yp)
    exp_of_row = np.repeat(np.arange(wl.N), counts)
    want = np.empty((wl.T, wl.d))
    for r in range(wl.T):
        e = exp_of_row[r]
        want[r] = oracle.ffn_row(xin[r], host["W1"][e], host["W3"][e] if act == "swiglu" else None,
                                 host["W2"][e], act)
    tol = 5e-3   # the oracle takes the same dequantised rows, so FP8 adds no error here
    for e in range(wl.N):
        lo, hi = offsets[e], offsets[e + 1]
        assert rel_l2(got[lo:hi], want[lo:hi]) <= tol, (e, "all rows")
        tail = lo + (counts[e] // 128) * 128
        if hi > tail and counts[e] > 128:
            assert rel_l2(got[tail:hi], want[tail:hi]) <= tol, (e, "rows past the last 128")


@pytest.mark.parametrize("act", ["swiglu", "relu"])
def test_transposed_tiles_small_experts_with_one_long_group(act):
    # experts averaging at most 64 rows run both projections on the transposed
    # CTA-pair kernel: rows are cut into chunks of up to 160 rows (one tile),
    # a longer group into chunks of at most 128 rows (here 330 -> 3 chunks,
    # 150 -> one tile of 129-160 rows holding both accumulator slots); empty
    # experts, single rows and a partial last feature tile (H = 384 and
    # d = 640 against 256- and 512-feature tiles) around them
    counts = np.array([330, 1, 0, 17, 150, 0, 32, 0, 3, 0, 0, 64, 0, 0, 0, 2])
    N = len(counts)
    wl = synth.Workload("transposed", T=int(counts.sum()), d=640, N=N, k=1, H=384, act=act,
                        dtype="bf16", gate_mode="R", seed=43)
    assert wl.T <= 64 * N
    dev, host = upload_inputs(wl)
    cfg = cfg_of(wl)
    ws = moe.workspace(cfg)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    yp = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, dev["x"], None, torch.from_numpy(offsets).cuda(), dev["W1"],
                       dev.get("W3"), dev["W2"], yp, ws)
    assert moe.moe_check_status(ws)[0] == moe.MOE_OK
    got = to_f64(yp)
    xin = oracle.decode(host["x"])
    exp_of_row = np.repeat(np.arange(N), counts)
    want = np.empty((wl.T, wl.d))
    for r in range(wl.T):
        e = exp_of_row[r]
        want[r] = oracle.ffn_row(xin[r], host["W1"][e], host["W3"][e] if act == "swiglu" else None,
                                 host["W2"][e], act)
    for e in range(N):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            assert rel_l2(got[lo:hi], want[lo:hi]) <= 5e-3, e
            # every row of the long group's chunks, one by one
            if counts[e] > 128:
                for r in range(lo, hi, 37):
                    assert rel_l2(got[r:r + 1], want[r:r + 1]) <= 1e-2, (e, r)
