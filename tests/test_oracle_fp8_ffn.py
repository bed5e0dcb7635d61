"""Pins for the oracle's FP8 E4M3 codec, per-token quantisation and expert FFN."""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # values fixed by the OCP E4M3 definition
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert got[0x38] == 1.0 and got[0xB8] == -1.0 and np.isnan(got[0x7F])


def test_e4m3_encode_rne_matches_torch_in_range():
    v = synth.normal(3, 21, 20000, 60.0, "f32")
    v = v[np.abs(v) < 448]
    got = oracle.e4m3_encode(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_midpoints_ties_to_even_and_saturation():
    table = oracle.e4m3_table()
    pos = np.array([table[c] for c in range(0x00, 0x7F)])      # 0 .. 448 ascending
    assert np.all(np.diff(pos) > 0)
    mids = (pos[:-1] + pos[1:]) / 2
    got = oracle.e4m3_encode(mids)
    lo, hi = np.arange(0, 0x7E), np.arange(1, 0x7F)
    even = np.where(lo % 2 == 0, lo, hi)                       # tie -> even mantissa
    assert np.array_equal(got, even.astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode(-mids), (even | 0x80).astype(np.uint8))
    assert np.all(oracle.e4m3_encode(np.array([448.0, 449.0, 470.0, 1e6])) == 0x7E)
    assert np.all(oracle.e4m3_encode(np.array([-500.0])) == 0xFE)


def test_quantize_rows_scale_and_roundtrip():
    x = synth.normal(4, 22, 16 * 96, 1.0, "bf16").reshape(16, 96)
    x[5] = 0
    q, s = oracle.quantize_rows(x)
    xv = oracle.decode(x)
    amax = np.abs(xv).max(1).astype(np.float32)
    assert s[5] == 1.0 and np.all(q[5] == 0)
    nz = np.arange(16) != 5
    assert np.array_equal(s[nz], amax[nz] / np.float32(448.0))
    # the largest element of each row maps to the largest finite code
    for t in np.where(nz)[0]:
        j = np.argmax(np.abs(xv[t]))
        assert q[t, j] & 0x7F == 0x7E
    # same codes as torch's E4M3 conversion of x/scale computed in fp32
    ref = torch.from_numpy((xv.astype(np.float32) / s[:, None]).astype(np.float32))
    ref = ref.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    deq = oracle.dequantize_rows(q, s)
    rel = np.abs(deq[nz] - xv[nz]) / np.maximum(np.abs(xv[nz]), 2.0 ** -6 * amax[nz, None])
    assert rel.max() <= 2.0 ** -4 + 1e-12


@pytest.mark.parametrize("act", ["relu", "swiglu"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_n1_k1_layer_is_dense_ffn(act, dt):
    # with one expert and k = 1 the gate is 1 and the layer is a dense FFN
    wl = synth.Workload("n1k1", T=24, d=32, N=1, k=1, H=48, act=act, dtype=dt, gate_mode="R", seed=9)
    inp = synth.make_host(wl)
    routing = oracle.route(wl, inp["x"], inp["Wg"])
    assert np.all(routing["idx"] == 0) and np.all(routing["gate"] == 1.0)
    y = oracle.forward_rows(wl, inp, routing, np.arange(wl.T))
    x = oracle.decode(inp["x"])
    W1 = oracle.decode(inp["W1"][0])
    W2 = oracle.decode(inp["W2"][0])
    a = x @ W1.T
    if act == "relu":
        h = np.maximum(a, 0)
    else:
        W3 = oracle.decode(inp["W3"][0])
        h = a * scipy.special.expit(a) * (x @ W3.T)
    np.testing.assert_allclose(y, h @ W2.T, rtol=1e-11, atol=1e-12)


def test_combine_matches_per_expert_library_ffn_and_drops():
    wl = synth.Workload("small", T=40, d=16, N=4, k=2, H=24, act="swiglu", dtype="bf16",
                        gate_mode="F", renormalize=True, capacity_factor=1.0, H_shared=8,
                        dispatch="fp8", seed=12)
    inp = synth.make_host(wl)
    routing = oracle.route(wl, inp["x"], inp["Wg"])
    y = oracle.forward_rows(wl, inp, routing, np.arange(wl.T))
    q, s = oracle.quantize_rows(inp["x"])
    xq = oracle.e4m3_table()[q] * s[:, None].astype(np.float64)
    xf = oracle.decode(inp["x"])

    def ffn(xr, W1, W3, W2):
        a = xr @ oracle.decode(W1).T
        return (a * scipy.special.expit(a) * (xr @ oracle.decode(W3).T)) @ oracle.decode(W2).T

    drop = routing["drop"].reshape(wl.T, wl.k)
    assert drop.sum() > 0                         # capacity 1.0 with skewed routing drops some
    for t in range(wl.T):
        ref = ffn(xf[t], inp["Ws1"], inp["Ws3"], inp["Ws2"])
        for j in range(wl.k):
            if not drop[t, j]:
                e = routing["idx"][t, j]
                ref = ref + routing["gate"][t, j] * ffn(xq[t], inp["W1"][e], inp["W3"][e], inp["W2"][e])
        np.testing.assert_allclose(y[t], ref, rtol=1e-10, atol=1e-12)


def test_lazy_rows_equal_stacked_rows():
    wl = synth.Workload("lazy", T=30, d=16, N=6, k=2, H=8, act="swiglu", dtype="bf16", gate_mode="R",
                        seed=13)
    inp = synth.make_host(wl)
    routing = oracle.route(wl, inp["x"], inp["Wg"])
    toks = [0, 7, 29]
    a = oracle.forward_rows(wl, inp, routing, toks)
    b = oracle.forward_rows_lazy(wl, inp["x"], routing, toks,
                                 lambda e: (inp["W1"][e], inp["W3"][e], inp["W2"][e]))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("variant", ["fp8-shared-drop", "fallback-slot"])
def test_rows_by_expert_equal_stacked_rows(variant):
    # the expert-by-expert evaluation (one expert's weights at a time) gives the
    # same sum as the per-token evaluation pinned above against numpy FFNs
    if variant == "fp8-shared-drop":
        wl = synth.Workload("byexp", T=40, d=16, N=4, k=2, H=24, act="swiglu", dtype="bf16",
                            gate_mode="F", renormalize=True, capacity_factor=1.0, H_shared=8,
                            dispatch="fp8", seed=12)
    else:
        wl = synth.Workload("byexp-fb", T=50, d=16, N=4, k=2, H=8, act="relu", dtype="bf16",
                            gate_mode="R", capacity_factor=0.6, overflow="fallback",
                            slot_priority=True, seed=14)
    inp = synth.make_host(wl)
    routing = oracle.route(wl, inp["x"], inp["Wg"])
    assert routing["drop"].sum() > 0 or wl.overflow == "fallback"
    toks = np.arange(wl.T)
    a = oracle.forward_rows(wl, inp, routing, toks)
    shared = (inp["Ws1"], inp.get("Ws3"), inp["Ws2"]) if wl.H_shared else None
    b = oracle.forward_rows_by_expert(
        wl, inp["x"], routing, toks,
        lambda e: (inp["W1"][e], inp["W3"][e] if wl.act == "swiglu" else None, inp["W2"][e]),
        shared)
    np.testing.assert_allclose(b, a, rtol=1e-13, atol=1e-14)


def test_combine_bruteforce():
    T, k, d = 17, 3, 5
    rng_rows = synth.normal(1, 40, 30 * d, 1.0, "f32").reshape(30, d).astype(np.float64)
    inv = synth.uniform_int(2, 41, T * k, 31) - 1          # -1 .. 29
    gate = synth.normal(3, 42, T * k, 1.0, "f32").reshape(T, k).astype(np.float64)
    ysh = synth.normal(4, 43, T * d, 1.0, "f32").reshape(T, d).astype(np.float64)
    y = oracle.combine(rng_rows, inv, gate, ysh)
    for t in range(T):
        ref = ysh[t].copy()
        for j in range(k):
            r = inv[t * k + j]
            if r >= 0:
                ref = ref + gate[t, j] * rng_rows[r]
        np.testing.assert_allclose(y[t], ref, rtol=1e-14, atol=1e-14)
