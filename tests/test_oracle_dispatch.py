"""Pins for the oracle's dispatch (counts, capacity, permutation) and aux statistics."""
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
import synth


def _check_permutation(idx, N, cf, disp):
    T, k = idx.shape
    flat = idx.ravel()
    counts = np.bincount(flat, minlength=N)
    assert np.array_equal(disp["counts"], counts)
    assert counts.sum() == T * k
    C = math.floor(cf * T / N) if cf > 0 else None
    kept = np.minimum(counts, C) if C is not None else counts
    assert np.array_equal(disp["kept"], kept)
    drops = int(disp["drop"].sum())
    assert kept.sum() == T * k - drops == disp["R"]
    assert np.array_equal(disp["offsets"], np.concatenate([[0], np.cumsum(kept)]))
    # brute force: walk tokens in order, keep the first C of every expert
    seen = [[] for _ in range(N)]
    for i in range(T * k):
        seen[flat[i]].append(i)
    rows = np.concatenate([np.array(s[:kept[e]], dtype=np.int64) for e, s in enumerate(seen)] or
                          [np.zeros(0, np.int64)])
    assert np.array_equal(disp["perm"], rows)
    # perm is a bijection between kept pairs and rows; inv_row inverts it
    R = disp["R"]
    assert np.array_equal(disp["inv_row"][disp["perm"]], np.arange(R))
    dropped = np.where(disp["drop"] == 1)[0]
    assert np.all(disp["inv_row"][dropped] == -1)
    assert len(set(disp["perm"].tolist())) == R
    # each segment is sorted by token
    for e in range(N):
        seg = disp["perm"][disp["offsets"][e]:disp["offsets"][e + 1]] // k
        assert np.all(np.diff(seg) > 0)


@pytest.mark.parametrize("T,N,k,cf,skew", [
    (1, 1, 1, 0.0, 0.0), (100, 8, 2, 0.0, 0.0), (300, 16, 4, 1.25, 0.6),
    (257, 5, 5, 0.0, 0.0), (64, 8, 1, 0.1, 0.9), (50, 64, 3, 1.0, 0.3), (40, 4, 1, 0.05, 0.0)])
def test_dispatch_against_bruteforce(T, N, k, cf, skew):
    idx = synth.synthetic_topk(T + N, T, N, k, skew=skew)
    disp = oracle.dispatch(idx, N, cf)
    _check_permutation(idx, N, cf, disp)


def test_no_capacity_equals_library_stable_argsort():
    idx = synth.synthetic_topk(3, 1000, 32, 4, skew=0.2)
    disp = oracle.dispatch(idx, 32, 0.0)
    assert np.array_equal(disp["perm"], np.argsort(idx.ravel(), kind="stable"))


def test_switch_capacity_is_80():
    # C = capacity_factor * T / N = 1.25 * 8192 / 128 = 80 (page 5, capacity factor)
    assert synth.SWITCH.capacity() == 80
    idx = np.zeros((8192, 1), np.int32)            # everyone picks expert 0
    disp = oracle.dispatch(idx, 128, 1.25)
    assert disp["kept"][0] == 80 and disp["R"] == 80
    assert np.array_equal(disp["perm"], np.arange(80))


def test_capacity_zero_drops_everything():
    idx = synth.synthetic_topk(1, 20, 8, 2)
    disp = oracle.dispatch(idx, 8, 0.1)             # floor(0.1*20/8) = 0
    assert disp["R"] == 0 and disp["drop"].sum() == 40
    assert np.all(disp["inv_row"] == -1)


def test_laux_equals_alpha_when_uniform():
    # d = N, W_g = I, x_t = c e_(t mod N): every softmax row is a cyclic shift of
    # the same vector, so p_i = 1/N; with k=1 every expert gets exactly T/N tokens,
    # so f_i = 1/N and L_aux = alpha * N * N * (1/N)(1/N) = alpha (page 5).
    for k in (1, 2):
        N, m, c, alpha = 8, 16, 3.0, 0.01
        T = N * m
        x = np.zeros((T, N), np.float32)
        x[np.arange(T), np.arange(T) % N] = c
        Wg = np.eye(N, dtype=np.float32)
        logits = oracle.router_logits(x, Wg)
        idx, gate, probs = oracle.topk_gate(logits, k, "F")
        disp = oracle.dispatch(idx, N, 0.0)
        f, pm, laux = oracle.aux(disp["counts"], probs, k, alpha)
        np.testing.assert_allclose(pm, 1.0 / N, rtol=1e-13)
        if k == 1:
            np.testing.assert_allclose(f, 1.0 / N, rtol=0)
            assert abs(laux - alpha) < 1e-12
        assert abs(f.sum() - 1.0) < 1e-15


def test_laux_collapsed_router_is_alpha_times_n():
    # every token sends all mass to expert 0: f_0 = 1, p_0 -> 1, L_aux -> alpha * N
    N, T = 16, 64
    x = np.ones((T, 1), np.float32)
    Wg = np.full((N, 1), -50.0, np.float32)
    Wg[0] = 50.0
    logits = oracle.router_logits(x, Wg)
    idx, gate, probs = oracle.topk_gate(logits, 1, "F")
    disp = oracle.dispatch(idx, N, 0.0)
    f, pm, laux = oracle.aux(disp["counts"], probs, 1, 0.05)
    assert f[0] == 1.0
    assert abs(laux - 0.05 * N) < 1e-12


# ------------------------------------------------- capacity variants (fallback expert, slot priority)
def _golden(name):
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, v = line.split(":", 1)
            vals[key.strip()] = [float(a) for a in v.split()]
    return vals


def test_capacity_priority_worked_example():
    g = _golden("capacity_priority_example.txt")
    T, k, N = int(g["T"][0]), int(g["k"][0]), int(g["N"][0])
    idx = np.array(g["idx"], np.int32).reshape(T, k)
    cf = g["capacity_factor"][0]
    ints = lambda key: [int(v) for v in g[key]]
    tok = oracle.dispatch(idx, N, cf)
    slot = oracle.dispatch(idx, N, cf, slot_priority=True)
    assert tok["drop"].tolist() == ints("drop_token_order")
    assert slot["drop"].tolist() == ints("drop_slot_order")
    assert tok["perm"].tolist() == ints("perm_token_order")
    assert slot["perm"].tolist() == ints("perm_slot_order")
    for prio, key in [(False, "fallback_rows_token_order"), (True, "fallback_rows_slot_order")]:
        fb = oracle.dispatch(idx, N, cf, fallback=True, slot_priority=prio)
        assert fb["R"] == T * k and not fb["drop"].any()
        assert fb["perm"][fb["offsets"][N]:fb["offsets"][N + 1]].tolist() == ints(key)
        assert fb["expert"][ints(key)].tolist() == [N, N]


def _brute(idx, N, C, slot_priority, fallback):
    """Walk the pairs in the stated order with per-expert counters."""
    T, k = idx.shape
    order = [(t, j) for j in range(k) for t in range(T)] if slot_priority else \
            [(t, j) for t in range(T) for j in range(k)]
    seen = [0] * N
    kept = {e: [] for e in range(N + 1)}
    for t, j in order:
        e = int(idx[t, j])
        if C < 0 or seen[e] < C:
            kept[e].append(t * k + j)
        elif fallback:
            kept[N].append(t * k + j)
        seen[e] += 1
    return [p for e in range(N + 1) for p in kept[e]]


@pytest.mark.parametrize("slot_priority", [False, True])
@pytest.mark.parametrize("fallback", [False, True])
def test_capacity_variants_match_bruteforce(slot_priority, fallback):
    for seed, (T, N, k, cf) in enumerate([(37, 5, 2, 0.9), (50, 8, 3, 1.0), (64, 4, 1, 0.5),
                                          (20, 3, 3, 1.25)]):
        idx = synth.synthetic_topk(100 + seed, T, N, k, skew=0.6)
        C = int(np.floor(float(np.float32(cf)) * T / N))
        ref = oracle.dispatch(idx, N, cf, fallback=fallback, slot_priority=slot_priority)
        want = _brute(idx, N, C, slot_priority, fallback)
        assert ref["perm"].tolist() == want
        inv = np.full(T * k, -1)
        inv[np.array(want, dtype=np.int64)] = np.arange(len(want))
        assert np.array_equal(ref["inv_row"], inv)
        assert np.array_equal(ref["drop"], (inv < 0).astype(np.uint8))


def test_fallback_is_drop_mode_plus_overflow_segment():
    T, N, k, cf = 300, 16, 2, 0.75
    idx = synth.synthetic_topk(7, T, N, k, skew=0.7)
    drop = oracle.dispatch(idx, N, cf)
    fb = oracle.dispatch(idx, N, cf, fallback=True)
    assert drop["drop"].sum() > 0
    # the routed experts' rows are unchanged; the fallback takes the dropped pairs in order
    assert np.array_equal(fb["offsets"][:N + 1], drop["offsets"])
    assert np.array_equal(fb["perm"][:drop["R"]], drop["perm"])
    assert fb["perm"][drop["R"]:].tolist() == np.nonzero(drop["drop"])[0].tolist()
    assert fb["R"] == T * k and not fb["drop"].any()
    assert np.array_equal(fb["counts"], drop["counts"])       # f_i: pre-drop counts
    # no capacity: nothing to re-route
    nocap = oracle.dispatch(idx, N, 0.0, fallback=True)
    assert nocap["offsets"][N + 1] == nocap["offsets"][N] == T * k
    # k = 1: slot priority is token order
    one = synth.synthetic_topk(8, T, N, 1, skew=0.7)
    a, b = oracle.dispatch(one, N, cf), oracle.dispatch(one, N, cf, slot_priority=True)
    assert all(np.array_equal(a[key], b[key]) for key in ("perm", "inv_row", "drop", "offsets"))


def test_fallback_layer_adds_the_fallback_expert_for_dropped_slots():
    # y(fallback) = y(drop) + sum over dropped slots of g * E_N(x), E_N by numpy
    wl = synth.Workload("fb", T=96, d=32, N=4, k=2, H=48, act="swiglu", dtype="f32",
                        gate_mode="R", capacity_factor=0.6, overflow="fallback", seed=9)
    host = synth.make_host(wl)
    ref_fb = oracle.route(wl, host["x"], host["Wg"])
    ref_dr = oracle.route(wl.with_(overflow="drop"), host["x"], host["Wg"])
    assert ref_dr["drop"].sum() > 0
    toks = np.arange(wl.T)
    y_fb = oracle.forward_rows(wl, host, ref_fb, toks)
    y_dr = oracle.forward_rows(wl.with_(overflow="drop"), host, ref_dr, toks)
    x = oracle.decode(host["x"])
    W1, W3, W2 = (oracle.decode(host[n])[wl.N] for n in ("W1", "W3", "W2"))
    h = scipy.special.expit(x @ W1.T) * (x @ W1.T) * (x @ W3.T)
    e_fb = h @ W2.T
    dropped = ref_dr["drop"].reshape(wl.T, wl.k).astype(bool)
    extra = (ref_dr["gate"] * dropped).sum(1)[:, None] * e_fb
    np.testing.assert_allclose(y_fb, y_dr + extra, rtol=1e-10, atol=1e-12)


def test_capacity_uses_the_fp32_capacity_factor():
    # The layer configuration carries the capacity factor in fp32.  0.7 is not a
    # binary fraction: its nearest fp32 value is 11744051 / 2^24 (the 24-bit
    # significand 0.7 * 2^24 = 11744051.2 rounded to the nearest integer), i.e.
    # 0.699999988079071044921875.  So with T = 400 and N = 8,
    # C = floor(11744051 * 400 / (8 * 2^24)) = floor(34.99999964...) = 34, not 35.
    from fractions import Fraction
    cf32 = Fraction(11744051, 1 << 24)
    assert abs(cf32 - Fraction(7, 10)) < Fraction(1, 1 << 25)      # the nearest fp32 value
    assert str(float(cf32)) == "0.699999988079071"
    assert cf32 * 400 / 8 < 35 and int(cf32 * 400 / 8) == 34
    wl = synth.Workload("c", T=400, d=8, N=8, k=1, H=8, act="relu", dtype="f32", gate_mode="R",
                        capacity_factor=0.7)
    assert wl.capacity() == 34
    idx = np.zeros((400, 1), np.int32)                 # every token on expert 0
    ref = oracle.dispatch(idx, 8, 0.7)
    assert ref["kept"][0] == 34 and ref["R"] == 34
    assert oracle.dispatch(idx, 8, 0.75)["kept"][0] == 37    # exact in fp32: floor(37.5)
