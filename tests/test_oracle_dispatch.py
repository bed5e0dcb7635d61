"""Pins for the oracle's dispatch (counts, capacity, permutation) and aux statistics."""
import math

import numpy as np
import pytest

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
