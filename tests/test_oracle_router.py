"""Pins for the oracle's router: logits, top-k order, gate weights in both modes.

Each check compares the oracle with something other than its own formula:
a library matmul, a brute-force stable sort, a closed form, or a special case
that reduces to a library softmax.
"""
import numpy as np
import pytest
import scipy.special

import oracle
import synth


def _rand(seed, shape, std=1.0, dt="f32"):
    n = int(np.prod(shape))
    return synth.normal(seed, 11, n, std, dt).reshape(shape)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_logits_match_library_matmul(dt):
    x = _rand(1, (37, 48), 1.0, dt)
    Wg = synth.normal(2, 12, 9 * 48, 0.2, dt).reshape(9, 48)
    bias = synth.normal(3, 13, 9, 1.5, "f32")
    got = oracle.router_logits(x, Wg, bias)
    ref = oracle.decode(x) @ oracle.decode(Wg).T + bias.astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # token sub-range
    part = oracle.router_logits(x, Wg, bias, t0=5, t1=20)
    assert np.array_equal(part, got[5:20])


@pytest.mark.parametrize("N,k", [(1, 1), (4, 2), (8, 2), (16, 1), (16, 5), (16, 16), (7, 7)])
def test_topk_equals_bruteforce_stable_sort_with_ties(N, k):
    T, d = 64, 8
    x = _rand(4, (T, d))
    Wg = synth.normal(5, 14, N * d, 0.5, "f32").reshape(N, d)
    # inject exact ties: duplicated router rows give bitwise-equal logits
    if N >= 4:
        Wg[N - 1] = Wg[0]
        Wg[2] = Wg[1]
    # and whole tokens of equal logits
    x[3] = 0.0
    logits = oracle.router_logits(x, Wg)
    idx, gate, probs = oracle.topk_gate(logits, k, "R")
    for t in range(T):
        order = sorted(range(N), key=lambda e: (-logits[t, e], e))   # brute force
        assert idx[t].tolist() == order[:k]
    # the all-zero token: every logit equals 0, so the lowest indices win
    assert idx[3].tolist() == list(range(k))
    if N >= 4 and k >= 2:
        # a duplicated pair, when both selected, appears lower index first
        for t in range(T):
            row = idx[t].tolist()
            if 0 in row and N - 1 in row:
                assert row.index(0) < row.index(N - 1)


def test_mode_r_sums_to_one_and_k2_closed_form():
    T, N, d = 200, 8, 16
    logits = oracle.router_logits(_rand(6, (T, d)), synth.normal(7, 15, N * d, 0.7, "f32").reshape(N, d))
    idx, gate, _ = oracle.topk_gate(logits, 2, "R")
    assert np.max(np.abs(gate.sum(1) - 1.0)) < 1e-15
    l1 = logits[np.arange(T), idx[:, 0]]
    l2 = logits[np.arange(T), idx[:, 1]]
    # top-2 sparse softmax: second weight = 1 / (1 + e^(l1 - l2))
    np.testing.assert_allclose(gate[:, 1], 1.0 / (1.0 + np.exp(l1 - l2)), rtol=1e-14)
    np.testing.assert_allclose(gate[:, 0], 1.0 / (1.0 + np.exp(l2 - l1)), rtol=1e-14)
    assert np.all(gate[:, 0] >= gate[:, 1])


def test_mode_r_with_k_equal_n_is_full_softmax():
    T, N, d = 50, 6, 12
    logits = oracle.router_logits(_rand(8, (T, d)), synth.normal(9, 16, N * d, 1.0, "f32").reshape(N, d))
    idx, gate, probs = oracle.topk_gate(logits, N, "R")
    ref = scipy.special.softmax(logits, axis=1)
    np.testing.assert_allclose(probs, ref, rtol=1e-13)
    np.testing.assert_allclose(gate, np.take_along_axis(ref, idx, 1), rtol=1e-13)


def test_mode_f_unnormalised_and_renormalised():
    T, N, d, k = 80, 32, 16, 4
    logits = oracle.router_logits(_rand(10, (T, d)), synth.normal(11, 17, N * d, 1.0, "f32").reshape(N, d))
    ref = scipy.special.softmax(logits, axis=1)
    idx, gate, probs = oracle.topk_gate(logits, k, "F", renormalize=False)
    np.testing.assert_allclose(gate, np.take_along_axis(ref, idx, 1), rtol=1e-13)
    assert np.all(gate.sum(1) < 1.0)
    idx2, gate2, _ = oracle.topk_gate(logits, k, "F", renormalize=True)
    idxr, gater, _ = oracle.topk_gate(logits, k, "R")
    assert np.array_equal(idx2, idx) and np.array_equal(idxr, idx)
    # renormalised full softmax restricted to the top-k equals the sparse softmax
    assert np.max(np.abs(gate2 - gater)) < 1e-15


def test_switch_style_top1_weight_is_pmax_not_one():
    logits = np.array([[0.0, 1.0, 2.0, -1.0]])
    idx, gate, _ = oracle.topk_gate(logits, 1, "F")
    assert idx[0, 0] == 2
    p = np.exp([0.0, 1.0, 2.0, -1.0])
    assert abs(gate[0, 0] - p[2] / p.sum()) < 1e-15
    _, gate_r, _ = oracle.topk_gate(logits, 1, "R")
    assert gate_r[0, 0] == 1.0


# ---------------------------------------------------------------- node-limited routing
def _golden(name):
    vals = {}
    with open(__file__.rsplit("/", 1)[0] + "/golden/" + name) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, v = line.split(":", 1)
            vals[key.strip()] = [float(a) for a in v.split()]
    return vals


def test_node_limited_worked_example():
    g = _golden("node_limited_example.txt")
    logits = np.array([g["logits"]])
    k, ng, tg = int(g["k"][0]), int(g["n_groups"][0]), int(g["topk_groups"][0])
    idx, gate, _ = oracle.topk_gate(logits, k, "F", renormalize=True, n_groups=ng, topk_groups=tg)
    assert idx[0].tolist() == [int(v) for v in g["expect_idx"]]
    plain, _, _ = oracle.topk_gate(logits, k, "F", renormalize=True)
    assert plain[0].tolist() == [int(v) for v in g["plain_idx"]]
    # renormalised gates are the softmax of the selected logits (library routine)
    np.testing.assert_allclose(gate[0], scipy.special.softmax(logits[0, idx[0]]), rtol=1e-14)
    # mode R picks the same experts with the same weights
    idx_r, gate_r, _ = oracle.topk_gate(logits, k, "R", n_groups=ng, topk_groups=tg)
    assert np.array_equal(idx_r, idx)
    np.testing.assert_allclose(gate_r, gate, rtol=1e-14)


@pytest.mark.parametrize("mode,renorm", [("R", False), ("F", False), ("F", True)])
def test_node_limited_reduces_to_plain_topk(mode, renorm):
    T, N, k = 200, 32, 4
    logits = _rand(31, (T, N), 2.0).astype(np.float64)
    logits[:, 7] = logits[:, 3]                      # exact ties across nodes
    ref = oracle.topk_gate(logits, k, mode, renorm)
    for ng, tg in [(1, 1), (4, 4), (8, 8), (N, k), (N, N)]:
        # one node, every node allowed, or one expert per node with M >= k
        got = oracle.topk_gate(logits, k, mode, renorm, n_groups=ng, topk_groups=tg)
        for a, b in zip(got, ref):
            assert np.array_equal(a, b), (ng, tg)


def test_node_limited_deepseek_shape_invariants():
    # 256 experts on 8 nodes of 32, top-8 from at most 4 nodes (the DeepSeek-V3
    # setting the page describes)
    T, N, k, ng, tg = 300, 256, 8, 8, 4
    logits = _rand(32, (T, N), 1.0).astype(np.float64)
    idx, gate, probs = oracle.topk_gate(logits, k, "F", True, n_groups=ng, topk_groups=tg)
    plain, _, probs0 = oracle.topk_gate(logits, k, "F", True)
    assert np.array_equal(probs, probs0)             # aux probabilities over all N, unchanged
    nodes = idx // (N // ng)
    assert all(len(set(r)) <= tg for r in nodes.tolist())
    np.testing.assert_allclose(gate.sum(1), 1.0, rtol=1e-14)
    # slot order: descending logit, distinct experts
    sel = np.take_along_axis(logits, idx, 1)
    assert np.all(np.diff(sel, axis=1) <= 0)
    assert all(len(set(r)) == k for r in idx.tolist())
    # the chosen experts are the k best of the chosen nodes (library sort)
    for t in range(T):
        allowed = np.isin(np.arange(N) // (N // ng), np.unique(nodes[t]))
        cand = np.where(allowed)[0]
        best = cand[np.lexsort((cand, -logits[t, cand]))][:k]
        assert idx[t].tolist() == best.tolist()
    # the limit binds for a good share of tokens
    assert np.mean([len(set(r)) > tg for r in (plain // (N // ng)).tolist()]) > 0.2
