"""Pins against values the pages print (tests/golden/, each file cites its passage)."""
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


def test_dispatch_payload_bytes_per_token():
    # The oracle's dispatch of a DeepSeek-V3-shaped micro-batch (k = 8, d = 7168,
    # no capacity limit) produces k rows per token; bytes = rows * d * s.
    wl = synth.DEEPSEEK
    for k, d, s, per_tok, tokens, per_mb in (map(int, r) for r in _rows("payload_bytes.txt")):
        assert (k, d) == (wl.k, wl.d)
        idx = synth.synthetic_topk(0, tokens, wl.N, k)
        disp = oracle.dispatch(idx, wl.N, 0.0)
        one = oracle.dispatch(idx[:1], wl.N, 0.0)
        assert one["R"] * d * s == per_tok
        assert disp["R"] * d * s == per_mb
        assert per_mb == 448 * 2 ** 20 // (2 // s)
    # the FP8 payload with its fp32 per-token scale
    q, sc = oracle.quantize_rows(synth.normal(3, 0, 2 * wl.d, 1.0, "bf16").reshape(2, wl.d))
    assert q[0].nbytes * wl.k == 57344 and sc.itemsize == 4


def test_experts_touched_matches_worked_example():
    # Uniform random router logits; share of experts with a kept token in a step
    # of B tokens, averaged over many steps, against the page's three values.
    rows = [(int(N), int(k), int(B), float(v)) for N, k, B, v in _rows("experts_touched.txt")]
    rng_seed = 100
    for N, k, B, share in rows:
        trials = 4000 if B == 1 else (400 if B == 32 else 200)
        got = []
        for i in range(trials):
            logits = synth.normal(rng_seed + i, 30 + B, B * N, 1.0, "f32").reshape(B, N).astype(np.float64)
            idx, _, _ = oracle.topk_gate(logits, k, "R")
            disp = oracle.dispatch(idx, N, 0.0)
            got.append(np.count_nonzero(disp["kept"]) / N)
        mean = float(np.mean(got))
        sem = float(np.std(got) / np.sqrt(trials)) + 1e-4
        assert abs(mean - share) < 4 * sem + 5e-4, (N, k, B, mean, share)
