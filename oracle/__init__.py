"""CPU oracle for the MoE layer forward (fp64, plain loops).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The GPU
path never imports it and shares no code with it; the two meet only through
the seeded inputs of ``synth``.

The arithmetic lives in ``moe_oracle.c`` (each function there names the page
passage it follows); this module marshals numpy arrays into it.

Pages followed:
  * "moe communication costs" - Router design (G(x), combine), Load balancing
    (L_aux), Capacity factor and token dropping.
  * "Advanced GPU Optimization: How to tech an LLM with CUDA and ROCm? - Part 5"
    section 1.1 (top-2 router, sparse softmax, earliest index wins ties).
  * "MoE: what it costs to train and serve" - Expert parallelism (dispatch /
    experts / combine), bytes-per-token worked example (FP8 payload),
    experts-touched worked example, Numerical precision.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1
GATE_R, GATE_F = 0, 1
RELU, SWIGLU = 0, 1

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_f64 = ctypes.c_double


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "moe_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        # -ffp-contract=off: no fused multiply-add, every operation rounds as written
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                               "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.orc_router_logits.argtypes = [_i64, _i64, _i32, _i32, _p, _i32, _p, _i32, _p, _p]
        lib.orc_topk_gate.argtypes = [_i64, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _i32, _i32]
        lib.orc_dispatch.argtypes = [_i64, _i32, _i32, _f64, _p, _p, _p, _p, _p, _p, _p, _i32, _i32, _p]
        lib.orc_dispatch.restype = _i64
        lib.orc_aux.argtypes = [_i64, _i32, _i32, _f64, _p, _p, _p, _p, _p]
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = _f64
        lib.orc_e4m3_encode.argtypes = [_f64]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_quantize_rows.argtypes = [_i64, _i32, _p, _i32, _p, _p]
        lib.orc_ffn_row.argtypes = [_i32, _i32, _i32, _p, _p, _p, _p, _i32, _p]
        lib.orc_layer_rows.argtypes = [_i64, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p,
                                       _p, _p, _p, _i32, _p, _p, _p, _p]
        for f in ("orc_router_logits", "orc_topk_gate", "orc_aux", "orc_quantize_rows",
                  "orc_ffn_row", "orc_layer_rows"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")


def _c(a):
    return np.ascontiguousarray(a)


def decode(a: np.ndarray) -> np.ndarray:
    """Exact fp64 value of stored float32 / bf16-bit arrays."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------- router
def router_logits(x: np.ndarray, Wg: np.ndarray, bias: np.ndarray | None = None,
                  t0: int = 0, t1: int | None = None) -> np.ndarray:
    """fp64 logits [t1-t0, N] = x W_g^T (+ bias) (page 5, Router design)."""
    x, Wg = _c(x), _c(Wg)
    T, d = x.shape
    N = Wg.shape[0]
    t1 = T if t1 is None else t1
    out = np.empty((t1 - t0, N), dtype=np.float64)
    b = None
    if bias is not None:
        bias = _c(bias.astype(np.float32))
        b = bias.ctypes.data
    _load().orc_router_logits(t0, t1, d, N, x.ctypes.data, _dt(x), Wg.ctypes.data, _dt(Wg), b,
                              out.ctypes.data)
    return out


def topk_gate(logits: np.ndarray, k: int, gate_mode: str, renormalize: bool = False,
              n_groups: int = 0, topk_groups: int = 0):
    """(idx [T,k] int32, gate [T,k] fp64, probs [T,N] fp64) from fp64 logits.

    n_groups > 1 and topk_groups < n_groups: node-limited routing ("MoE: what it
    costs to train and serve", Limit how many machines a token touches) -- the
    top-k is taken among the experts of the topk_groups nodes (blocks of
    N / n_groups consecutive experts) with the largest sums of their
    ceil(k / topk_groups) highest router probabilities."""
    logits = _c(logits.astype(np.float64))
    T, N = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float64)
    probs = np.empty((T, N), dtype=np.float64)
    if n_groups > 1 and topk_groups < n_groups:
        assert N % n_groups == 0 and 1 <= topk_groups and k <= topk_groups * (N // n_groups)
    _load().orc_topk_gate(T, N, k, GATE_R if gate_mode == "R" else GATE_F, int(renormalize),
                          logits.ctypes.data, idx.ctypes.data, gate.ctypes.data, probs.ctypes.data,
                          int(n_groups), int(topk_groups))
    return idx, gate, probs


# ------------------------------------------------------------------- dispatch
def dispatch(idx: np.ndarray, N: int, capacity_factor: float, fallback: bool = False,
             slot_priority: bool = False) -> dict:
    """Local permutation: counts, kept, offsets, perm, inv_row, drop, R, expert.

    fallback: pairs over capacity go to a fallback expert N (offsets gets N + 2
    entries) instead of being dropped; slot_priority: pairs are taken slot by
    slot (every token's first choice first) instead of token by token
    ("moe communication costs", Capacity factor and token dropping)."""
    idx = _c(idx.astype(np.int32))
    T, k = idx.shape
    # the capacity factor is the fp32 value a layer configuration carries:
    # C = floor(cf * T / N) with cf rounded to fp32 (e.g. 0.7 -> 0.69999999,
    # so 0.7 * 400 / 8 gives C = 34)
    capacity_factor = float(np.float32(capacity_factor))
    counts = np.empty(N, np.int32)
    kept = np.empty(N, np.int32)
    offsets = np.empty(N + 2 if fallback else N + 1, np.int32)
    perm = np.full(T * k, -1, np.int32)
    inv_row = np.empty(T * k, np.int32)
    drop = np.empty(T * k, np.uint8)
    expert = np.empty(T * k, np.int32)
    R = _load().orc_dispatch(T, N, k, float(capacity_factor), idx.ctypes.data, counts.ctypes.data,
                             kept.ctypes.data, offsets.ctypes.data, perm.ctypes.data,
                             inv_row.ctypes.data, drop.ctypes.data, int(bool(fallback)),
                             int(bool(slot_priority)), expert.ctypes.data)
    return dict(counts=counts, kept=kept, offsets=offsets, perm=perm[:R], inv_row=inv_row,
                drop=drop, R=int(R), expert=expert)


def aux(counts: np.ndarray, probs: np.ndarray, k: int, alpha: float):
    """(f [N], p_mean [N], L_aux) (page 5, Load balancing)."""
    probs = _c(probs.astype(np.float64))
    T, N = probs.shape
    counts = _c(counts.astype(np.int32))
    f = np.empty(N)
    pm = np.empty(N)
    laux = np.zeros(1)
    _load().orc_aux(T, N, k, float(alpha), counts.ctypes.data, probs.ctypes.data, f.ctypes.data,
                    pm.ctypes.data, laux.ctypes.data)
    return f, pm, float(laux[0])


# ------------------------------------------------------------------------ FP8
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.orc_e4m3_decode(int(v)) for v in c]).reshape(np.shape(codes))


def e4m3_encode(values: np.ndarray) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64).ravel()
    return np.array([lib.orc_e4m3_encode(float(a)) for a in v], dtype=np.uint8).reshape(np.shape(values))


_E4M3_TABLE = None


def e4m3_table() -> np.ndarray:
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = e4m3_decode(np.arange(256, dtype=np.uint8))
    return _E4M3_TABLE


def quantize_rows(x: np.ndarray):
    """Per-row FP8 payload: (codes [n,d] uint8, scale [n] float32)."""
    x = _c(x)
    n, d = x.shape
    q = np.empty((n, d), np.uint8)
    s = np.empty(n, np.float32)
    _load().orc_quantize_rows(n, d, x.ctypes.data, _dt(x), q.ctypes.data, s.ctypes.data)
    return q, s


def dequantize_rows(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    return e4m3_table()[q] * s.astype(np.float64)[:, None]


# ------------------------------------------------------------------------ FFN
def ffn_row(xrow: np.ndarray, W1e, W3e, W2e, act: str) -> np.ndarray:
    """One expert on one fp64 row; W1e/W3e [H,d], W2e [d,H] stored arrays."""
    xrow = _c(np.asarray(xrow, np.float64))
    d = xrow.shape[0]
    W1e, W2e = _c(W1e), _c(W2e)
    H = W1e.shape[0]
    W3p = None
    if act == "swiglu":
        W3e = _c(W3e)
        W3p = W3e.ctypes.data
    y = np.empty(d)
    _load().orc_ffn_row(d, H, RELU if act == "relu" else SWIGLU, xrow.ctypes.data, W1e.ctypes.data,
                        W3p, W2e.ctypes.data, _dt(W1e), y.ctypes.data)
    return y


def layer_rows(act: str, xin: np.ndarray, idx: np.ndarray, gate: np.ndarray, drop: np.ndarray,
               W1, W3, W2, xsh=None, Ws1=None, Ws3=None, Ws2=None) -> np.ndarray:
    """y rows [n, d] for n tokens given their expert inputs and routing (fp64).

    W1/W3/W2 are stacked over experts as in ``synth``; idx indexes them.
    """
    xin = _c(np.asarray(xin, np.float64))
    n, d = xin.shape
    k = idx.shape[1]
    W1, W2 = _c(W1), _c(W2)
    H = W1.shape[1]
    idx = _c(idx.astype(np.int32))
    gate = _c(gate.astype(np.float64))
    drop = _c(drop.astype(np.uint8))
    Hs = 0
    xshp = ws1 = ws3 = ws2 = None
    keep = []
    if Ws1 is not None:
        Hs = Ws1.shape[0]
        xsh = _c(np.asarray(xsh, np.float64))
        Ws1c, Ws2c = _c(Ws1), _c(Ws2)
        keep += [xsh, Ws1c, Ws2c]
        xshp, ws1, ws2 = xsh.ctypes.data, Ws1c.ctypes.data, Ws2c.ctypes.data
        if act == "swiglu":
            Ws3c = _c(Ws3)
            keep.append(Ws3c)
            ws3 = Ws3c.ctypes.data
    W3c = _c(W3) if act == "swiglu" else None
    w3p = W3c.ctypes.data if W3c is not None else None
    y = np.empty((n, d))
    _load().orc_layer_rows(n, d, H, k, RELU if act == "relu" else SWIGLU, _dt(W1), xin.ctypes.data,
                           xshp, idx.ctypes.data, gate.ctypes.data, drop.ctypes.data, W1.ctypes.data,
                           w3p, W2.ctypes.data, Hs, ws1, ws3, ws2, y.ctypes.data)
    return y


# ------------------------------------------------------------- whole routing
def route(wl, x: np.ndarray, Wg: np.ndarray, bias=None) -> dict:
    """Router + top-k + aux + dispatch for every token of workload ``wl``."""
    logits = router_logits(x, Wg, bias)
    idx, gate, probs = topk_gate(logits, wl.k, wl.gate_mode, wl.renormalize,
                                 wl.n_groups, wl.topk_groups)
    disp = dispatch(idx, wl.N, wl.capacity_factor, wl.overflow == "fallback", wl.slot_priority)
    f, pm, laux = aux(disp["counts"], probs, wl.k, wl.aux_alpha)
    out = dict(logits=logits, idx=idx, gate=gate, probs=probs, f=f, p_mean=pm, L_aux=laux)
    out.update(disp)
    return out


def expert_inputs(wl, x_rows: np.ndarray):
    """fp64 expert-input rows for the given token rows (dequantised FP8 payload if so configured)."""
    if wl.dispatch_dtype == "fp8":
        q, s = quantize_rows(x_rows)
        return dequantize_rows(q, s)
    return decode(x_rows)


def _effective_experts(wl, routing: dict) -> np.ndarray:
    """[T, k] expert each pair runs on (the fallback N for re-routed pairs)."""
    if "expert" not in routing:
        return routing["idx"]
    return np.where(routing["drop"].reshape(wl.T, wl.k) != 0, routing["idx"],
                    routing["expert"].reshape(wl.T, wl.k)).astype(np.int32)


def forward_rows(wl, inputs: dict, routing: dict, tokens) -> np.ndarray:
    """Layer output y [len(tokens), d] in fp64 for the listed tokens."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x = inputs["x"]
    xr = x[tokens]
    xin = expert_inputs(wl, xr)
    # the expert each (token, slot) pair runs on: its own, or the fallback
    idx = _effective_experts(wl, routing)[tokens]
    gate = routing["gate"][tokens]
    drop = routing["drop"].reshape(wl.T, wl.k)[tokens]
    W1, W2 = inputs["W1"], inputs["W2"]
    W3 = inputs.get("W3")
    sh = {}
    if wl.H_shared > 0:
        sh = dict(xsh=decode(xr), Ws1=inputs["Ws1"], Ws3=inputs.get("Ws3"), Ws2=inputs["Ws2"])
    return layer_rows(wl.act, xin, idx, gate, drop, W1, W3, W2, **sh)


def forward_rows_lazy(wl, x: np.ndarray, routing: dict, tokens, get_expert, shared=None) -> np.ndarray:
    """Like ``forward_rows`` but fetches expert weights one expert at a time.

    ``get_expert(e)`` returns (W1e [H,d], W3e or None, W2e [d,H]); used when the
    stacked weights are too large to hold on the host.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    xr = x[tokens]
    xin = expert_inputs(wl, xr)
    idx = _effective_experts(wl, routing)[tokens]
    gate = routing["gate"][tokens]
    drop = routing["drop"].reshape(wl.T, wl.k)[tokens]
    used = sorted(set(int(e) for e, dr in zip(idx.ravel(), drop.ravel()) if not dr))
    remap = {e: i for i, e in enumerate(used)}
    if not used:
        used, remap = [0], {0: 0}
    ws = [get_expert(e) for e in used]
    W1 = np.stack([w[0] for w in ws])
    W3 = np.stack([w[1] for w in ws]) if wl.act == "swiglu" else None
    W2 = np.stack([w[2] for w in ws])
    lidx = np.vectorize(lambda e: remap.get(int(e), 0))(idx).astype(np.int32)
    sh = {}
    if shared is not None:
        sh = dict(xsh=decode(xr), Ws1=shared[0], Ws3=shared[1], Ws2=shared[2])
    return layer_rows(wl.act, xin, lidx, gate, drop, W1, W3, W2, **sh)


def forward_rows_by_expert(wl, x: np.ndarray, routing: dict, tokens, get_expert,
                           shared=None) -> np.ndarray:
    """Layer output y [len(tokens), d] in fp64, the same sum as ``forward_rows``,
    y_t = sum over kept slots j of g_tj * E_e(t,j)(x_t) (+ shared(x_t))
    ("moe communication costs", Router design), evaluated expert by expert so
    that only one expert's weights are held at a time: each expert's pairs go
    through ``layer_rows`` as one-slot rows with weight 1, then the slots are
    weighed and summed in slot order, then the shared expert is added.
    ``get_expert(e)`` returns (W1e [H,d], W3e or None, W2e [d,H])."""
    tokens = np.asarray(tokens, dtype=np.int64)
    n, k, d = len(tokens), wl.k, wl.d
    xr = x[tokens]
    xin = expert_inputs(wl, xr)
    idx = _effective_experts(wl, routing)[tokens]
    gate = routing["gate"][tokens]
    drop = routing["drop"].reshape(wl.T, wl.k)[tokens]
    Y = np.zeros((n, k, d))
    live = drop == 0
    for e in sorted(set(int(v) for v in idx[live].ravel())):
        sel = np.argwhere((idx == e) & live)            # (position in tokens, slot)
        W1e, W3e, W2e = get_expert(e)
        m = len(sel)
        Y[sel[:, 0], sel[:, 1]] = layer_rows(
            wl.act, xin[sel[:, 0]], np.zeros((m, 1), np.int32), np.ones((m, 1)),
            np.zeros((m, 1), np.uint8), W1e[None], None if W3e is None else W3e[None], W2e[None])
    y = np.zeros((n, d))
    for j in range(k):
        y[live[:, j]] += gate[live[:, j], j, None] * Y[live[:, j], j]
    if shared is not None:
        Ws1, Ws3, Ws2 = shared
        # every routed slot marked dropped: layer_rows then returns the shared expert alone
        y += layer_rows(wl.act, np.zeros((n, d)), np.zeros((n, 1), np.int32), np.zeros((n, 1)),
                        np.ones((n, 1), np.uint8), Ws1[None], None if Ws3 is None else Ws3[None],
                        Ws2[None], xsh=decode(xr), Ws1=Ws1, Ws3=Ws3, Ws2=Ws2)
    return y


def combine(y_rows: np.ndarray, inv_row: np.ndarray, gate: np.ndarray, y_shared=None) -> np.ndarray:
    """y[t] = sum over kept slots j of gate[t,j] * y_rows[inv_row[t*k+j]] (+ y_shared[t]).

    "moe communication costs", Router design (weighted sum over the selected
    experts); a dropped slot (inv_row = -1) contributes nothing.  fp64.
    """
    y_rows = np.asarray(y_rows, dtype=np.float64)
    T, k = gate.shape
    d = y_rows.shape[1]
    rows = np.asarray(inv_row).reshape(T, k)
    y = np.zeros((T, d))
    for j in range(k):
        m = rows[:, j] >= 0
        y[m] += gate[m, j, None] * y_rows[rows[m, j]]
    if y_shared is not None:
        y += np.asarray(y_shared, dtype=np.float64)
    return y
