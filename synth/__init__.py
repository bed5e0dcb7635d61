"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

Holds no arithmetic of the MoE method: only the counter-based normal generator
(SplitMix64 + Box-Muller, see ``synth.c``) and the five workload shapes.

Storage layouts (all row-major, experts stacked on the leading axis):

* ``x``    ``[T, d]``        tokens
* ``Wg``   ``[N, d]``        router matrix W_g (page 5 "Router design")
* ``bias`` ``[N]`` fp32      per-expert logit bias (Switch-shaped workload only)
* ``W1``, ``W3`` ``[N, H, d]`` row ``h`` of expert ``e`` is column ``h`` of the
  d x H matrix that multiplies ``x`` (so the reduction axis d is contiguous)
* ``W2``   ``[N, d, H]``     row ``i`` of expert ``e`` is column ``i`` of the H x d matrix
* ``Ws1``, ``Ws3`` ``[Hs, d]``, ``Ws2`` ``[d, Hs]`` the always-on shared expert.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None

TENSOR_IDS = {"x": 0, "Wg": 1, "bias": 2, "W1": 3, "W3": 4, "W2": 5,
              "Ws1": 6, "Ws3": 7, "Ws2": 8, "topk": 9}


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_double, ctypes.c_int, ctypes.c_void_p]
        lib.synth_normal.restype = None
        lib.synth_uniform_int.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p]
        lib.synth_uniform_int.restype = None
        lib.synth_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_u64.restype = ctypes.c_uint64
        _lib = lib
    return _lib


def u64(seed: int, tensor_id: int, n: int) -> int:
    """Raw SplitMix64 output ``n`` (n >= 1) of stream (seed, tensor_id)."""
    return int(_load().synth_u64(seed, tensor_id, n))


def normal(seed: int, tensor_id: int, count: int, stddev: float, dtype: str,
           start: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """Elements [start, start+count) of tensor (seed, tensor_id) scaled by ``stddev``.

    ``dtype`` "f32" returns float32, "bf16" returns the bf16 bit patterns as uint16.
    """
    npdt = np.float32 if dtype == "f32" else np.uint16
    if out is None:
        out = np.empty(count, dtype=npdt)
    assert out.dtype == npdt and out.size >= count and out.flags["C_CONTIGUOUS"]
    _load().synth_normal(seed, tensor_id, start, count, float(stddev),
                         0 if dtype == "f32" else 1, out.ctypes.data)
    return out


def uniform_int(seed: int, tensor_id: int, count: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.int32)
    _load().synth_uniform_int(seed, tensor_id, start, count, n, out.ctypes.data)
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic MoE layer: shapes, routing mode, dtypes and seed."""
    name: str
    T: int
    d: int
    N: int
    k: int
    H: int
    act: str            # "relu" | "swiglu"
    dtype: str          # "f32" | "bf16"   (x, weights, y)
    gate_mode: str      # "R": softmax over the top-k logits; "F": full softmax then top-k
    renormalize: bool = False   # mode F only: divide the k selected probabilities by their sum
    capacity_factor: float = 0.0  # <= 0: no capacity limit
    H_shared: int = 0
    dispatch: str = ""  # "" = same as dtype, "fp8" = e4m3 codes + per-token fp32 scale
    aux_alpha: float = 0.01
    bias_std: float = 0.0   # > 0: per-expert logit bias ~ N(0, bias_std^2)
    seed: int = 0
    n_groups: int = 0       # > 1: experts on n_groups nodes of N / n_groups consecutive experts
    topk_groups: int = 0    # ... and a token may use at most topk_groups of them
    overflow: str = "drop"  # pairs over capacity: "drop", or "fallback" to expert N
    slot_priority: bool = False   # capacity filled slot by slot (first choices first)

    @property
    def n_stored(self) -> int:
        """Expert blocks in W1/W3/W2: the N routed experts (+ the fallback)."""
        return self.N + (1 if self.overflow == "fallback" else 0)

    @property
    def dispatch_dtype(self) -> str:
        return self.dispatch or self.dtype

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def capacity(self) -> int:
        """C = floor(capacity_factor * T / N), or -1 when unlimited (page 5)."""
        if self.capacity_factor <= 0:
            return -1
        # the factor as the fp32 value the layer configuration carries
        return int(math.floor(float(np.float32(self.capacity_factor)) * self.T / self.N))


# The five workloads.  Names say what they are shaped like.
TINY_F32 = Workload("tiny-fp32 T256 d64 N8 k2 H128 relu", T=256, d=64, N=8, k=2, H=128,
                    act="relu", dtype="f32", gate_mode="R", seed=0)
MIXTRAL = Workload("mixtral-shaped T4096 d4096 N8 k2 H14336 swiglu bf16", T=4096, d=4096, N=8, k=2,
                   H=14336, act="swiglu", dtype="bf16", gate_mode="R", seed=1)
SWITCH = Workload("switch-shaped T8192 d1024 N128 k1 H4096 relu bf16 cf1.25", T=8192, d=1024, N=128,
                  k=1, H=4096, act="relu", dtype="bf16", gate_mode="F", capacity_factor=1.25,
                  aux_alpha=0.01, bias_std=math.sqrt(2.0), seed=2)
DEEPSEEK = Workload("deepseek-v3-shaped T4096 d7168 N256+1 k8 H2048 swiglu bf16 fp8-dispatch",
                    T=4096, d=7168, N=256, k=8, H=2048, act="swiglu", dtype="bf16", gate_mode="F",
                    renormalize=True, H_shared=2048, dispatch="fp8", seed=3)
GROK = Workload("grok1-shaped decode T32 d6144 N8 k2 H32768 swiglu bf16", T=32, d=6144, N=8, k=2,
                H=32768, act="swiglu", dtype="bf16", gate_mode="R", seed=4)

# The DeepSeek-shaped layer with node-limited routing: 8 nodes of 32 experts,
# at most 4 nodes per token ("MoE: what it costs to train and serve", Limit how
# many machines a token touches).
DEEPSEEK_NODE_LIMITED = DEEPSEEK.with_(
    name="deepseek-v3-shaped node-limited (8 nodes x 32 experts, <= 4 nodes per token)",
    n_groups=8, topk_groups=4)

# The Switch-shaped layer with its overflow re-routed to a fallback expert
# instead of dropped ("moe communication costs", Capacity factor and token
# dropping).
SWITCH_FALLBACK = SWITCH.with_(
    name="switch-shaped T8192 d1024 N128+fallback k1 H4096 relu bf16 cf1.25, overflow to a fallback expert",
    overflow="fallback")

WORKLOADS = {"tiny": TINY_F32, "mixtral": MIXTRAL, "switch": SWITCH, "deepseek": DEEPSEEK, "grok": GROK,
             "deepseek-nl": DEEPSEEK_NODE_LIMITED, "switch-fb": SWITCH_FALLBACK}


def tensor_specs(wl: Workload):
    """(name, shape, stddev, dtype) of every input tensor of ``wl``."""
    specs = [("x", (wl.T, wl.d), 1.0, wl.dtype),
             ("Wg", (wl.N, wl.d), 1.0 / math.sqrt(wl.d), wl.dtype)]
    if wl.bias_std > 0:
        specs.append(("bias", (wl.N,), wl.bias_std, "f32"))
    E = wl.n_stored
    specs.append(("W1", (E, wl.H, wl.d), 1.0 / math.sqrt(wl.d), wl.dtype))
    if wl.act == "swiglu":
        specs.append(("W3", (E, wl.H, wl.d), 1.0 / math.sqrt(wl.d), wl.dtype))
    specs.append(("W2", (E, wl.d, wl.H), 1.0 / math.sqrt(wl.H), wl.dtype))
    if wl.H_shared > 0:
        specs.append(("Ws1", (wl.H_shared, wl.d), 1.0 / math.sqrt(wl.d), wl.dtype))
        if wl.act == "swiglu":
            specs.append(("Ws3", (wl.H_shared, wl.d), 1.0 / math.sqrt(wl.d), wl.dtype))
        specs.append(("Ws2", (wl.d, wl.H_shared), 1.0 / math.sqrt(wl.H_shared), wl.dtype))
    return specs


def make_host(wl: Workload, names=None) -> dict:
    """Generate the named input tensors on the host as numpy arrays (bf16 as uint16 bits)."""
    out = {}
    for name, shape, std, dt in tensor_specs(wl):
        if names is not None and name not in names:
            continue
        n = int(np.prod(shape))
        out[name] = normal(wl.seed, TENSOR_IDS[name], n, std, dt).reshape(shape)
    return out


def expert_slice(wl: Workload, name: str, e: int) -> np.ndarray:
    """Regenerate only expert ``e`` of a stacked weight (``W1``, ``W3`` or ``W2``)."""
    spec = {s[0]: s for s in tensor_specs(wl)}[name]
    _, shape, std, dt = spec
    per = int(np.prod(shape[1:]))
    return normal(wl.seed, TENSOR_IDS[name], per, std, dt, start=e * per).reshape(shape[1:])


def synthetic_topk(seed: int, T: int, N: int, k: int, skew: float = 0.0) -> np.ndarray:
    """Distinct expert ids per token ([T, k] int32) for dispatch tests.

    Draws uniform candidates (optionally biased toward low ids with ``skew`` in
    [0, 1): candidate = floor(u^(1+8 skew) N)) and keeps the first k distinct ones.
    """
    out = np.empty((T, k), dtype=np.int32)
    draws = uniform_int(seed, TENSOR_IDS["topk"], T * 64, 1 << 30).reshape(T, 64)
    u = draws.astype(np.float64) / float(1 << 30)
    cand = np.minimum((u ** (1.0 + 8.0 * skew) * N).astype(np.int64), N - 1)
    for t in range(T):
        seen = []
        for c in cand[t]:
            if c not in seen:
                seen.append(int(c))
                if len(seen) == k:
                    break
        c = 0
        while len(seen) < k:       # fall back to the lowest unused ids
            if c not in seen:
                seen.append(c)
            c += 1
        out[t] = seen
    return out
