"""Helpers shared by the GPU parity tests, the smoke check and the benchmark.

Inputs come from ``synth`` (host, seeded) and are uploaded unchanged, so the
oracle and the CUDA path see bit-identical values.  Nothing here computes any
part of the MoE method.
"""
from __future__ import annotations

import numpy as np
import torch

import synth
import top_routing_expert_warp_b200 as moe


def cfg_of(wl: synth.Workload) -> moe.moe_config:
    return moe.config_from(wl)


def tdtype(wl: synth.Workload):
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Host array (float32, or bf16 bits as uint16) -> device tensor, bit-exact."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host array in the storage convention of ``synth``."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def upload_inputs(wl: synth.Workload, device="cuda", keep_host=True):
    """Device tensors for every input of ``wl``; large stacked weights are
    generated and uploaded one expert at a time.  Returns (dev, host) where
    host holds the arrays kept on the host (all of them if keep_host)."""
    dev, host = {}, {}
    for name, shape, std, dt in synth.tensor_specs(wl):
        n = int(np.prod(shape))
        if len(shape) == 3 and not keep_host:
            t = torch.empty(shape, dtype=torch.float32 if dt == "f32" else torch.bfloat16,
                            device=device)
            per = int(np.prod(shape[1:]))
            for e in range(shape[0]):
                a = synth.normal(wl.seed, synth.TENSOR_IDS[name], per, std, dt, start=e * per)
                t[e].copy_(to_dev(a.reshape(shape[1:]), device))
            dev[name] = t
        else:
            a = synth.normal(wl.seed, synth.TENSOR_IDS[name], n, std, dt).reshape(shape)
            dev[name] = to_dev(a, device)
            if keep_host or len(shape) < 3:
                host[name] = a
    return dev, host


class LayerRun:
    """Device buffers for one ``moe_layer_forward`` call of workload ``wl``."""

    def __init__(self, wl: synth.Workload, dev: dict, device="cuda"):
        self.wl = wl
        self.cfg = cfg_of(wl)
        self.dev = dev
        T, k, N, d = wl.T, wl.k, wl.N, wl.d
        self.y = torch.empty((T, d), dtype=tdtype(wl), device=device)
        self.topk_idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.counts = torch.empty(N, dtype=torch.int32, device=device)
        self.f = torch.empty(N, dtype=torch.float32, device=device)
        self.p_mean = torch.empty(N, dtype=torch.float32, device=device)
        self.aux = torch.empty(1, dtype=torch.float32, device=device)
        self.ws = moe.workspace(self.cfg, device)

    def __call__(self, stream=None):
        d = self.dev
        moe.moe_layer_forward(self.cfg, d["x"], d["Wg"], d.get("bias"), d["W1"], d.get("W3"),
                              d["W2"], d.get("Ws1"), d.get("Ws3"), d.get("Ws2"), self.y,
                              self.topk_idx, self.topk_w, self.counts, self.f, self.p_mean,
                              self.aux, self.ws, stream)
        return self.y

    def check_status(self):
        return moe.moe_check_status(self.ws)


def near_tie_tokens(logits: np.ndarray, idx: np.ndarray, k: int, rel: float = 1e-3) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest oracle logits are within ``rel``
    relative of each other (the routing there may legitimately differ)."""
    T, N = logits.shape
    if k >= N:
        return np.zeros(T, dtype=bool)
    srt = -np.sort(-logits, axis=1)
    a, b = srt[:, k - 1], srt[:, k]
    return np.abs(a - b) <= rel * np.maximum(np.abs(a), np.abs(b))


def node_near_ties(probs: np.ndarray, k: int, n_groups: int, topk_groups: int,
                   rel: float = 1e-3) -> np.ndarray:
    """Node-limited routing: tokens whose topk_groups-th and next node scores
    (sum of a node's ceil(k / topk_groups) highest probabilities) are within rel."""
    T, N = probs.shape
    S = N // n_groups
    m = -(-k // topk_groups)
    top = -np.sort(-probs.reshape(T, n_groups, S), axis=2)[:, :, :m].sum(2)
    srt = -np.sort(-top, axis=1)
    a, b = srt[:, topk_groups - 1], srt[:, topk_groups]
    return np.abs(a - b) <= rel * np.maximum(a, b)


def chosen_node_near_ties(logits: np.ndarray, idx: np.ndarray, k: int, n_groups: int,
                          rel: float = 1e-3) -> np.ndarray:
    """Node-limited routing: near-ties between the k-th and next logits among the
    experts of the nodes the oracle chose."""
    T, N = logits.shape
    S = N // n_groups
    masked = np.full_like(logits, -np.inf)
    for t in range(T):
        for g in np.unique(idx[t] // S):
            masked[t, g * S:(g + 1) * S] = logits[t, g * S:(g + 1) * S]
    srt = -np.sort(-masked, axis=1)
    a, b = srt[:, k - 1], srt[:, k]
    fin = np.isfinite(b)
    out = np.zeros(T, bool)
    out[fin] = np.abs(a[fin] - b[fin]) <= rel * np.maximum(np.abs(a[fin]), np.abs(b[fin]))
    return out


def route_near_ties(wl: synth.Workload, ref: dict) -> np.ndarray:
    """Tokens whose routing may legitimately differ from the oracle's."""
    tie = near_tie_tokens(ref["logits"], ref["idx"], wl.k)
    if wl.n_groups > 1 and wl.topk_groups < wl.n_groups:
        tie |= node_near_ties(ref["probs"], wl.k, wl.n_groups, wl.topk_groups)
        tie |= chosen_node_near_ties(ref["logits"], ref["idx"], wl.k, wl.n_groups)
    return tie


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


TOL_Y = {"f32": 1e-5, "bf16": 5e-3, "fp8": 3e-2}


def y_tol(wl: synth.Workload) -> float:
    return TOL_Y["fp8"] if wl.dispatch == "fp8" else TOL_Y[wl.dtype]
