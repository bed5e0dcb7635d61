"""Expert-parallel MoE layer forward over a torch.distributed process group.

"MoE: what it costs to train and serve", Expert parallelism and two
all-to-alls: the N experts are spread over the P ranks (rank q holds experts
[q E, (q + 1) E), E = N / P); step 1 sends every (token, slot) row to the rank
that owns its expert, step 2 runs each rank's experts on the rows it received,
step 3 sends the outputs back, and the combine weighs them.  "Advanced GPU
Optimization ... Part 5", section 1.2 runs the same exchange with an
all-to-all collective.

Every computation runs in this library's kernels (router, dispatch, the
grouped GEMM over the rows from every rank, combine); the exchanges are
torch.distributed.all_to_all_single calls on device buffers (NCCL on GPUs).
The local dispatch already orders the rows by expert, so the rows for rank q
are one contiguous slice; the receiver gets them grouped by source rank and,
inside each, by its local experts, which is the layout moe_expert_ffn_multi
takes.  The host reads the expert offsets once per layer: the collectives need
the per-rank row counts as split sizes.

Capacity (if configured) applies to each rank's own batch: C = floor(cf T_r /
N) with T_r the rank's tokens.  The fallback expert is not supported here.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import (make_config, moe_combine, moe_dispatch, moe_expert_ffn, moe_expert_ffn_multi,
               moe_router, workspace)


@dataclass
class SendPlan:
    """Row counts of one rank's exchange: what it sends to and receives from
    every rank, per local expert of the owner."""
    send_counts: np.ndarray   # [P, E]: rows this rank sends to rank q for its expert e
    recv_counts: np.ndarray   # [P, E]: rows this rank receives from rank s for expert e

    @property
    def send_rows(self) -> list:
        return [int(v) for v in self.send_counts.sum(1)]

    @property
    def recv_rows(self) -> list:
        return [int(v) for v in self.recv_counts.sum(1)]

    def recv_offsets(self) -> np.ndarray:
        """[P E + 1] row offsets of the received rows, source-major."""
        flat = self.recv_counts.reshape(-1).astype(np.int64)
        return np.concatenate([[0], np.cumsum(flat)]).astype(np.int32)


def send_counts_of(offsets: np.ndarray, n_ranks: int) -> np.ndarray:
    """[P, E] rows per (destination rank, its local expert) from the local
    dispatch's expert offsets [N + 1] (experts ordered by owner)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    N = offsets.shape[0] - 1
    if N % n_ranks:
        raise ValueError(f"{N} experts do not split over {n_ranks} ranks")
    return np.diff(offsets).reshape(n_ranks, N // n_ranks)


def exchange_counts(send_counts: np.ndarray, group=None) -> SendPlan:
    """All-to-all of the per-expert row counts (rank q receives row q of every
    rank's send_counts)."""
    import torch.distributed as dist
    P, E = send_counts.shape
    backend = dist.get_backend(group)
    dev = "cuda" if backend == "nccl" else "cpu"
    send = torch.from_numpy(np.ascontiguousarray(send_counts, dtype=np.int64)).reshape(-1).to(dev)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return SendPlan(send_counts=np.asarray(send_counts, dtype=np.int64),
                    recv_counts=recv.cpu().numpy().reshape(P, E))


def exchange_rows(rows: torch.Tensor, plan: SendPlan, group=None) -> torch.Tensor:
    """Step 1: the first sum(send_rows) rows of `rows` (ordered by owner) go to
    their owners; returns the received rows, grouped by source rank."""
    import torch.distributed as dist
    out = rows.new_empty((sum(plan.recv_rows),) + tuple(rows.shape[1:]))
    n = sum(plan.send_rows)
    dist.all_to_all_single(out, rows[:n].contiguous(), output_split_sizes=plan.recv_rows,
                           input_split_sizes=plan.send_rows, group=group)
    return out


def return_rows(rows: torch.Tensor, plan: SendPlan, group=None) -> torch.Tensor:
    """Step 3: the inverse of exchange_rows (outputs back to the ranks that sent
    the rows, in their original order)."""
    import torch.distributed as dist
    out = rows.new_empty((sum(plan.send_rows),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.send_rows,
                           input_split_sizes=plan.recv_rows, group=group)
    return out


def ep_layer_forward(cfg, x, Wg, bias, W1, W3, W2, *, group=None, Ws1=None, Ws3=None, Ws2=None,
                     recv_capacity=None, stream=None):
    """One expert-parallel MoE layer forward on this rank.

    cfg: the layer as this rank sees it (T = its tokens, N = all experts);
    x [T, d]; Wg [N, d] and bias as for moe_router (replicated); W1, W3, W2 the
    weights of this rank's E = N / P experts ([E, H, d], [E, H, d], [E, d, H]);
    Ws1, Ws3, Ws2 the shared expert (run locally on this rank's tokens).
    recv_capacity: rows this rank can receive (default T * k * P).
    Returns (y [T, d], topk_idx [T, k], topk_w [T, k]).
    """
    from . import MOE_OVERFLOW_FALLBACK
    if cfg.overflow == MOE_OVERFLOW_FALLBACK:
        raise ValueError("the fallback expert is not supported by the expert-parallel layer")
    import torch.distributed as dist
    P = dist.get_world_size(group)
    T, k, N, d = cfg.T, cfg.k, cfg.N, cfg.d
    if N % P:
        raise ValueError(f"{N} experts do not split over {P} ranks")
    E = N // P
    dev = x.device
    ws = workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gw = torch.empty((T, k), dtype=torch.float32, device=dev)
    moe_router(cfg, x, Wg, bias, None, idx, gw, None, ws, stream)
    fp8 = cfg.dispatch_dtype != cfg.dtype
    rows = T * k
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 2, dtype=torch.int32, device=dev)
    perm = torch.empty(rows, dtype=torch.int32, device=dev)
    inv_row = torch.empty(rows, dtype=torch.int32, device=dev)
    drop = torch.empty(rows, dtype=torch.uint8, device=dev)
    x_perm = torch.empty((rows, d), dtype=torch.uint8 if fp8 else x.dtype, device=dev)
    x_scale = torch.empty(rows, dtype=torch.float32, device=dev) if fp8 else None
    moe_dispatch(cfg, x, idx, counts, offsets, perm, inv_row, drop, x_perm, x_scale, None, None,
                 None, ws, stream)

    # step 1: counts, then rows (and FP8 scales) to the owners of their experts
    plan = exchange_counts(send_counts_of(offsets[:N + 1].cpu().numpy(), P), group)
    recv_x = exchange_rows(x_perm, plan, group)
    recv_scale = exchange_rows(x_scale, plan, group) if fp8 else None

    # step 2: the local experts on every source's rows, one launch per projection
    cap = recv_capacity if recv_capacity is not None else rows * P
    n_recv = recv_x.shape[0]
    if n_recv > cap:
        raise ValueError(f"received {n_recv} rows, capacity {cap}")
    cfg_e = make_config(cap, d, E, 1, cfg.H, capacity_factor=0.0, act=_act(cfg),
                        dtype=_dtype(cfg), dispatch_dtype="fp8" if fp8 else None)
    ws_e = workspace(cfg_e)
    x_rows = torch.zeros((cap, d), dtype=recv_x.dtype, device=dev)
    x_rows[:n_recv] = recv_x
    s_rows = None
    if fp8:
        s_rows = torch.ones(cap, dtype=torch.float32, device=dev)
        s_rows[:n_recv] = recv_scale
    y_rows = torch.empty((cap, d), dtype=x.dtype, device=dev)
    recv_off = torch.from_numpy(plan.recv_offsets()).to(dev)
    moe_expert_ffn_multi(cfg_e, P, cap, x_rows, s_rows, recv_off, W1, W3, W2, y_rows, ws_e, stream)

    # step 3: outputs back to the ranks that routed them, then the combine
    y_back = return_rows(y_rows[:n_recv], plan, group)
    y_perm = torch.zeros((rows, d), dtype=x.dtype, device=dev)
    y_perm[:y_back.shape[0]] = y_back
    y_sh = None
    if cfg.H_shared > 0:
        y_sh = _shared_expert(cfg, x, Ws1, Ws3, Ws2, stream)
    y = torch.empty((T, d), dtype=x.dtype, device=dev)
    moe_combine(cfg, y_perm, inv_row, gw, y_sh, y, ws, stream)
    return y, idx, gw


def _act(cfg) -> str:
    from . import MOE_ACT_RELU
    return "relu" if cfg.act == MOE_ACT_RELU else "swiglu"


def _dtype(cfg) -> str:
    from . import MOE_F32
    return "f32" if cfg.dtype == MOE_F32 else "bf16"


def _shared_expert(cfg, x, Ws1, Ws3, Ws2, stream):
    """The always-on shared expert on this rank's tokens (one group of T rows)."""
    T, d = cfg.T, cfg.d
    cfg_s = make_config(T, d, 1, 1, cfg.H_shared, act=_act(cfg), dtype=_dtype(cfg))
    ws_s = workspace(cfg_s)
    off = torch.tensor([0, T], dtype=torch.int32, device=x.device)
    y = torch.empty((T, d), dtype=x.dtype, device=x.device)
    moe_expert_ffn(cfg_s, x, None, off, Ws1, Ws3, Ws2, y, ws_s, stream)
    return y
