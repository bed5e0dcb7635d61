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
the per-rank row counts as split sizes, and every rank agrees (one
all-reduce) that no rank would overflow its receive buffer before any row
moves, so an overflow raises on every rank instead of leaving the others
waiting in a collective.

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


def exchange_rows(rows: torch.Tensor, plan: SendPlan, group=None, out=None) -> torch.Tensor:
    """Step 1: the first sum(send_rows) rows of `rows` (ordered by owner) go to
    their owners; returns the received rows, grouped by source rank (in `out`,
    a contiguous [sum(recv_rows), ...] tensor, when given)."""
    import torch.distributed as dist
    if out is None:
        out = rows.new_empty((sum(plan.recv_rows),) + tuple(rows.shape[1:]))
    n = sum(plan.send_rows)
    dist.all_to_all_single(out, rows[:n].contiguous(), output_split_sizes=plan.recv_rows,
                           input_split_sizes=plan.send_rows, group=group)
    return out


def return_rows(rows: torch.Tensor, plan: SendPlan, group=None, out=None) -> torch.Tensor:
    """Step 3: the inverse of exchange_rows (outputs back to the ranks that sent
    the rows, in their original order; into `out` when given)."""
    import torch.distributed as dist
    if out is None:
        out = rows.new_empty((sum(plan.send_rows),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.send_rows,
                           input_split_sizes=plan.recv_rows, group=group)
    return out


class ExpertParallelLayer:
    """The expert-parallel layer forward of one configuration on this rank,
    with its workspaces and row buffers allocated once and reused by every
    call.

    cfg: the layer as this rank sees it (T = its tokens, N = all experts);
    group: the torch.distributed group whose P ranks each hold N / P experts;
    recv_capacity: rows this rank can receive (default T * k * P, every row
    of every rank).  The received rows land directly in preallocated buffers
    (no padded copies); rows past the received count are never read.
    """

    def __init__(self, cfg, group=None, recv_capacity=None, device=None):
        import torch.distributed as dist
        from . import MOE_OVERFLOW_FALLBACK
        if cfg.overflow == MOE_OVERFLOW_FALLBACK:
            raise ValueError("the fallback expert is not supported by the expert-parallel layer")
        self.cfg = cfg
        self.group = group
        self.P = dist.get_world_size(group)
        T, k, N, d = cfg.T, cfg.k, cfg.N, cfg.d
        if N % self.P:
            raise ValueError(f"{N} experts do not split over {self.P} ranks")
        self.E = N // self.P
        self.fp8 = cfg.dispatch_dtype != cfg.dtype
        rows = T * k
        self.cap = int(recv_capacity) if recv_capacity is not None else rows * self.P
        dev = torch.device(device) if device is not None else (
            torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available()
            else torch.device("cpu"))
        self.device = dev
        tdt = torch.float32 if _dtype(cfg) == "f32" else torch.bfloat16
        rdt = torch.uint8 if self.fp8 else tdt
        self.ws = workspace(cfg, dev)
        self.cfg_e = make_config(self.cap, d, self.E, 1, cfg.H, capacity_factor=0.0,
                                 act=_act(cfg), dtype=_dtype(cfg),
                                 dispatch_dtype="fp8" if self.fp8 else None)
        self.ws_e = workspace(self.cfg_e, dev)
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        self.idx, self.gw = e((T, k), torch.int32), e((T, k), torch.float32)
        self.counts, self.offsets = e(N, torch.int32), e(N + 2, torch.int32)
        self.perm, self.inv_row, self.drop = e(rows, torch.int32), e(rows, torch.int32), \
            e(rows, torch.uint8)
        self.x_perm = e((rows, d), rdt)
        self.x_scale = e(rows, torch.float32) if self.fp8 else None
        self.x_rows = e((self.cap, d), rdt)
        self.s_rows = e(self.cap, torch.float32) if self.fp8 else None
        self.y_rows = e((self.cap, d), tdt)
        self.y_perm = e((rows, d), tdt)
        self.y = e((T, d), tdt)
        if cfg.H_shared > 0:
            self.cfg_s = make_config(T, d, 1, 1, cfg.H_shared, act=_act(cfg), dtype=_dtype(cfg))
            self.ws_s = workspace(self.cfg_s, dev)
            self.off_s = torch.tensor([0, T], dtype=torch.int32, device=dev)
            self.y_s = e((T, d), tdt)

    def _agree_capacity(self, plan: SendPlan):
        """Every rank learns, before any row moves, whether some rank would
        receive more rows than it can hold; then all raise together."""
        import torch.distributed as dist
        n_recv = sum(plan.recv_rows)
        dev = "cuda" if dist.get_backend(self.group) == "nccl" else "cpu"
        flag = torch.tensor([n_recv, 1 if n_recv > self.cap else 0], dtype=torch.int64,
                            device=dev)
        dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=self.group)
        if int(flag[1].item()):
            raise ValueError(f"a rank would receive more rows than its capacity {self.cap} "
                             f"(largest: {int(flag[0].item())}; this rank: {n_recv})")
        return n_recv

    def forward(self, x, Wg, bias, W1, W3, W2, Ws1=None, Ws3=None, Ws2=None, stream=None):
        """One layer forward; returns (y [T, d], topk_idx [T, k], topk_w [T, k]),
        views of this layer's buffers (overwritten by the next call).  With a
        stream (torch.cuda.Stream or a raw cudaStream_t handle), the kernels,
        the exchanges and the copies all run on it, in order."""
        if stream is None:
            return self._forward(x, Wg, bias, W1, W3, W2, Ws1, Ws3, Ws2, None)
        s = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.ExternalStream(stream)
        with torch.cuda.stream(s):
            return self._forward(x, Wg, bias, W1, W3, W2, Ws1, Ws3, Ws2, s)

    def _forward(self, x, Wg, bias, W1, W3, W2, Ws1, Ws3, Ws2, s):
        cfg, N, P = self.cfg, self.cfg.N, self.P
        moe_router(cfg, x, Wg, bias, None, self.idx, self.gw, None, self.ws, s)
        moe_dispatch(cfg, x, self.idx, self.counts, self.offsets, self.perm, self.inv_row,
                     self.drop, self.x_perm, self.x_scale, None, None, None, self.ws, s)
        # step 1: counts (the host needs them as split sizes), then rows and
        # FP8 scales straight into the receive buffers
        plan = exchange_counts(send_counts_of(self.offsets[:N + 1].cpu().numpy(), P), self.group)
        n_recv = self._agree_capacity(plan)
        exchange_rows(self.x_perm, plan, self.group, out=self.x_rows[:n_recv])
        if self.fp8:
            exchange_rows(self.x_scale, plan, self.group, out=self.s_rows[:n_recv])
        # step 2: the local experts on every source's rows, one launch per projection
        recv_off = torch.from_numpy(plan.recv_offsets()).to(self.device)
        moe_expert_ffn_multi(self.cfg_e, P, self.cap, self.x_rows, self.s_rows, recv_off, W1, W3,
                             W2, self.y_rows, self.ws_e, s)
        # step 3: outputs back to the ranks that routed them, then the combine
        return_rows(self.y_rows[:n_recv], plan, self.group, out=self.y_perm[:sum(plan.send_rows)])
        y_sh = None
        if cfg.H_shared > 0:
            moe_expert_ffn(self.cfg_s, x, None, self.off_s, Ws1, Ws3, Ws2, self.y_s, self.ws_s, s)
            y_sh = self.y_s
        moe_combine(cfg, self.y_perm, self.inv_row, self.gw, y_sh, self.y, self.ws, s)
        return self.y, self.idx, self.gw


_LAYERS = {}


def _cfg_key(cfg):
    return tuple(getattr(cfg, n) for n, _ in cfg._fields_)


def ep_layer_forward(cfg, x, Wg, bias, W1, W3, W2, *, group=None, Ws1=None, Ws3=None, Ws2=None,
                     recv_capacity=None, stream=None):
    """One expert-parallel MoE layer forward on this rank (see
    ExpertParallelLayer; the layer object of each configuration, group,
    capacity and device is built on first use and reused).

    x [T, d]; Wg [N, d] and bias as for moe_router (replicated); W1, W3, W2
    the weights of this rank's E = N / P experts ([E, H, d], [E, H, d],
    [E, d, H]); Ws1, Ws3, Ws2 the shared expert (run locally on this rank's
    tokens).  Returns (y [T, d], topk_idx [T, k], topk_w [T, k]); the tensors
    are the layer object's buffers, overwritten by the next call."""
    device = x.device if x is not None else None
    key = (_cfg_key(cfg), id(group), recv_capacity, str(device))
    layer = _LAYERS.get(key)
    if layer is None:
        layer = _LAYERS[key] = ExpertParallelLayer(cfg, group, recv_capacity, device)
    return layer.forward(x, Wg, bias, W1, W3, W2, Ws1, Ws3, Ws2, stream)


def _act(cfg) -> str:
    from . import MOE_ACT_RELU
    return "relu" if cfg.act == MOE_ACT_RELU else "swiglu"


def _dtype(cfg) -> str:
    from . import MOE_F32
    return "f32" if cfg.dtype == MOE_F32 else "bf16"
