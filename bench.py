#!/usr/bin/env python
"""Benchmark of the MoE layer forward on B200: tokens/s and fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ``moe_layer_forward`` (router -> dispatch -> grouped expert FFN
-> combine) over one batch of synthetic tokens whose inputs are resident in
HBM.  The headline workload is the DeepSeek-V3-shaped layer (T=4096, d=7168,
N=256 + 1 shared expert, k=8, SwiGLU H=2048, bf16, FP8-E4M3 dispatch), the
largest configuration; the line also carries, under ``workloads``, the same
measurement of every other workload (Tiny fp32, Mixtral-, Switch- and
Grok-1-shaped layers, and the node-limited and fallback-expert variants),
taken in the same process.  For N > 1 (torchrun) every rank runs its own
replica of the headline on its own tokens (weak scaling, no data-path
collective); the time is the max over ranks and ``value`` counts the tokens
of all ranks.

``--impl reference`` times the CPU oracle (fp64, the reference arm) on a
bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200 + % of roofline (HBM GB/s or BF16 TFLOP/s)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank time over all ranks (the job is as slow as its slowest rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch in the step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def mult(wl):
    return 3 if wl.act == "swiglu" else 2


def algorithmic(wl, kept: np.ndarray):
    """Active FLOPs and algorithmic bytes of one layer forward (touched expert
    weights + x + y + W_g (+ bias, shared expert)); per-stage FLOPs/bytes of
    the expert up-projection."""
    es = 4 if wl.dtype == "f32" else 2
    m = mult(wl)
    R = int(kept.sum())
    touched = int(np.count_nonzero(kept))
    flops = 2.0 * wl.T * wl.N * wl.d + R * 2.0 * m * wl.d * wl.H
    wbytes = touched * m * wl.d * wl.H * es
    if wl.H_shared:
        flops += wl.T * 2.0 * m * wl.d * wl.H_shared
        wbytes += m * wl.d * wl.H_shared * es
    abytes = 2 * wl.T * wl.d * es + wl.N * wl.d * es + (wl.N * 4 if wl.bias_std > 0 else 0)
    up_mult = 2 if wl.act == "swiglu" else 1
    up_flops = R * 2.0 * wl.d * wl.H * up_mult
    up_bytes = touched * up_mult * wl.d * wl.H * es          # weights read
    up_bytes += R * wl.d * (1 if wl.dispatch == "fp8" else es) + R * wl.H * es  # A rows in, h out
    return dict(flops=flops, bytes=wbytes + abytes, R=R, touched=touched,
                up_flops=up_flops, up_bytes=up_bytes)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons.  Started before the
    warm-up (nvidia-smi takes a moment to start), stopped after the timed
    region; the summary keeps the samples stamped inside the region (within
    one sampling period of its ends)."""
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap",
             "hw_power_brake_slowdown", "applications_clocks_setting", "sync_boost"]

    BASIC = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.names = list(self.NAMES)
        # a driver without one of the extra fields rejects the whole query:
        # fall back to the four reasons every driver reports
        try:
            ok = subprocess.run(["nvidia-smi", "-i", str(index), f"--query-gpu={self.fields()}",
                                 "--format=csv,noheader"], capture_output=True,
                                timeout=10).returncode == 0
        except (OSError, subprocess.TimeoutExpired):
            ok = False
        if not ok:
            self.names = list(self.BASIC)

    def fields(self):
        return ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                + ",".join("clocks_event_reasons." + n for n in self.names))

    def start(self):
        import atexit
        self.out = ""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.fields()}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            atexit.register(self.stop)   # no sampler outlives an error path
        except OSError:
            self.proc = None
        return self

    def stop(self):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
            self.proc = None

    def __enter__(self):
        return self.start()

    def __exit__(self, *a):
        self.stop()

    def summary(self, t0=None, t1=None):
        """Median SM clock and power, max clock, every reason seen active, and the
        active-reasons bitmasks seen (nvidia-smi's clocks_event_reasons.active), over
        the samples stamped in [t0 - 0.06 s, t1 + 0.06 s] (host wall clock) when given."""
        import datetime
        sm, mx, pw, reasons, masks = [], [], [], set(), set()
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 5 + len(self.names):
                continue
            if t0 is not None:
                try:
                    ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                if ts < t0 - 0.06 or ts > t1 + 0.06:
                    continue
            f = f[1:]
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            try:
                pw.append(float(f[2]))
            except ValueError:
                pass
            masks.add(f[3])
            for n, v in zip(self.names, f[4:4 + len(self.names)]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "power_w": None, "reasons": [],
                    "active_masks": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(mx),
                "power_w": statistics.median(pw) if pw else None, "reasons": sorted(reasons),
                "active_masks": sorted(masks), "samples": len(sm)}


def single_launch(wl) -> bool:
    """fp32 layers without a capacity limit run as one kernel (the whole layer)."""
    return wl.dtype == "f32" and wl.capacity_factor <= 0


def up_kernel(wl):
    """(kernel name, source file) of the dominant kernel the library runs for
    this workload: the single-launch kernel for small fp32 layers without a
    capacity limit, else the expert up-projection (fp32 layers: the SIMT
    kernel; bf16 layers whose experts average at least 512 rows, T k >= 512 G
    with G the expert groups, the fallback expert included: the CTA-pair
    kernel; otherwise the transposed CTA-pair kernel, or with a fallback
    expert the one-CTA kernel; the up-projection is the dominant kernel, and
    the down-projection of layers whose experts average more than 64 rows
    runs on the one-CTA kernel)."""
    if single_launch(wl):
        return "layer_small_f32", "layer_small.cu"
    if wl.dtype == "f32":
        return "grouped_gemm_simt_f32", "ffn_simt.cu"
    fallback = wl.overflow == "fallback"
    if wl.T * wl.k >= 512 * (wl.N + (1 if fallback else 0)):
        return "grouped_gemm_tc_pair", "gemm_tc2.cu"
    if fallback:
        return "grouped_gemm_tc", "gemm_tc.cu"
    return "grouped_gemm_tc_pairt", "gemm_tc2t.cu"


def traffic_from_profile(kernel_key: str, workload_key: str, source: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kernel_key}_{workload_key}.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    src = os.path.join(ROOT, "top_routing_expert_warp_b200", "csrc", source)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if vals.get("source_sha256_16") != h:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------- oracle legs
def oracle_sample(wl, budget_s: float, max_tokens: int = 4096):
    """Time the CPU oracle on a bounded sample of the workload's tokens.

    Routing (router + dispatch) of the sampled tokens and their expert rows and
    combine.  Returns (tokens/s, tokens, seconds, description)."""
    import oracle
    host = synth.make_host(wl, names={"x", "Wg", "bias", "Ws1", "Ws3", "Ws2"})

    def expert(e):
        return (synth.expert_slice(wl, "W1", e),
                synth.expert_slice(wl, "W3", e) if wl.act == "swiglu" else None,
                synth.expert_slice(wl, "W2", e))
    cache = {}

    def get_expert(e):
        if e not in cache:
            cache[e] = expert(e)
        return cache[e]

    shared = (host["Ws1"], host.get("Ws3"), host["Ws2"]) if wl.H_shared else None

    def run(tokens):
        t0 = time.perf_counter()
        sub = wl.with_(T=len(tokens), capacity_factor=0.0)
        xs = host["x"][tokens]
        r = oracle.route(sub, xs, host["Wg"], host.get("bias"))
        oracle.forward_rows_lazy(sub, xs, r, np.arange(len(tokens)), get_expert, shared)
        return time.perf_counter() - t0

    # warm the weight cache outside the timed region (weights are resident, like HBM)
    for e in range(wl.N):
        get_expert(e)
    # grow the sample until it takes a quarter of the budget, then scale to the budget
    n = 1
    while True:
        pilot = run(np.linspace(0, wl.T - 1, n).astype(np.int64))
        if pilot >= budget_s / 4 or n >= max_tokens:
            break
        n *= 2
    n = int(max(1, min(max_tokens, n * budget_s / max(pilot, 1e-3))))
    toks = np.linspace(0, wl.T - 1, n).astype(np.int64)
    secs = run(toks)
    desc = (f"{n} of {wl.T} tokens (router, top-k, dispatch and expert FFN + combine of their "
            f"{n * wl.k} rows; capacity not applied to the sample), fp64, "
            f"{len(os.sched_getaffinity(0))} host threads (OpenMP)")
    return n / secs, n, secs, desc


def run_reference(args, wl):
    """The reference arm: the CPU oracle, timed as it stands on this host's cores.

    Each step is the oracle forward of n evenly spaced tokens of the workload,
    n chosen so that the whole --warmup + --steps run stays within a few
    minutes.  Under torchrun only rank 0 runs; the other ranks exit at once."""
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    cores = len(os.sched_getaffinity(0))
    per_step_budget = min(1.0, 150.0 / max(1, args.steps + args.warmup))
    _oracle_tokens(wl, 1)                      # builds the host inputs once
    n = 1
    while n < 64:
        t0 = time.perf_counter()
        _oracle_tokens(wl, 2 * n)
        if time.perf_counter() - t0 > per_step_budget:
            break
        n *= 2
    for _ in range(args.warmup):
        _oracle_tokens(wl, n)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_tokens(wl, n)
        times.append(time.perf_counter() - t0)
    ms = 1000.0 * statistics.mean(times)
    value = n / (ms / 1000.0)
    desc = (f"each step: {n} of {wl.T} tokens (router, top-k, dispatch, expert FFN and combine "
            f"of their {n * wl.k} rows; capacity not applied to the sample), fp64, {cores} host "
            f"threads (OpenMP)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


_REF_STATE = {}


def _oracle_tokens(wl, n):
    """One reference step: the oracle forward of n evenly spaced tokens."""
    import oracle
    st = _REF_STATE.get(wl.name)
    if st is None:
        host = synth.make_host(wl, names={"x", "Wg", "bias", "Ws1", "Ws3", "Ws2"})
        experts = {e: (synth.expert_slice(wl, "W1", e),
                       synth.expert_slice(wl, "W3", e) if wl.act == "swiglu" else None,
                       synth.expert_slice(wl, "W2", e)) for e in range(wl.N)}
        st = _REF_STATE[wl.name] = (host, experts)
    host, experts = st
    toks = np.linspace(0, wl.T - 1, n).astype(np.int64)
    sub = wl.with_(T=n, capacity_factor=0.0)
    xs = host["x"][toks]
    r = oracle.route(sub, xs, host["Wg"], host.get("bias"))
    shared = (host["Ws1"], host.get("Ws3"), host["Ws2"]) if wl.H_shared else None
    oracle.forward_rows_lazy(sub, xs, r, np.arange(n), lambda e: experts[e], shared)


def config_of(wl):
    c = {"workload": wl.name, "T": wl.T, "d": wl.d, "N": wl.N, "k": wl.k, "H": wl.H,
         "act": wl.act, "gate_mode": wl.gate_mode, "renormalize": wl.renormalize,
         "capacity_factor": wl.capacity_factor, "H_shared": wl.H_shared,
         "dispatch": wl.dispatch_dtype, "seed": wl.seed,
         "n_groups": wl.n_groups, "topk_groups": wl.topk_groups, "overflow": wl.overflow,
         "slot_priority": wl.slot_priority,
         "l2": "inputs larger than L2: expert weights read every step exceed 126 MB and the "
               "token batch rotates over 4 resident copies"}
    return c


# ----------------------------------------------------------------- our arm
L2_BYTES = 126 * 1024 * 1024


def near_ties(wl, x_bits, Wg_bits, bias, idx) -> int:
    """Tokens whose routing may legitimately differ from an exact computation:
    the k-th and (k+1)-th largest fp64 logits within 1e-3 relative (with
    node-limited routing also the topk_groups-th and next node scores, and the
    k-th / next logits among the chosen nodes' experts).  A reported statistic
    of the run's batch, computed on the host with numpy in fp64."""
    x = synth.bf16_to_f32(x_bits).astype(np.float64) if x_bits.dtype == np.uint16 else \
        x_bits.astype(np.float64)
    W = synth.bf16_to_f32(Wg_bits).astype(np.float64) if Wg_bits.dtype == np.uint16 else \
        Wg_bits.astype(np.float64)
    lg = x @ W.T
    if bias is not None:
        lg += bias.astype(np.float64)[None, :]
    T, N = lg.shape
    k = wl.k

    def gap_tie(v, j):
        srt = -np.sort(-v, axis=1)
        a, b = srt[:, j - 1], srt[:, j]
        fin = np.isfinite(a) & np.isfinite(b)
        out = np.zeros(len(v), bool)
        out[fin] = np.abs(a[fin] - b[fin]) <= 1e-3 * np.maximum(np.abs(a[fin]), np.abs(b[fin]))
        return out

    tie = gap_tie(lg, k) if k < N else np.zeros(T, bool)
    if wl.n_groups > 1 and 0 < wl.topk_groups < wl.n_groups:
        S = N // wl.n_groups
        m = -(-k // wl.topk_groups)
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        node = -np.sort(-p.reshape(T, wl.n_groups, S), axis=2)[:, :, :m].sum(2)
        tie |= gap_tie(node, wl.topk_groups)
        chosen = np.zeros((T, wl.n_groups), bool)
        chosen[np.arange(T)[:, None], idx // S] = True
        masked = np.where(np.repeat(chosen, S, axis=1), lg, -np.inf)
        tie |= gap_tie(masked, k)
    return int(tie.sum())


def device_inputs(wl, cache: dict) -> dict:
    """Device tensors of every input of ``wl`` (seeded, generated on the host
    one expert slice at a time through pinned memory).  Tensors already in
    ``cache`` under the same seed, name, shape and scale are reused (the
    node-limited DeepSeek-shaped variant shares the plain layer's weights)."""
    import torch
    dev = {}
    for name, shape, std, dt in synth.tensor_specs(wl):
        key = (wl.seed, name, tuple(shape), float(std), dt)
        if key in cache:
            dev[name] = cache[key]
            continue
        tdt = torch.float32 if dt == "f32" else torch.bfloat16
        t = torch.empty(shape, dtype=tdt, device="cuda")
        n = int(np.prod(shape))
        per = int(np.prod(shape[1:])) if len(shape) == 3 else n
        pinned = torch.empty(per, dtype=tdt, pin_memory=True)
        pin_np = pinned.view(torch.int16 if dt == "bf16" else torch.float32).numpy()
        flat = t.view(-1)
        for s0 in range(0, n, per):
            synth.normal(wl.seed, synth.TENSOR_IDS[name], per, std, dt, start=s0,
                         out=pin_np.view(np.uint16) if dt == "bf16" else pin_np)
            flat[s0:s0 + per].copy_(pinned)
        torch.cuda.synchronize()
        cache[key] = dev[name] = t
    return dev


def measure(wl, dev, args, rank, local, world, dist, headline: bool):
    """Time ``moe_layer_forward`` of workload ``wl`` on resident inputs.

    Returns the per-workload record (and, for the headline, the e2e and launch
    figures).  Layers whose whole per-step footprint fits in L2 are timed step by
    step with L2 flushed between steps; the others in one region of K steps."""
    import torch
    import top_routing_expert_warp_b200 as moe

    def barrier():
        if dist is not None:
            dist.barrier()

    cfg = moe.config_from(wl)
    ws = moe.workspace(cfg)
    tdt = dev["x"].dtype
    # 4 resident token batches (distinct seeds), rotated per step
    xs = [dev["x"]]
    for i in range(1, 4):
        x = torch.empty_like(dev["x"])
        x.view(-1).copy_(torch.from_numpy(
            synth.normal(wl.seed + 1000 * i, 0, wl.T * wl.d, 1.0, wl.dtype).view(
                np.int16 if wl.dtype == "bf16" else np.float32)).view(tdt).to("cuda"))
        xs.append(x)
    y = torch.empty((wl.T, wl.d), dtype=tdt, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gw = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.N, dtype=torch.int32, device="cuda")
    f = torch.empty(wl.N, dtype=torch.float32, device="cuda")
    pm = torch.empty(wl.N, dtype=torch.float32, device="cuda")
    aux = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i, x=None, y_out=None):
        moe.moe_layer_forward(cfg, xs[i % 4] if x is None else x, dev["Wg"], dev.get("bias"),
                              dev["W1"], dev.get("W3"), dev["W2"], dev.get("Ws1"), dev.get("Ws3"),
                              dev.get("Ws2"), y if y_out is None else y_out, idx, gw, counts, f, pm,
                              aux, ws, stream)

    clk = Clocks(local).start()   # running (and started up) well before the timed region
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st, word = moe.moe_check_status(ws)
    if st != moe.MOE_OK:
        clk.stop()
        raise RuntimeError(f"{wl.name}: device status after warm-up: {moe.status_string(st)} "
                           f"({word:#x})")
    C = wl.capacity()
    kept_steps, stats = [], None
    for i in range(4):                       # routing of each rotated batch
        step(i)
        torch.cuda.synchronize()
        cnt = counts.cpu().numpy().astype(np.int64)
        kept = cnt.copy()
        over = 0
        if C >= 0:
            over = int((cnt - np.minimum(cnt, C)).sum())
            kept = np.minimum(cnt, C)
            if wl.overflow == "fallback":
                kept = np.append(kept, over)      # the fallback expert's rows
        kept_steps.append(kept)
        if i == 0:
            stats = {"near_ties": None, "rows": int(kept.sum()),
                     "drops": over if wl.overflow != "fallback" else 0,
                     "rerouted_to_fallback": over if wl.overflow == "fallback" else 0,
                     "touched_experts": int(np.count_nonzero(kept)),
                     "L_aux": float(aux.item()), "aux_alpha": wl.aux_alpha}
            if rank == 0 and not args.no_near_ties:
                host_x = synth.normal(wl.seed, synth.TENSOR_IDS["x"], wl.T * wl.d, 1.0,
                                      wl.dtype).reshape(wl.T, wl.d)
                spec = {s_[0]: s_ for s_ in synth.tensor_specs(wl)}
                host_wg = synth.normal(wl.seed, synth.TENSOR_IDS["Wg"], wl.N * wl.d,
                                       spec["Wg"][2], wl.dtype).reshape(wl.N, wl.d)
                host_b = (synth.normal(wl.seed, synth.TENSOR_IDS["bias"], wl.N, wl.bias_std, "f32")
                          if wl.bias_std > 0 else None)
                stats["near_ties"] = near_ties(wl, host_x, host_wg, host_b, idx.cpu().numpy())
    alg = [algorithmic(wl, k) for k in kept_steps]
    flush = statistics.mean(a["bytes"] for a in alg) < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if flush else None

    # ---- timed region (device events, max over ranks).  Nothing but the
    # layer calls in it: events recorded between the kernels would cut the
    # programmatic launch overlap and cost time of their own.
    barrier()
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    t_region = [time.time(), None]
    if not flush:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_local = e0.elapsed_time(e1) / args.steps
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            scratch.fill_(i & 0xFF)           # L2 flush, outside the timed events
            evs[i][0].record(stream)
            step(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms_local = statistics.mean(a.elapsed_time(b) for a, b in evs)
    t_region[1] = time.time()
    clk.stop()
    clocks = clk.summary(*t_region)
    launches = moe.moe_launch_count() - l0
    barrier()
    ms = max_over_ranks(ms_local, dist, "cuda")
    st, word = moe.moe_check_status(ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{wl.name}: device status after timing: {moe.status_string(st)} "
                           f"({word:#x})")

    # ---- kernel-timing pass: the same steps again with the library's stage
    # events (recorded on the launching stream between the stages); gives the
    # dominant kernel's launch duration for the roofline and the stage split
    barrier()
    torch.cuda.synchronize()
    moe.moe_profile_begin(args.steps)
    for i in range(args.steps):
        if flush:
            scratch.fill_(i & 0xFF)
        step(i)
    torch.cuda.synchronize()
    stages, nrec = moe.moe_profile_end()
    barrier()

    e2e = None
    if headline:
        e2e = measure_e2e(wl, xs, y, step, args, dist, stream)

    pk, pk_src = peaks()
    flops = statistics.mean(a["flops"] for a in alg)
    byts = statistics.mean(a["bytes"] for a in alg)
    up_flops = statistics.mean(a["up_flops"] for a in alg)
    up_bytes = statistics.mean(a["up_bytes"] for a in alg)
    peak_tf_b = pk["bf16_tflops"]
    peak_tf_s = pk["bf16_tflops_sustained"]
    peak_bw = pk["hbm_gbs"]
    up_ms = stages["expert_up"] / max(1, nrec)
    kname, ksrc = up_kernel(wl)
    kdesc = "expert up-projection + activation epilogue"
    if single_launch(wl):
        # one kernel does the whole layer: its work is the layer's
        up_flops, up_bytes = flops, byts
        kdesc = "the whole layer in one launch"
    # bound of the dominant kernel: arithmetic intensity vs the ridge point.
    # It runs inside a step far shorter than a second, so the burst tensor
    # peak applies; the sustained one is reported beside it
    ridge = peak_tf_b * 1e12 / (peak_bw * 1e9)
    if (up_flops / max(up_bytes, 1)) >= ridge:
        achieved = up_flops / (up_ms * 1e-3) / 1e12
        roof = {"kernel": f"{kname} ({kdesc})",
                "bound": "tensor", "achieved": achieved, "peak": peak_tf_b, "unit": "TFLOP/s",
                "frac": achieved / peak_tf_b, "peak_kind": f"bf16_tflops burst ({pk_src})",
                "frac_of_sustained_peak": achieved / peak_tf_s,
                "algorithmic_per_launch": up_flops, "launch_ms": up_ms}
    else:
        achieved = up_bytes / (up_ms * 1e-3) / 1e9
        roof = {"kernel": f"{kname} ({kdesc})",
                "bound": "hbm", "achieved": achieved, "peak": peak_bw, "unit": "GB/s",
                "frac": achieved / peak_bw, "peak_kind": f"hbm_gbs ({pk_src})",
                "algorithmic_per_launch": up_bytes, "launch_ms": up_ms}
    roof["traffic"] = traffic_from_profile("grouped_gemm_up", wl_key(wl), ksrc)
    # the whole layer against its own roofline (slower of the two bounds)
    t_roof_meas = max(flops / (peak_tf_b * 1e12), byts / (peak_bw * 1e9))
    t_roof_spec = max(flops / 2.25e15, byts / 8.0e12)
    layer = {"active_flops": flops, "algorithmic_bytes": byts,
             "bound": "tensor" if flops / (peak_tf_b * 1e12) >= byts / (peak_bw * 1e9) else "hbm",
             "roofline_ms_measured_peaks": 1e3 * t_roof_meas,
             "roofline_ms_spec_peaks": 1e3 * t_roof_spec,
             "frac_of_roofline_measured": 1e3 * t_roof_meas / ms,
             "frac_of_roofline_spec": 1e3 * t_roof_spec / ms}
    rec = {"ms_per_step": ms, "tokens_per_s": weak_value(wl.T, world, ms),
           "timing": ("per step between CUDA events, L2 flushed (256 MB write) before each step"
                      if flush else "one region of K steps between CUDA events; inputs larger "
                                    "than L2 (expert weights streamed from HBM every step, "
                                    "token batch rotated over 4 resident copies)"),
           "roofline": roof, "layer_roofline": layer,
           "stages_ms": {k: v / max(1, nrec) for k, v in stages.items()},
           "routing": stats, "clocks": clocks, "config": config_of(wl)}
    if headline:
        rec["e2e"] = e2e
        rec["gpu_launches"] = int(launches)
    del ws, xs, scratch
    return rec


def measure_e2e(wl, xs, y, step, args, dist, stream):
    """End to end through the C ABI with host buffers (pinned): every step
    copies its tokens in from the host and its output back.  As a serving loop
    would, the copies run on two copy streams with double buffers, so step
    i+1's input and step i-1's output move while step i computes; the timed
    region ends only after the last output has reached the host."""
    import torch
    tdt = xs[0].dtype
    x_host = [xs[i].cpu().pin_memory() for i in range(4)]
    y_host = [torch.empty((wl.T, wl.d), dtype=tdt).pin_memory() for _ in range(2)]
    xin = [torch.empty_like(xs[0]) for _ in range(2)]
    yout = [torch.empty_like(y) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]     # xin[b] holds its step's tokens
    done = [torch.cuda.Event() for _ in range(2)]         # the layer that used xin[b] / yout[b] ended
    out_free = [torch.cuda.Event() for _ in range(2)]     # yout[b] has been copied to the host
    e_steps = max(3, args.steps)        # as many steps as the timed region: same power state

    def load(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            h2d.wait_event(done[b])                       # the layer two steps back read xin[b]
            xin[b].copy_(x_host[i % 4], non_blocking=True)
            in_ready[b].record(h2d)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    with torch.cuda.stream(h2d):
        h2d.wait_event(a0)
    load(0)
    for i in range(e_steps):
        b = i % 2
        if i + 1 < e_steps:
            load(i + 1)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_free[b])                    # yout[b] of step i-2 reached the host
        step(i, xin[b], yout[b])
        done[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(done[b])
            y_host[b].copy_(yout[b], non_blocking=True)
            out_free[b].record(d2h)
    stream.wait_stream(d2h)
    a1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    world = dist.get_world_size() if dist is not None else 1
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, "cuda") / e_steps
    return {"value": weak_value(wl.T, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
            "copies": "pinned host buffers, double-buffered on two copy streams overlapping the "
                      "layer",
            "h2d_bytes_per_step": int(xs[0].numel() * xs[0].element_size()),
            "d2h_bytes_per_step": int(y.numel() * y.element_size())}


def run_ours(args, wl):
    import torch
    import top_routing_expert_warp_b200 as moe

    moe.lib()                            # fails loudly when the library is missing
    rank, local, world = env_rank()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    cache = {}
    t_up = time.perf_counter()
    dev = device_inputs(wl, cache)
    gen_s = time.perf_counter() - t_up
    head = measure(wl, dev, args, rank, local, world, dist, headline=True)

    # the other workloads, each measured the same way in this process (one
    # GPU only: under torchrun the scaling run times the headline alone)
    extra = {}
    names = [] if (world > 1 or args.workloads == "none") else \
        [n for n in (args.workloads.split(",") if args.workloads else synth.WORKLOADS)
         if n != wl_key(wl)]
    # workloads sharing the headline's tensors first, then free them
    names.sort(key=lambda n: 0 if synth.WORKLOADS[n].seed == wl.seed else 1)
    for n in names:
        w2 = synth.WORKLOADS[n]
        if w2.seed != wl.seed and cache:
            dev = None
            cache.clear()
            torch.cuda.empty_cache()
        d2 = device_inputs(w2, cache)
        extra[n] = measure(w2, d2, args, rank, local, world, dist, headline=False)
        del d2

    out = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, n, secs, desc = oracle_sample(wl, args.cpu_budget)
            cpu = {"value": rate, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
                   "kind": "oracle", "sample": desc, "seconds": secs}
        out = {"metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s",
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": wl.dtype,
               "data": "synthetic (seeded SplitMix64 + Box-Muller normals; weights N(0, 1/fan_in))",
               "config": config_of(wl), "roofline": head["roofline"],
               "layer_roofline": head["layer_roofline"], "cpu_baseline": cpu,
               "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
               "stages_ms": head["stages_ms"], "routing": head["routing"],
               "clocks": head["clocks"], "timing": head["timing"], "input_gen_s": gen_s,
               "workloads": {n: {k: v for k, v in r.items()} for n, r in extra.items()}}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


def wl_key(wl):
    for k, v in synth.WORKLOADS.items():
        if v == wl:
            return k
    return "custom"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(synth.WORKLOADS), default="deepseek",
                    help="the headline workload (default: the DeepSeek-V3-shaped layer, the "
                         "largest configuration)")
    ap.add_argument("--workloads", default="",
                    help="comma list of further workloads measured in the same run and reported "
                         "under 'workloads' (default: all others; 'none' for the headline only)")
    ap.add_argument("--no-near-ties", action="store_true",
                    help="skip the host fp64 near-tie count")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
