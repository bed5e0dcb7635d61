"""Run one stage (or the whole layer) of a workload a few times, for profilers.

    python -m top_routing_expert_warp_b200.profile_case --workload deepseek \
        --stage router --iters 3 [--T 512] [--N 32]

Generates the workload's seeded inputs on the device (only those the stage
reads), runs the chosen entry point ``--warmup`` + ``--iters`` times on one
stream and synchronises.  ``--T`` and ``--N`` shrink the token batch and the
number of routed experts so that a capture under a profiler holds a few GB at
most; a layer with T' = T N' / N keeps the rows per expert (and so the tile
structure of the grouped GEMMs) of the full layer, and its weight traffic
scales with the experts touched.

Stages: ``router`` (moe_router), ``dispatch`` (moe_router once, then
moe_dispatch), ``ffn`` (router and dispatch once, then moe_expert_ffn),
``layer`` (moe_layer_forward).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    import torch

    import synth
    import top_routing_expert_warp_b200 as moe

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", choices=list(synth.WORKLOADS), default="deepseek")
    ap.add_argument("--stage", choices=["router", "dispatch", "ffn", "layer"], default="layer")
    ap.add_argument("--T", type=int, default=0, help="tokens (default: the workload's)")
    ap.add_argument("--N", type=int, default=0, help="routed experts (default: the workload's)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args(argv)

    wl = synth.WORKLOADS[a.workload]
    kw = {}
    if a.T:
        kw["T"] = a.T
    if a.N:
        kw["N"] = a.N
        if wl.n_groups > 1:
            kw["n_groups"] = min(wl.n_groups, a.N)
    if kw:
        wl = wl.with_(**kw)
    need = {"x", "Wg", "bias"}
    if a.stage in ("ffn", "layer"):
        need |= {"W1", "W3", "W2"}
    if a.stage == "layer":
        need |= {"Ws1", "Ws3", "Ws2"}

    torch.cuda.set_device(0)
    dev = {}
    for name, shape, std, dt in synth.tensor_specs(wl):
        if name not in need:
            continue
        tdt = torch.float32 if dt == "f32" else torch.bfloat16
        t = torch.empty(shape, dtype=tdt, device="cuda")
        per = int(np.prod(shape[1:])) if len(shape) == 3 else int(np.prod(shape))
        flat = t.view(-1)
        for s0 in range(0, t.numel(), per):
            h = synth.normal(wl.seed, synth.TENSOR_IDS[name], per, std, dt, start=s0)
            flat[s0:s0 + per].copy_(torch.from_numpy(
                h.view(np.int16) if dt == "bf16" else h).view(tdt))
        dev[name] = t
    cfg = moe.config_from(wl)
    ws = moe.workspace(cfg)
    T, k, N, d = wl.T, wl.k, wl.N, wl.d
    tdt = dev["x"].dtype
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    pm = torch.empty(N, dtype=torch.float32, device="cuda")
    fb = 1 if wl.overflow == "fallback" else 0
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    offs = torch.empty(N + 1 + fb, dtype=torch.int32, device="cuda")
    fp8 = wl.dispatch == "fp8"
    perm = inv = drop = xp = xs = yp = None
    if a.stage in ("dispatch", "ffn"):
        perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
        drop = torch.empty(T * k, dtype=torch.uint8, device="cuda")
        xp = torch.empty((T * k, d), dtype=torch.uint8 if fp8 else tdt, device="cuda")
        xs = torch.empty(T * k, dtype=torch.float32, device="cuda") if fp8 else None
        yp = torch.empty((T * k, d), dtype=tdt, device="cuda")
    y = torch.empty((T, d), dtype=tdt, device="cuda")

    def router():
        moe.moe_router(cfg, dev["x"], dev["Wg"], dev.get("bias"), None, idx, gw, pm, ws)

    def dispatch():
        moe.moe_dispatch(cfg, dev["x"], idx, counts, offs, perm, inv, drop, xp, xs, pm, None,
                         None, ws)

    def ffn():
        moe.moe_expert_ffn(cfg, xp, xs, offs, dev["W1"], dev.get("W3"), dev["W2"], yp, ws)

    def layer():
        moe.moe_layer_forward(cfg, dev["x"], dev["Wg"], dev.get("bias"), dev["W1"], dev.get("W3"),
                              dev["W2"], dev.get("Ws1"), dev.get("Ws3"), dev.get("Ws2"), y, idx,
                              gw, counts, None, pm, None, ws)

    if a.stage in ("dispatch", "ffn"):
        router()
    if a.stage == "ffn":
        dispatch()
    run = {"router": router, "dispatch": dispatch, "ffn": ffn, "layer": layer}[a.stage]
    for _ in range(a.warmup + a.iters):
        run()
    torch.cuda.synchronize()
    st, word = moe.moe_check_status(ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status {moe.status_string(st)} ({word:#x})")
    print(f"{a.stage} of {wl.name} (T={T}, N={N}): {a.warmup + a.iters} runs, "
          f"{moe.moe_launch_count()} kernel launches")
    return 0


if __name__ == "__main__":
    sys.exit(main())
