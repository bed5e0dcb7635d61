"""C-ABI checks that need no GPU: the library loads, exports every function
include/moe.h declares, and rejects bad arguments on the host before any
launch."""
import ctypes
import os
import re

import pytest

import top_routing_expert_warp_b200 as moe
from top_routing_expert_warp_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "moe_layer_forward" in names and len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(moe.EXPORTS) | {"moe_layer_forward"}


def test_version_and_status_strings(lib):
    assert "sm_100a" in moe.moe_version()
    assert moe.status_string(moe.MOE_OK) == "ok"
    assert "workspace" in moe.status_string(moe.MOE_ERR_WORKSPACE)


def test_workspace_bytes_and_config_validation(lib):
    good = moe.make_config(4096, 4096, 8, 2, 14336)
    n = moe.moe_workspace_bytes(good)
    # the hidden activations h and y_perm dominate: 8192 rows x (14336 + 4096) bf16
    # (the fused path gathers token rows straight from x, so no x_perm copy)
    assert n >= 8192 * (14336 + 4096) * 2
    assert n % 256 == 0
    bad = [moe.make_config(16, 4096, 8, 9, 128),          # k > 8
           moe.make_config(16, 4096, 4, 5, 128),          # k > N
           moe.make_config(16, 4100, 8, 2, 128),          # d not a multiple of 8 (bf16)
           moe.make_config(16, 64, 300, 2, 128),          # N > 256
           moe.make_config(16, 64, 32, 2, 128, dtype="f32"),  # fp32 layers: N <= 16
           moe.make_config(16, 64, 8, 2, 128, dtype="f32", dispatch_dtype="fp8")]
    for c in bad:
        assert moe.moe_workspace_bytes(c) == 0


def test_entry_points_reject_bad_arguments_before_launch(lib):
    cfg = moe.make_config(16, 64, 8, 2, 128)
    nbytes = moe.moe_workspace_bytes(cfg)
    P = ctypes.c_void_p
    fake = 1 << 40          # never dereferenced: validation fails first
    # null workspace
    r = lib.moe_combine(ctypes.byref(cfg), P(fake), P(fake), P(fake), None, P(fake), None, nbytes, None)
    assert r == moe.MOE_ERR_WORKSPACE
    # misaligned workspace
    r = lib.moe_combine(ctypes.byref(cfg), P(fake), P(fake), P(fake), None, P(fake), P(fake + 8),
                        nbytes, None)
    assert r == moe.MOE_ERR_WORKSPACE
    # too small
    r = lib.moe_combine(ctypes.byref(cfg), P(fake), P(fake), P(fake), None, P(fake), P(fake),
                        nbytes - 256, None)
    assert r == moe.MOE_ERR_WORKSPACE
    # null required pointer
    r = lib.moe_router(ctypes.byref(cfg), None, P(fake), None, None, P(fake), P(fake), None,
                       P(fake), nbytes, None)
    assert r == moe.MOE_ERR_INVALID_ARG
    # misaligned activation
    r = lib.moe_router(ctypes.byref(cfg), P(fake + 2), P(fake), None, None, P(fake), P(fake), None,
                       P(fake), nbytes, None)
    assert r == moe.MOE_ERR_INVALID_ARG
    # aux loss without p_mean
    r = lib.moe_dispatch(ctypes.byref(cfg), P(fake), P(fake), P(fake), P(fake), P(fake), P(fake),
                         P(fake), P(fake), None, None, None, P(fake), P(fake), nbytes, None)
    assert r == moe.MOE_ERR_INVALID_ARG
    # FP8 dispatch without the scale buffer
    c8 = moe.make_config(16, 64, 8, 2, 128, dispatch_dtype="fp8")
    r = lib.moe_dispatch(ctypes.byref(c8), P(fake), P(fake), P(fake), P(fake), P(fake), P(fake),
                         P(fake), P(fake), None, None, None, None, P(fake),
                         moe.moe_workspace_bytes(c8), None)
    assert r == moe.MOE_ERR_INVALID_ARG
    # invalid config
    badc = moe.make_config(16, 64, 8, 9, 128)
    r = lib.moe_layer_forward(ctypes.byref(badc), *([None] * 17), 0, None)
    assert r == moe.MOE_ERR_INVALID_ARG


def test_node_limited_config_validation(lib):
    # host-only: invalid node layouts make the configuration invalid (0 bytes)
    ok = dict(T=64, d=128, N=64, k=4, H=128, dtype="bf16", gate_mode="R", n_groups=8, topk_groups=2)
    assert moe.moe_workspace_bytes(moe.make_config(**ok)) > 0
    assert moe.moe_workspace_bytes(moe.make_config(**{**ok, "n_groups": 0, "topk_groups": 0})) > 0
    for bad in ({"n_groups": 7},                          # N not a multiple of the nodes
                {"N": 128, "n_groups": 64},               # more than 32 nodes
                {"k": 8, "topk_groups": 1, "n_groups": 16},   # 4 experts allowed, k = 8
                {"n_groups": -1}, {"topk_groups": -2}):
        assert moe.moe_workspace_bytes(moe.make_config(**{**ok, **bad})) == 0, bad
    # the C struct and its ctypes mirror agree on the appended fields
    import ctypes
    assert ctypes.sizeof(moe.moe_config) == 72


def test_config_struct_matches_its_ctypes_mirror():
    # the header's moe_config fields, in order, against the binding's mirror
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    body = re.search(r"typedef struct moe_config \{(.*?)\} moe_config;", txt, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    decl = re.findall(r"\b(int64_t|int32_t|float)\s+([^;]+);", body)
    fields = []
    for ctype, names in decl:
        for n in names.split(","):
            fields.append((n.strip(), ctype))
    ct = {"int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "float": ctypes.c_float}
    mirror = [(n, t) for n, t in moe.moe_config._fields_]
    assert [n for n, _ in fields] == [n for n, _ in mirror]
    assert all(ct[c] is t for (_, c), (_, t) in zip(fields, mirror))


def test_capacity_variant_config_validation(lib):
    ok = dict(T=64, d=128, N=8, k=2, H=128, dtype="bf16", capacity_factor=1.0)
    assert moe.moe_workspace_bytes(moe.make_config(**ok, overflow="fallback", slot_priority=True)) > 0
    for field, bad in (("overflow", 2), ("slot_priority", 2), ("overflow", -1)):
        cfg = moe.make_config(**ok)
        setattr(cfg, field, bad)
        assert moe.moe_workspace_bytes(cfg) == 0, (field, bad)


def test_workspace_layout_regions(lib):
    # host-only: the regions of the layer's intermediates lie inside the workspace,
    # 256-byte aligned, in the header's order, each large enough for its array
    cfg = moe.make_config(4096, 7168, 256, 8, 2048, H_shared=2048, gate_mode="F",
                          renormalize=True, dispatch_dtype="fp8")
    r = moe.moe_workspace_layout(cfg)
    assert r["total"] == moe.moe_workspace_bytes(cfg)
    order = ["topk_idx", "topk_w", "counts", "offsets", "perm", "inv_row", "drop", "x_scale",
             "x_gemm"]
    offs = [r[n] for n in order]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs) and offs[-1] < r["total"]
    rows = 4096 * 8
    need = {"topk_idx": rows * 4, "topk_w": rows * 4, "counts": 256 * 4, "offsets": 258 * 4,
            "perm": rows * 4, "inv_row": rows * 4, "drop": rows, "x_scale": rows * 4,
            "x_gemm": rows * 7168 * 2}
    nxt = offs[1:] + [r["total"]]
    for n, o, e in zip(order, offs, nxt):
        assert e - o >= need[n], n
    # the ctypes mirror has the header's fields in order
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    body = re.search(r"typedef struct moe_workspace_regions \{(.*?)\} moe_workspace_regions;", txt,
                     flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    assert re.findall(r"size_t\s+(\w+);", body) == [n for n, _ in moe.moe_workspace_regions._fields_]
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_layout(moe.make_config(16, 64, 8, 9, 128))   # k > 8
