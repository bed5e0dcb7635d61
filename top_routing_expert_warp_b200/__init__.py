"""Python binding of libmoe_b200: the forward pass of one Mixture-of-Experts layer
on an NVIDIA B200 (sm_100a).

The binding only marshals arguments: every stage runs in the CUDA kernels of
``libmoe_b200.so`` (declared in ``include/moe.h``).  PyTorch supplies device
memory and streams.  There is no CPU path: when the library is missing or no
CUDA device is present, the calls raise.

Entry points (same names as the C ABI):
    moe_workspace_bytes, moe_router, moe_dispatch, moe_expert_ffn, moe_combine,
    moe_layer_forward, moe_check_status, moe_status_string, moe_version.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_DEVICE_STATUS, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_F32, MOE_BF16, MOE_FP8_E4M3 = 0, 1, 2
MOE_GATE_TOPK_THEN_SOFTMAX, MOE_GATE_SOFTMAX_THEN_TOPK = 0, 1
MOE_ACT_RELU, MOE_ACT_SWIGLU = 0, 1
MOE_OVERFLOW_DROP, MOE_OVERFLOW_FALLBACK = 0, 1

EXPORTS = ("moe_workspace_bytes", "moe_router", "moe_dispatch", "moe_expert_ffn", "moe_combine",
           "moe_layer_forward", "moe_check_status", "moe_status_string", "moe_last_error_string",
           "moe_version", "moe_launch_count", "moe_profile_begin", "moe_profile_end",
           "moe_dispatch_noalloc", "moe_expert_ffn_multi", "moe_workspace_layout")
PROFILE_STAGES = ("router", "dispatch", "expert_up", "expert_down", "shared_expert", "combine")


class moe_config(ctypes.Structure):
    """Mirror of ``struct moe_config`` in include/moe.h."""
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("k", ctypes.c_int32), ("H", ctypes.c_int32), ("H_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("gate_mode", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("act", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("dispatch_dtype", ctypes.c_int32),
                ("aux_alpha", ctypes.c_float), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("overflow", ctypes.c_int32),
                ("slot_priority", ctypes.c_int32)]


class moe_workspace_regions(ctypes.Structure):
    """Mirror of ``struct moe_workspace_regions`` in include/moe.h."""
    _fields_ = [(n, ctypes.c_size_t) for n in ("topk_idx", "topk_w", "counts", "offsets", "perm",
                                               "inv_row", "drop", "x_scale", "x_gemm",
                                               "total")]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == MOE_ERR_CUDA:
            msg += f" ({last_error_string()})"
        super().__init__(msg)


_lib = None


def lib():
    """The loaded ``libmoe_b200.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               f"`python -m top_routing_expert_warp_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        cfgp = ctypes.POINTER(moe_config)
        L.moe_workspace_bytes.argtypes = [cfgp]
        L.moe_workspace_bytes.restype = ctypes.c_size_t
        L.moe_workspace_layout.argtypes = [cfgp, ctypes.POINTER(moe_workspace_regions)]
        L.moe_workspace_layout.restype = ctypes.c_int
        L.moe_router.argtypes = [cfgp, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_dispatch.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_dispatch_noalloc.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.moe_dispatch_noalloc.restype = ctypes.c_int
        L.moe_expert_ffn.argtypes = [cfgp, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_expert_ffn_multi.argtypes = [cfgp, ctypes.c_int32, ctypes.c_int64, P, P, P, P, P, P, P,
                                           P, ctypes.c_size_t, P]
        L.moe_combine.argtypes = [cfgp, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_layer_forward.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                        ctypes.c_size_t, P]
        L.moe_check_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
        for f in ("moe_router", "moe_dispatch", "moe_expert_ffn", "moe_expert_ffn_multi",
                  "moe_combine", "moe_layer_forward", "moe_check_status"):
            getattr(L, f).restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_last_error_string.restype = ctypes.c_char_p
        L.moe_version.restype = ctypes.c_char_p
        L.moe_launch_count.restype = ctypes.c_uint64
        L.moe_profile_begin.argtypes = [ctypes.c_int]
        L.moe_profile_begin.restype = ctypes.c_int
        L.moe_profile_end.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
        L.moe_profile_end.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


def last_error_string() -> str:
    return lib().moe_last_error_string().decode()


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_status_string(s: int) -> str:
    return status_string(s)


# ------------------------------------------------------------------ marshalling
def _ptr(t):
    """Device (or host) address of a tensor, or None for NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def make_config(T, d, N, k, H, *, H_shared=0, capacity_factor=0.0, gate_mode="R",
                renormalize=False, act="swiglu", dtype="bf16", dispatch_dtype=None,
                aux_alpha=0.01, n_groups=0, topk_groups=0, overflow="drop",
                slot_priority=False) -> moe_config:
    dt = {"f32": MOE_F32, "bf16": MOE_BF16}[dtype]
    dd = dt if dispatch_dtype in (None, "", dtype) else {"fp8": MOE_FP8_E4M3}[dispatch_dtype]
    return moe_config(int(T), int(d), int(N), int(k), int(H), int(H_shared),
                      float(capacity_factor),
                      MOE_GATE_TOPK_THEN_SOFTMAX if gate_mode == "R" else MOE_GATE_SOFTMAX_THEN_TOPK,
                      int(bool(renormalize)), MOE_ACT_RELU if act == "relu" else MOE_ACT_SWIGLU,
                      dt, dd, float(aux_alpha), int(n_groups), int(topk_groups),
                      {"drop": MOE_OVERFLOW_DROP, "fallback": MOE_OVERFLOW_FALLBACK}[overflow],
                      int(bool(slot_priority)))


def config_from(spec) -> moe_config:
    """``make_config`` from any object with the layer's fields as attributes
    (T, d, N, k, H, act, dtype, gate_mode and, when present, H_shared,
    capacity_factor, renormalize, dispatch, aux_alpha, n_groups, topk_groups,
    overflow, slot_priority), so that every switch of the layer is passed."""
    g = lambda name, default: getattr(spec, name, default)  # noqa: E731
    return make_config(spec.T, spec.d, spec.N, spec.k, spec.H, H_shared=g("H_shared", 0),
                       capacity_factor=g("capacity_factor", 0.0), gate_mode=spec.gate_mode,
                       renormalize=g("renormalize", False), act=spec.act, dtype=spec.dtype,
                       dispatch_dtype=g("dispatch", None) or None, aux_alpha=g("aux_alpha", 0.01),
                       n_groups=g("n_groups", 0), topk_groups=g("topk_groups", 0),
                       overflow=g("overflow", "drop"), slot_priority=g("slot_priority", False))


def moe_workspace_bytes(cfg: moe_config) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(cfg)))


def moe_workspace_layout(cfg: moe_config) -> dict:
    """Byte offsets of the layer forward's intermediate regions in the workspace."""
    r = moe_workspace_regions()
    _check(lib().moe_workspace_layout(ctypes.byref(cfg), ctypes.byref(r)), "moe_workspace_layout")
    return {n: int(getattr(r, n)) for n, _ in moe_workspace_regions._fields_}


def workspace_view(ws, cfg: moe_config, region: str, dtype, count: int):
    """A typed view of ``count`` elements of a workspace region (no copy)."""
    import torch
    off = moe_workspace_layout(cfg)[region]
    esz = torch.empty((), dtype=dtype).element_size()
    return ws[off:off + count * esz].view(dtype)


def moe_router(cfg, x, Wg, bias, logits, topk_idx, topk_w, p_mean, workspace, stream=None):
    _check(lib().moe_router(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(logits),
                            _ptr(topk_idx), _ptr(topk_w), _ptr(p_mean), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_router")


def moe_dispatch(cfg, x, topk_idx, expert_counts, expert_offsets, perm, inv_row, drop_mask,
                 x_perm, x_scale, p_mean, f, aux_loss, workspace, stream=None):
    _check(lib().moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(expert_counts),
                              _ptr(expert_offsets), _ptr(perm), _ptr(inv_row), _ptr(drop_mask),
                              _ptr(x_perm), _ptr(x_scale), _ptr(p_mean), _ptr(f), _ptr(aux_loss),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)),
           "moe_dispatch")


def moe_dispatch_noalloc(cfg, x, topk_idx, expert_counts, expert_offsets, perm, inv_row,
                         drop_mask, x_perm, x_scale, p_mean, f, aux_loss, stream=None):
    """moe_dispatch for callers that cannot allocate a workspace: the library's
    built-in scratch array is used instead (T*k <= 262144, N <= 256; calls on
    one device must not overlap on the GPU)."""
    _check(lib().moe_dispatch_noalloc(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx),
                                      _ptr(expert_counts), _ptr(expert_offsets), _ptr(perm),
                                      _ptr(inv_row), _ptr(drop_mask), _ptr(x_perm), _ptr(x_scale),
                                      _ptr(p_mean), _ptr(f), _ptr(aux_loss), _stream(stream)),
           "moe_dispatch_noalloc")


def moe_expert_ffn(cfg, x_perm, x_scale, expert_offsets, W1, W3, W2, y_perm, workspace,
                   stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(x_perm), _ptr(x_scale),
                                _ptr(expert_offsets), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(y_perm),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)),
           "moe_expert_ffn")


def moe_expert_ffn_multi(cfg, n_src, rows_cap, x_rows, x_scale, offsets, W1, W3, W2, y_rows,
                         workspace, stream=None):
    _check(lib().moe_expert_ffn_multi(ctypes.byref(cfg), int(n_src), int(rows_cap), _ptr(x_rows),
                                      _ptr(x_scale), _ptr(offsets), _ptr(W1), _ptr(W3), _ptr(W2),
                                      _ptr(y_rows), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)),
           "moe_expert_ffn_multi")


def moe_combine(cfg, y_perm, inv_row, topk_w, y_shared, y, workspace, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _ptr(y_perm), _ptr(inv_row), _ptr(topk_w),
                             _ptr(y_shared), _ptr(y), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_combine")


def moe_layer_forward(cfg, x, Wg, bias, W1, W3, W2, Ws1, Ws3, Ws2, y, topk_idx, topk_w,
                      expert_counts, f, p_mean, aux_loss, workspace, stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1),
                                   _ptr(W3), _ptr(W2), _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _ptr(y),
                                   _ptr(topk_idx), _ptr(topk_w), _ptr(expert_counts), _ptr(f),
                                   _ptr(p_mean), _ptr(aux_loss), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_layer_forward")


def moe_check_status(workspace, stream=None):
    """(status, raw word); synchronises the stream and clears the word."""
    word = ctypes.c_uint32(0)
    s = lib().moe_check_status(_ptr(workspace), _stream(stream), ctypes.byref(word))
    return int(s), int(word.value)


def moe_launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().moe_launch_count())


def moe_profile_begin(max_steps: int):
    _check(lib().moe_profile_begin(int(max_steps)), "moe_profile_begin")


def moe_profile_end():
    """(dict stage -> summed ms, number of recorded moe_layer_forward calls)."""
    arr = (ctypes.c_float * len(PROFILE_STAGES))()
    n = ctypes.c_int(0)
    _check(lib().moe_profile_end(arr, ctypes.byref(n)), "moe_profile_end")
    return {name: float(arr[i]) for i, name in enumerate(PROFILE_STAGES)}, int(n.value)


def workspace(cfg: moe_config, device="cuda"):
    """A zero-filled workspace tensor of the size ``cfg`` needs."""
    import torch
    n = moe_workspace_bytes(cfg)
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)
