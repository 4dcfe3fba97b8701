"""Python binding of ``libmoe_w8a8.so``, the B200 W8A8 mixture-of-experts layer.

Argument marshalling only: every function here has the name of the C entry
point it calls (see ``include/moe_w8a8.h``), turns tensors into pointers,
checks their dtype / device / contiguity, and raises ``MoeError`` on a
non-OK status.  All of the layer's work runs in the library's CUDA kernels;
there is no fallback, and importing a missing library fails loudly.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_w8a8.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_OOM = 6

MOE_F32 = 0
MOE_BF16 = 1

MOE_FMT_INT8 = 0
MOE_FMT_E4M3 = 1

MOE_PATH_AUTO = 0
MOE_PATH_STREAM = 1
MOE_PATH_TENSOR = 2

# Every entry point declared in include/moe_w8a8.h.
EXPORTS = (
    "moe_w8a8_calibrate_absmax", "moe_w8a8_prepare", "moe_w8a8_workspace_size",
    "moe_w8a8_forward", "moe_w8a8_forward_host", "moe_w8a8_set_path",
    "moe_w8a8_set_stream_threshold", "moe_w8a8_get_smooth_scales", "moe_w8a8_export_weights",
    "moe_w8a8_check_status", "moe_w8a8_destroy", "moe_status_string",
    "moe_w8a8_last_launch_count", "moe_w8a8_profile_start", "moe_w8a8_profile_start_stages", "moe_w8a8_profile_read",
    "moe_w8a8_profile_stop", "moe_w8a8_stage_name", "moe_w8a8_forward_noalloc",
    "moe_w8a8_status_words", "moe_w8a8_set_act_clip", "moe_w8a8_calibrate_act_clip",
    "moe_w8a8_ep_row_bytes", "moe_w8a8_gateup_absmax", "moe_w8a8_prepare_shard",
    "moe_w8a8_ep_dispatch_workspace_size", "moe_w8a8_ep_experts_workspace_size",
    "moe_w8a8_ep_dispatch", "moe_w8a8_ep_experts", "moe_w8a8_ep_combine",
    "moe_w8a8_tensor_peak_loop", "moe_w8a8_set_wait_budget", "moe_w8a8_test_withhold_release",
    "moe_w8a8_set_fused_threshold", "moe_w8a8_set_cta_pairs",
    "moe_w8a8_ep_block_rows", "moe_w8a8_ep_pack", "moe_w8a8_ep_experts_blocked_workspace_size",
    "moe_w8a8_ep_experts_blocked", "moe_w8a8_ep_combine_blocked",
)

MOE_NOALLOC_SCRATCH_BYTES = 8 << 20
MOE_PEAK_MAX_MMA = 1 << 24

MOE_N_STAGES = 8


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")


class moe_w8a8_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("capacity_factor", ctypes.c_float), ("renormalize", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("expert_format", ctypes.c_int32)]


_DBG_FIELDS = ("logits", "topk_idx", "topk_w", "offsets", "row2ts", "ts2row", "xq", "sx", "acc1",
               "hq", "sh", "acc2", "o")


class moe_w8a8_debug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _DBG_FIELDS]


_lib = None


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m w8a8_quantized_moe_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        cfgp = ctypes.POINTER(moe_w8a8_config)
        sig = {
            "moe_w8a8_calibrate_absmax": ([vp, i64, i32, i32, vp, vp], i32),
            "moe_w8a8_prepare": ([cfgp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(vp)], i32),
            "moe_w8a8_workspace_size": ([vp, i32], sz),
            "moe_w8a8_forward": ([vp, vp, i32, vp, vp, vp, vp, sz, vp, vp], i32),
            "moe_w8a8_forward_host": ([vp, vp, i32, vp, vp, vp, vp, sz, vp], i32),
            "moe_w8a8_set_path": ([vp, i32], i32),
            "moe_w8a8_set_stream_threshold": ([vp, i32], i32),
            "moe_w8a8_set_act_clip": ([vp, ctypes.c_float], i32),
            "moe_w8a8_calibrate_act_clip": ([vp, vp, i64, i32, ctypes.c_double, vp, vp], i32),
            "moe_w8a8_get_smooth_scales": ([vp, vp], i32),
            "moe_w8a8_export_weights": ([vp, vp, vp, vp, vp, vp, vp, vp, vp], i32),
            "moe_w8a8_check_status": ([vp, vp], i32),
            "moe_w8a8_destroy": ([vp], None),
            "moe_status_string": ([i32], ctypes.c_char_p),
            "moe_w8a8_last_launch_count": ([vp], i32),
            "moe_w8a8_profile_start": ([vp, i32], i32),
            "moe_w8a8_profile_start_stages": ([vp, i32, ctypes.c_uint32], i32),
            "moe_w8a8_profile_read": ([vp, vp, i32], i32),
            "moe_w8a8_profile_stop": ([vp], i32),
            "moe_w8a8_stage_name": ([i32], ctypes.c_char_p),
            "moe_w8a8_forward_noalloc": ([vp, vp, i32, vp, vp, vp, vp], i32),
            "moe_w8a8_status_words": ([vp, vp, i32, vp], i32),
            "moe_w8a8_ep_row_bytes": ([vp], i32),
            "moe_w8a8_gateup_absmax": ([cfgp, i32, vp, vp, vp, vp], i32),
            "moe_w8a8_prepare_shard": ([cfgp, i32, i32, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(vp)], i32),
            "moe_w8a8_ep_dispatch_workspace_size": ([vp, i32], sz),
            "moe_w8a8_ep_experts_workspace_size": ([vp, i32], sz),
            "moe_w8a8_ep_dispatch": ([vp, vp, i32, vp, vp, vp, vp, vp, sz, vp, vp], i32),
            "moe_w8a8_ep_experts": ([vp, vp, i32, vp, vp, sz, vp, vp], i32),
            "moe_w8a8_ep_combine": ([vp, vp, i32, vp, vp, sz, vp], i32),
            "moe_w8a8_tensor_peak_loop": ([i32, i64, ctypes.POINTER(ctypes.c_double), vp], i32),
            "moe_w8a8_set_wait_budget": ([vp, i64], i32),
            "moe_w8a8_set_fused_threshold": ([vp, i64], i32),
            "moe_w8a8_set_cta_pairs": ([vp, i32], i32),
            "moe_w8a8_test_withhold_release": ([vp, i32], i32),
            "moe_w8a8_ep_block_rows": ([vp, i32], i32),
            "moe_w8a8_ep_pack": ([vp, vp, vp, vp, i32, i32, vp, vp], i32),
            "moe_w8a8_ep_experts_blocked_workspace_size": ([vp, i32, i32], sz),
            "moe_w8a8_ep_experts_blocked": ([vp, vp, i32, i32, vp, vp, sz, vp, vp], i32),
            "moe_w8a8_ep_combine_blocked": ([vp, vp, i32, vp, i32, i32, vp, vp, sz, vp], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers

def _torch():
    import torch
    return torch


def _dev_ptr(t, dtype=None, name="tensor", allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _need(t, n: int, name: str):
    """A tensor passed for n elements must hold at least n of them (the
    library indexes it up to there)."""
    if t is None:
        return
    count = int(t.size) if not callable(getattr(t, "size", None)) else t.numel()   # numpy or torch
    if count < n:
        raise ValueError(f"{name} holds {count} elements, the call reads or writes {n}")


def _layer_io(w, x, T: int, router_bias, router_logits, y, suffix: str = ""):
    c = w.cfg
    _need(x, T * c.d, "x" + suffix)
    _need(y, T * c.d, "y" + suffix)
    _need(router_logits, T * c.n_experts, "router_logits" + suffix)
    _need(router_bias, c.n_experts, "router_bias" + suffix)


def _host_ptr(a, name="array", allow_none=False):
    if a is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    try:
        import numpy as np
        if isinstance(a, np.ndarray):
            if not a.flags["C_CONTIGUOUS"]:
                raise ValueError(f"{name} must be C-contiguous")
            return ctypes.c_void_p(a.ctypes.data)
    except ImportError:  # pragma: no cover
        pass
    torch = _torch()
    if isinstance(a, torch.Tensor) and not a.is_cuda and a.is_contiguous():
        return ctypes.c_void_p(a.data_ptr())
    raise TypeError(f"{name} must be a contiguous host array")


def _stream(stream):
    if stream is None:
        torch = _torch()
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _act_dtype(code: int):
    torch = _torch()
    return torch.bfloat16 if code == MOE_BF16 else torch.float32


# ------------------------------------------------------------------ entry points

def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_w8a8_calibrate_absmax(x, absmax, stream=None):
    torch = _torch()
    dt = MOE_BF16 if x.dtype == torch.bfloat16 else MOE_F32
    _check(lib().moe_w8a8_calibrate_absmax(_dev_ptr(x, name="x"), x.shape[0], x.shape[1], dt,
                                           _dev_ptr(absmax, torch.float32, "absmax"),
                                           _stream(stream)), "moe_w8a8_calibrate_absmax")


class Weights:
    """Owner of a prepared-weights handle (destroyed with the object); it
    holds experts [expert_first, expert_first + n_local) of the layer."""

    def __init__(self, handle: ctypes.c_void_p, cfg: moe_w8a8_config, expert_first: int = 0,
                 n_local: int | None = None):
        self.handle = handle
        self.cfg = cfg
        self.expert_first = expert_first
        self.n_local = cfg.n_experts if n_local is None else n_local

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.moe_w8a8_destroy(self.handle)
            self.handle = None


def make_config(d, f, n_experts, top_k, alpha=0.6, capacity_factor=0.0, renormalize=True,
                in_dtype=MOE_BF16, out_dtype=MOE_BF16, expert_format=MOE_FMT_INT8) -> moe_w8a8_config:
    return moe_w8a8_config(d, f, n_experts, top_k, alpha, capacity_factor, 1 if renormalize else 0,
                           in_dtype, out_dtype, expert_format)


def moe_w8a8_prepare(cfg: moe_w8a8_config, w_gate, w_up, w_down, w_router, act_absmax,
                     stream=None) -> Weights:
    torch = _torch()
    f32 = torch.float32
    h = ctypes.c_void_p()
    _check(lib().moe_w8a8_prepare(ctypes.byref(cfg), _dev_ptr(w_gate, f32, "w_gate"),
                                  _dev_ptr(w_up, f32, "w_up"), _dev_ptr(w_down, f32, "w_down"),
                                  _dev_ptr(w_router, f32, "w_router"),
                                  _dev_ptr(act_absmax, f32, "act_absmax"), _stream(stream),
                                  ctypes.byref(h)), "moe_w8a8_prepare")
    return Weights(h, cfg)


def moe_w8a8_workspace_size(w: Weights, max_tokens: int) -> int:
    return int(lib().moe_w8a8_workspace_size(w.handle, int(max_tokens)))


def _debug_struct(dbg: dict | None):
    if not dbg:
        return None, None
    s = moe_w8a8_debug()
    for n in _DBG_FIELDS:
        t = dbg.get(n)
        setattr(s, n, None if t is None else _dev_ptr(t, name=f"dbg.{n}").value)
    return s, ctypes.byref(s)


def moe_w8a8_forward(w: Weights, x, T: int, router_bias, router_logits, y, workspace,
                     dbg: dict | None = None, stream=None):
    torch = _torch()
    _layer_io(w, x, T, router_bias, router_logits, y)
    _s, dptr = _debug_struct(dbg)
    _check(lib().moe_w8a8_forward(
        w.handle, _dev_ptr(x, _act_dtype(w.cfg.in_dtype), "x"), int(T),
        _dev_ptr(router_bias, torch.float32, "router_bias", True),
        _dev_ptr(router_logits, torch.float32, "router_logits", True),
        _dev_ptr(y, _act_dtype(w.cfg.out_dtype), "y"), _dev_ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), dptr, _stream(stream)), "moe_w8a8_forward")


def moe_w8a8_forward_host(w: Weights, x_host, T: int, router_bias_host, router_logits_host,
                          y_host, workspace, stream=None):
    _layer_io(w, x_host, T, router_bias_host, router_logits_host, y_host, "_host")
    _check(lib().moe_w8a8_forward_host(
        w.handle, _host_ptr(x_host, "x_host"), int(T),
        _host_ptr(router_bias_host, "router_bias_host", True),
        _host_ptr(router_logits_host, "router_logits_host", True), _host_ptr(y_host, "y_host"),
        _dev_ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)), "moe_w8a8_forward_host")


def moe_w8a8_set_path(w: Weights, path: int):
    _check(lib().moe_w8a8_set_path(w.handle, int(path)), "moe_w8a8_set_path")


def moe_w8a8_set_stream_threshold(w: Weights, max_rows: int):
    _check(lib().moe_w8a8_set_stream_threshold(w.handle, int(max_rows)),
           "moe_w8a8_set_stream_threshold")


def moe_w8a8_set_fused_threshold(w: Weights, max_rows: int):
    _check(lib().moe_w8a8_set_fused_threshold(w.handle, int(max_rows)), "moe_w8a8_set_fused_threshold")


def moe_w8a8_set_cta_pairs(w: Weights, mode: int):
    _check(lib().moe_w8a8_set_cta_pairs(w.handle, int(mode)), "moe_w8a8_set_cta_pairs")


def moe_w8a8_set_act_clip(w: Weights, clip: float):
    _check(lib().moe_w8a8_set_act_clip(w.handle, float(clip)), "moe_w8a8_set_act_clip")


def moe_w8a8_calibrate_act_clip(w: Weights, x, percent: float, stream=None) -> float:
    torch = _torch()
    dt = MOE_BF16 if x.dtype == torch.bfloat16 else MOE_F32
    out = ctypes.c_float(0.0)
    _check(lib().moe_w8a8_calibrate_act_clip(w.handle, _dev_ptr(x, name="x"), x.shape[0], dt, float(percent),
                                             ctypes.byref(out), _stream(stream)),
           "moe_w8a8_calibrate_act_clip")
    return float(out.value)


def moe_w8a8_get_smooth_scales(w: Weights):
    import numpy as np
    out = np.empty(w.cfg.d, dtype=np.float32)
    _check(lib().moe_w8a8_get_smooth_scales(w.handle, ctypes.c_void_p(out.ctypes.data)),
           "moe_w8a8_get_smooth_scales")
    return out


def moe_w8a8_export_weights(w: Weights, stream=None) -> dict:
    torch = _torch()
    c = w.cfg
    E, d, f = w.n_local, c.d, c.f
    dev = torch.device("cuda")
    out = dict(wq_gate=torch.empty((E, f, d), dtype=torch.int8, device=dev),
               wq_up=torch.empty((E, f, d), dtype=torch.int8, device=dev),
               sw_gate=torch.empty((E, f), dtype=torch.float32, device=dev),
               sw_up=torch.empty((E, f), dtype=torch.float32, device=dev),
               wq_down=torch.empty((E, d, f), dtype=torch.int8, device=dev),
               sw_down=torch.empty((E, d), dtype=torch.float32, device=dev),
               inv_s=torch.empty((d,), dtype=torch.float32, device=dev))
    _check(lib().moe_w8a8_export_weights(w.handle, *(ctypes.c_void_p(out[k].data_ptr()) for k in
                                                     ("wq_gate", "wq_up", "sw_gate", "sw_up",
                                                      "wq_down", "sw_down", "inv_s")),
                                         _stream(stream)), "moe_w8a8_export_weights")
    return out


def moe_w8a8_check_status(w: Weights, stream=None):
    _check(lib().moe_w8a8_check_status(w.handle, _stream(stream)), "moe_w8a8_check_status")


def moe_w8a8_last_launch_count(w: Weights) -> int:
    return int(lib().moe_w8a8_last_launch_count(w.handle))


def moe_w8a8_profile_start(w: Weights, max_forwards: int):
    _check(lib().moe_w8a8_profile_start(w.handle, int(max_forwards)), "moe_w8a8_profile_start")


def moe_w8a8_profile_start_stages(w: Weights, max_forwards: int, stages):
    """Event pairs around the listed stages only (indices into STAGE_NAMES)."""
    mask = 0
    for st in stages:
        mask |= 1 << int(st)
    _check(lib().moe_w8a8_profile_start_stages(w.handle, int(max_forwards), mask),
           "moe_w8a8_profile_start_stages")


def moe_w8a8_profile_read(w: Weights, capacity: int):
    """Per-stage milliseconds of the recorded forwards: numpy [n][MOE_N_STAGES]."""
    import numpy as np
    out = np.zeros((capacity, MOE_N_STAGES), dtype=np.float32)
    n = lib().moe_w8a8_profile_read(w.handle, ctypes.c_void_p(out.ctypes.data), int(capacity))
    if n < 0:
        raise MoeError(MOE_ERR_CUDA, "moe_w8a8_profile_read")
    return out[:n]


def moe_w8a8_profile_stop(w: Weights):
    _check(lib().moe_w8a8_profile_stop(w.handle), "moe_w8a8_profile_stop")


def moe_w8a8_stage_name(stage: int) -> str:
    return lib().moe_w8a8_stage_name(int(stage)).decode()


STAGE_NAMES = ("router", "topk", "permute", "quant", "gemm1", "requant", "gemm2", "combine")


def moe_w8a8_forward_noalloc(w: Weights, x, T: int, router_bias, router_logits, y, stream=None):
    """Forward for callers that cannot allocate: scratch comes from the
    library's fixed device array (see the header); no workspace argument."""
    torch = _torch()
    _layer_io(w, x, T, router_bias, router_logits, y)
    _check(lib().moe_w8a8_forward_noalloc(
        w.handle, _dev_ptr(x, _act_dtype(w.cfg.in_dtype), "x"), int(T),
        _dev_ptr(router_bias, torch.float32, "router_bias", True),
        _dev_ptr(router_logits, torch.float32, "router_logits", True),
        _dev_ptr(y, _act_dtype(w.cfg.out_dtype), "y"), _stream(stream)), "moe_w8a8_forward_noalloc")


def moe_w8a8_set_wait_budget(w: Weights, ns: int):
    _check(lib().moe_w8a8_set_wait_budget(w.handle, int(ns)), "moe_w8a8_set_wait_budget")


def moe_w8a8_test_withhold_release(w: Weights, m_tile: int):
    _check(lib().moe_w8a8_test_withhold_release(w.handle, int(m_tile)), "moe_w8a8_test_withhold_release")


def moe_w8a8_status_words(w: Weights, n: int = 5, stream=None):
    """The handle's status words (code, then where a bounded wait gave up)."""
    import numpy as np
    out = np.zeros(n, dtype=np.int32)
    _check(lib().moe_w8a8_status_words(w.handle, ctypes.c_void_p(out.ctypes.data), int(n),
                                       _stream(stream)), "moe_w8a8_status_words")
    return out


# ------------------------------------------------------------------ expert parallelism

def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def moe_w8a8_ep_row_bytes(w: Weights) -> int:
    return int(lib().moe_w8a8_ep_row_bytes(w.handle))


def moe_w8a8_gateup_absmax(cfg: moe_w8a8_config, w_gate, w_up, aw, stream=None):
    torch = _torch()
    f32 = torch.float32
    _check(lib().moe_w8a8_gateup_absmax(ctypes.byref(cfg), int(w_gate.shape[0]), _dev_ptr(w_gate, f32, "w_gate"),
                                        _dev_ptr(w_up, f32, "w_up"), _dev_ptr(aw, f32, "aw"), _stream(stream)),
           "moe_w8a8_gateup_absmax")


def moe_w8a8_prepare_shard(cfg: moe_w8a8_config, expert_first: int, w_gate, w_up, w_down, w_router,
                           act_absmax, gateup_absmax, stream=None) -> Weights:
    torch = _torch()
    f32 = torch.float32
    n_local = int(w_gate.shape[0])
    h = ctypes.c_void_p()
    _check(lib().moe_w8a8_prepare_shard(ctypes.byref(cfg), int(expert_first), n_local,
                                        _dev_ptr(w_gate, f32, "w_gate"), _dev_ptr(w_up, f32, "w_up"),
                                        _dev_ptr(w_down, f32, "w_down"), _dev_ptr(w_router, f32, "w_router"),
                                        _dev_ptr(act_absmax, f32, "act_absmax"),
                                        _dev_ptr(gateup_absmax, f32, "gateup_absmax"), _stream(stream),
                                        ctypes.byref(h)), "moe_w8a8_prepare_shard")
    return Weights(h, cfg, int(expert_first), n_local)


def moe_w8a8_ep_dispatch_workspace_size(w: Weights, max_tokens: int) -> int:
    return int(lib().moe_w8a8_ep_dispatch_workspace_size(w.handle, int(max_tokens)))


def moe_w8a8_ep_experts_workspace_size(w: Weights, rows: int) -> int:
    return int(lib().moe_w8a8_ep_experts_workspace_size(w.handle, int(rows)))


def moe_w8a8_ep_dispatch(w: Weights, x, T: int, router_bias, router_logits, send, expert_offsets, workspace,
                         dbg: dict | None = None, stream=None):
    torch = _torch()
    c = w.cfg
    _need(x, T * c.d, "x")
    _need(router_logits, T * c.n_experts, "router_logits")
    _need(router_bias, c.n_experts, "router_bias")
    _need(send, T * c.top_k * moe_w8a8_ep_row_bytes(w), "send")
    _need(expert_offsets, c.n_experts + 1, "expert_offsets")
    _s, dptr = _debug_struct(dbg)
    _check(lib().moe_w8a8_ep_dispatch(
        w.handle, _dev_ptr(x, _act_dtype(w.cfg.in_dtype), "x", T == 0), int(T),
        _dev_ptr(router_bias, torch.float32, "router_bias", True),
        _dev_ptr(router_logits, torch.float32, "router_logits", True),
        _dev_ptr(send, torch.uint8, "send", T == 0), _dev_ptr(expert_offsets, torch.int32, "expert_offsets"),
        _dev_ptr(workspace, name="workspace", allow_none=T == 0),
        0 if workspace is None else _nbytes(workspace), dptr, _stream(stream)), "moe_w8a8_ep_dispatch")


def moe_w8a8_ep_experts(w: Weights, recv, R: int, o_rows, workspace, dbg: dict | None = None, stream=None):
    torch = _torch()
    if R == 0:
        return
    _need(recv, R * moe_w8a8_ep_row_bytes(w), "recv")
    _need(o_rows, R * w.cfg.d, "o_rows")
    _s, dptr = _debug_struct(dbg)
    _check(lib().moe_w8a8_ep_experts(
        w.handle, _dev_ptr(recv, torch.uint8, "recv"), int(R), _dev_ptr(o_rows, torch.float32, "o_rows"),
        _dev_ptr(workspace, name="workspace"), _nbytes(workspace), dptr, _stream(stream)), "moe_w8a8_ep_experts")


def moe_w8a8_ep_combine(w: Weights, o_rows, T: int, y, workspace, stream=None):
    torch = _torch()
    if T == 0:
        return
    _need(y, T * w.cfg.d, "y")
    # o_rows may hold no rows (every slot dropped), but its pointer must be a
    # real device address: the library refuses NULL
    o_ptr = ctypes.c_void_p(o_rows.data_ptr()) if o_rows is not None and o_rows.is_cuda else None
    _check(lib().moe_w8a8_ep_combine(
        w.handle, o_ptr, int(T), _dev_ptr(y, _act_dtype(w.cfg.out_dtype), "y"),
        _dev_ptr(workspace, name="workspace"), _nbytes(workspace), _stream(stream)), "moe_w8a8_ep_combine")


# fixed-block exchange (no row count reaches the host)

def moe_w8a8_ep_block_rows(w: Weights, block_tokens: int) -> int:
    return int(lib().moe_w8a8_ep_block_rows(w.handle, int(block_tokens)))


def _rank_first(rank_first):
    """Host int32 [G + 1] array of the ranks' first experts (kept alive by the caller)."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(rank_first, dtype=np.int32))
    return a, ctypes.c_void_p(a.ctypes.data), len(a) - 1


def moe_w8a8_ep_pack(w: Weights, send, expert_offsets, rank_first, block_tokens: int, blocks, stream=None):
    torch = _torch()
    a, ptr, world = _rank_first(rank_first)
    rb = moe_w8a8_ep_row_bytes(w)
    _need(expert_offsets, w.cfg.n_experts + 1, "expert_offsets")
    _need(blocks, world * moe_w8a8_ep_block_rows(w, block_tokens) * rb, "blocks")
    _check(lib().moe_w8a8_ep_pack(
        w.handle, _dev_ptr(send, torch.uint8, "send"), _dev_ptr(expert_offsets, torch.int32, "expert_offsets"),
        ptr, int(world), int(block_tokens), _dev_ptr(blocks, torch.uint8, "blocks"), _stream(stream)),
        "moe_w8a8_ep_pack")


def moe_w8a8_ep_experts_blocked_workspace_size(w: Weights, world: int, block_tokens: int) -> int:
    return int(lib().moe_w8a8_ep_experts_blocked_workspace_size(w.handle, int(world), int(block_tokens)))


def moe_w8a8_ep_experts_blocked(w: Weights, blocks, world: int, block_tokens: int, o_blocks, workspace,
                                dbg: dict | None = None, stream=None):
    torch = _torch()
    rows = int(world) * moe_w8a8_ep_block_rows(w, block_tokens)
    _need(blocks, rows * moe_w8a8_ep_row_bytes(w), "blocks")
    _need(o_blocks, rows * w.cfg.d, "o_blocks")
    _s, dptr = _debug_struct(dbg)
    _check(lib().moe_w8a8_ep_experts_blocked(
        w.handle, _dev_ptr(blocks, torch.uint8, "blocks"), int(world), int(block_tokens),
        _dev_ptr(o_blocks, torch.float32, "o_blocks"), _dev_ptr(workspace, name="workspace"), _nbytes(workspace),
        dptr, _stream(stream)), "moe_w8a8_ep_experts_blocked")


def moe_w8a8_ep_combine_blocked(w: Weights, o_blocks, T: int, rank_first, block_tokens: int, y, workspace,
                                stream=None):
    torch = _torch()
    a, ptr, world = _rank_first(rank_first)
    if T == 0:
        return
    _need(y, T * w.cfg.d, "y")
    _need(o_blocks, world * moe_w8a8_ep_block_rows(w, block_tokens) * w.cfg.d, "o_blocks")
    _check(lib().moe_w8a8_ep_combine_blocked(
        w.handle, _dev_ptr(o_blocks, torch.float32, "o_blocks"), int(T), ptr, int(world), int(block_tokens),
        _dev_ptr(y, _act_dtype(w.cfg.out_dtype), "y"), _dev_ptr(workspace, name="workspace"), _nbytes(workspace),
        _stream(stream)), "moe_w8a8_ep_combine_blocked")


# ------------------------------------------------------------------ measurement aid

def moe_w8a8_tensor_peak_loop(expert_format: int, mma_per_sm: int, stream=None) -> float:
    """Enqueue the tensor-core rate loop; returns its operation count (the
    caller times the launch)."""
    ops = ctypes.c_double(0.0)
    _check(lib().moe_w8a8_tensor_peak_loop(int(expert_format), int(mma_per_sm), ctypes.byref(ops),
                                           _stream(stream)), "moe_w8a8_tensor_peak_loop")
    return float(ops.value)
