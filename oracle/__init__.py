"""CPU oracle of the W8A8 MoE layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
library never calls it and shares no code with it.

This module is a ctypes wrapper around ``moe_oracle.c`` (plain single-threaded
C, ``-ffp-contract=off``) plus the bookkeeping that strings its steps together
in the order the layer runs them: prepare (smoothing + per-channel weight
quantisation), route (logits, top-k, gate softmax), permute (with capacity),
and the per-token expert FFN and combine.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

# -mfma only lets fmaf() compile to the fused instruction (it is exact either
# way); -ffp-contract=off forbids any fusion that is not written out.
CFLAGS = ["-O2", "-mfma", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _SO, _SRC, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        sig = {
            "oracle_expf": ([f32], f32),
            "oracle_expf_array": ([vp, i64, vp], None),
            "oracle_quantize_rows": ([vp, i64, i64, vp, vp], None),
            "oracle_channel_absmax": ([vp, i64, i32, vp], None),
            "oracle_gateup_input_absmax": ([vp, vp, i32, i32, i32, vp], None),
            "oracle_smooth_scales": ([vp, vp, i32, f32, vp, vp], None),
            "oracle_quantize_gateup_expert": ([vp, vp, i32, i32, vp, vp], None),
            "oracle_quantize_down_expert": ([vp, i32, i32, vp, vp], None),
            "oracle_router_logits": ([vp, vp, i64, i32, i32, vp], None),
            "oracle_topk_softmax": ([vp, vp, i64, i32, i32, i32, vp, vp], None),
            "oracle_capacity": ([f32, i64, i32, i32], i32),
            "oracle_permute": ([vp, i64, i32, i32, i32, vp, vp, vp], i32),
            "oracle_quantize_tokens": ([vp, vp, i64, i32, f32, vp, vp], None),
            "oracle_act_clip_percentile": ([vp, vp, i64, i32, ctypes.c_double], f32),
            "oracle_gemm_i8": ([vp, vp, i64, i64, i64, vp], None),
            "oracle_swiglu_requant": ([vp, vp, f32, vp, vp, i32, vp, vp, vp], None),
            "oracle_down_epilogue": ([vp, f32, vp, f32, i32, vp], None),
            "oracle_round_bf16": ([f32], f32),
            "oracle_moe_tokens": ([vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp,
                                   vp, vp, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp], None),
            "oracle_e4m3_round": ([f32], f32),
            "oracle_e4m3_encode": ([f32], ctypes.c_uint8),
            "oracle_e4m3_decode": ([ctypes.c_uint8], f32),
            "oracle_e4m3_encode_array": ([vp, i64, vp], None),
            "oracle_e4m3_decode_array": ([vp, i64, vp], None),
            "oracle_quantize_rows_fp8": ([vp, i64, i64, vp, vp], None),
            "oracle_quantize_gateup_expert_fp8": ([vp, vp, i32, i32, vp, vp], None),
            "oracle_quantize_down_expert_fp8": ([vp, i32, i32, vp, vp], None),
            "oracle_quantize_tokens_fp8": ([vp, vp, i64, i32, f32, vp, vp], None),
            "oracle_gemm_fp8": ([vp, vp, i64, i64, i64, vp], None),
            "oracle_swiglu_requant_fp8": ([vp, vp, f32, vp, vp, i32, vp, vp, vp], None),
            "oracle_moe_tokens_fp8": ([vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp,
                                       vp, vp, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp], None),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def P(a):
    """Pointer of a C-contiguous numpy array (None passes NULL)."""
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need a C-contiguous array"
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ single steps

def expf(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    y = np.empty_like(x)
    lib().oracle_expf_array(P(x), x.size, P(y))
    return y


def quantize_rows(v) -> tuple[np.ndarray, np.ndarray]:
    v = _c(v, np.float32)
    v2 = v.reshape(-1, v.shape[-1])
    q = np.empty(v2.shape, dtype=np.int8)
    s = np.empty(v2.shape[0], dtype=np.float32)
    lib().oracle_quantize_rows(P(v2), v2.shape[0], v2.shape[1], P(q), P(s))
    return q.reshape(v.shape), s.reshape(v.shape[:-1])


def channel_absmax(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape[1], dtype=np.float32)
    lib().oracle_channel_absmax(P(x), x.shape[0], x.shape[1], P(out))
    return out


def gateup_input_absmax(w_gate, w_up, aw=None) -> np.ndarray:
    w_gate, w_up = _c(w_gate, np.float32), _c(w_up, np.float32)
    E, d, f = w_gate.shape
    aw = np.zeros(d, dtype=np.float32) if aw is None else aw
    lib().oracle_gateup_input_absmax(P(w_gate), P(w_up), E, d, f, P(aw))
    return aw


def smooth_scales(ax, aw, alpha: float):
    ax, aw = _c(ax, np.float32), _c(aw, np.float32)
    s = np.empty_like(ax)
    inv = np.empty_like(ax)
    lib().oracle_smooth_scales(P(ax), P(aw), ax.size, alpha, P(s), P(inv))
    return s, inv


def quantize_gateup_expert(w, s):
    w = _c(w, np.float32)
    d, f = w.shape
    q = np.empty((f, d), dtype=np.int8)
    sw = np.empty(f, dtype=np.float32)
    lib().oracle_quantize_gateup_expert(P(w), P(_c(s, np.float32)), d, f, P(q), P(sw))
    return q, sw


def quantize_down_expert(w):
    w = _c(w, np.float32)
    f, d = w.shape
    q = np.empty((d, f), dtype=np.int8)
    sw = np.empty(d, dtype=np.float32)
    lib().oracle_quantize_down_expert(P(w), f, d, P(q), P(sw))
    return q, sw


def router_logits(x, w_router) -> np.ndarray:
    x, wr = _c(x, np.float32), _c(w_router, np.float32)
    T, d = x.shape
    E = wr.shape[1]
    out = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(P(x), P(wr), T, d, E, P(out))
    return out


def topk_softmax(logits, k: int, bias=None, renormalize: bool = True):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    lib().oracle_topk_softmax(P(logits), P(_c(bias, np.float32)), T, E, k, 1 if renormalize else 0,
                              P(idx), P(w))
    return idx, w


def capacity(cf: float, T: int, k: int, E: int) -> int:
    return int(lib().oracle_capacity(cf, T, k, E))


def permute(idx, E: int, cap: int = -1):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    row2ts = np.empty(max(T * k, 1), dtype=np.int32)
    ts2row = np.empty((T, k), dtype=np.int32)
    R = lib().oracle_permute(P(idx), T, k, E, cap, P(offsets), P(row2ts), P(ts2row))
    return offsets, row2ts[:R].copy(), ts2row


def quantize_tokens(x, inv_s, act_clip: float = 0.0):
    """Per-token INT8 codes of x' = x * inv_s; act_clip > 0 caps each token's
    range at act_clip (values beyond it saturate at +-127)."""
    x = _c(x, np.float32)
    T, d = x.shape
    q = np.empty((T, d), dtype=np.int8)
    sx = np.empty(T, dtype=np.float32)
    lib().oracle_quantize_tokens(P(x), P(_c(inv_s, np.float32)), T, d, float(act_clip), P(q), P(sx))
    return q, sx


def act_clip_percentile(x, inv_s, percent: float) -> float:
    """Nearest-rank percentile of |x * inv_s| over every element of x [rows][d]."""
    x = _c(x, np.float32)
    rows, d = x.shape
    return float(lib().oracle_act_clip_percentile(P(x), P(_c(inv_s, np.float32)), rows, d, float(percent)))


def gemm_i8(a, b) -> np.ndarray:
    a, b = _c(a, np.int8), _c(b, np.int8)
    M, K = a.shape
    N = b.shape[0]
    c = np.empty((M, N), dtype=np.int32)
    lib().oracle_gemm_i8(P(a), P(b), M, N, K, P(c))
    return c


def swiglu_requant(acc_g, acc_u, sx: float, sw_g, sw_u):
    acc_g, acc_u = _c(acc_g, np.int32), _c(acc_u, np.int32)
    f = acc_g.size
    h = np.empty(f, dtype=np.float32)
    hq = np.empty(f, dtype=np.int8)
    sh = np.empty(1, dtype=np.float32)
    lib().oracle_swiglu_requant(P(acc_g), P(acc_u), sx, P(_c(sw_g, np.float32)),
                                P(_c(sw_u, np.float32)), f, P(h), P(hq), P(sh))
    return h, hq, float(sh[0])


def down_epilogue(acc2, sh: float, sw_dn, w: float) -> np.ndarray:
    acc2 = _c(acc2, np.int32)
    o = np.empty(acc2.size, dtype=np.float32)
    lib().oracle_down_epilogue(P(acc2), sh, P(_c(sw_dn, np.float32)), w, acc2.size, P(o))
    return o


def round_bf16(v) -> np.ndarray:
    v = _c(np.atleast_1d(v), np.float32)
    return np.array([lib().oracle_round_bf16(float(a)) for a in v.ravel()],
                    dtype=np.float32).reshape(v.shape)


# ------------------------------------------------------------------ the whole layer

@dataclass
class Prepared:
    ax: np.ndarray        # [d] calibration absmax of X
    aw: np.ndarray        # [d] absmax of gate/up weight rows over all experts
    s: np.ndarray         # [d] smoothing scales
    inv_s: np.ndarray     # [d]
    wq_gate: np.ndarray   # [E][f][d] int8
    wq_up: np.ndarray     # [E][f][d] int8
    sw_gate: np.ndarray   # [E][f]
    sw_up: np.ndarray     # [E][f]
    wq_down: np.ndarray   # [E][d][f] int8
    sw_down: np.ndarray   # [E][d]


def prepare(w_gate, w_up, w_down, calib_x, alpha: float, smooth: bool = True) -> Prepared:
    """Weights [E][d][f] / [E][f][d] fp32 -> smoothed per-channel INT8 weights."""
    E, d, f = w_gate.shape
    ax = channel_absmax(calib_x)
    aw = gateup_input_absmax(w_gate, w_up)
    if smooth:
        s, inv_s = smooth_scales(ax, aw, alpha)
    else:
        s, inv_s = None, None
    wq_gate = np.empty((E, f, d), dtype=np.int8)
    wq_up = np.empty((E, f, d), dtype=np.int8)
    sw_gate = np.empty((E, f), dtype=np.float32)
    sw_up = np.empty((E, f), dtype=np.float32)
    wq_down = np.empty((E, d, f), dtype=np.int8)
    sw_down = np.empty((E, d), dtype=np.float32)
    for e in range(E):
        wq_gate[e], sw_gate[e] = quantize_gateup_expert(w_gate[e], s)
        wq_up[e], sw_up[e] = quantize_gateup_expert(w_up[e], s)
        wq_down[e], sw_down[e] = quantize_down_expert(w_down[e])
    if not smooth:
        s = np.ones(d, dtype=np.float32)
        inv_s = None
    return Prepared(ax, aw, s, inv_s, wq_gate, wq_up, sw_gate, sw_up, wq_down, sw_down)


@dataclass
class Routing:
    logits: np.ndarray    # [T][E] (before bias)
    idx: np.ndarray       # [T][k]
    w: np.ndarray         # [T][k]
    cap: int              # -1: none
    offsets: np.ndarray   # [E+1]
    row2ts: np.ndarray    # [R]
    ts2row: np.ndarray    # [T][k]


def route(x, k: int, E: int, w_router=None, logits=None, bias=None, renormalize=True,
          capacity_factor: float = 0.0) -> Routing:
    if logits is None:
        logits = router_logits(x, w_router)
    idx, w = topk_softmax(logits, k, bias, renormalize)
    T = idx.shape[0]
    cap = capacity(capacity_factor, T, k, E)
    offsets, row2ts, ts2row = permute(idx, E, cap)
    return Routing(logits, idx, w, cap, offsets, row2ts, ts2row)


def moe_tokens(x, prep: Prepared, rt: Routing, tokens=None, out_bf16=False, debug=True,
               act_clip: float = 0.0):
    """Expert FFN + combine for the listed tokens (all by default); act_clip > 0
    caps the per-token activation range (saturating clip)."""
    x = _c(x, np.float32)
    T, d = x.shape
    E, f, _ = prep.wq_gate.shape
    k = rt.idx.shape[1]
    tok = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = tok.size
    y = np.empty((n, d), dtype=np.float32)
    dbg = {}
    if debug:
        dbg = dict(xq=np.empty((n, d), np.int8), sx=np.empty(n, np.float32),
                   acc1=np.zeros((n, k, 2 * f), np.int32), hq=np.zeros((n, k, f), np.int8),
                   sh=np.zeros((n, k), np.float32), acc2=np.zeros((n, k, d), np.int32),
                   o=np.zeros((n, k, d), np.float32))
    g = dbg.get
    lib().oracle_moe_tokens(P(x), d, f, E, k, P(prep.wq_gate), P(prep.wq_up), P(prep.sw_gate),
                            P(prep.sw_up), P(prep.wq_down), P(prep.sw_down), P(prep.inv_s),
                            float(act_clip), P(rt.idx), P(rt.w), P(_c(rt.ts2row, np.int32)), P(tok), n,
                            1 if out_bf16 else 0, P(y), P(g("xq")), P(g("sx")), P(g("acc1")),
                            P(g("hq")), P(g("sh")), P(g("acc2")), P(g("o")))
    return y, dbg


# ------------------------------------------------------------------ FP8 (E4M3) experts

def e4m3_encode(v) -> np.ndarray:
    """E4M3 codes (uint8) of fp32 values: nearest, ties to even, saturating at 448."""
    v = _c(np.atleast_1d(v), np.float32)
    q = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(P(v), v.size, P(q))
    return q


def e4m3_decode(q) -> np.ndarray:
    q = _c(np.atleast_1d(q), np.uint8)
    v = np.empty(q.shape, dtype=np.float32)
    lib().oracle_e4m3_decode_array(P(q), q.size, P(v))
    return v


def quantize_rows_fp8(v) -> tuple[np.ndarray, np.ndarray]:
    v = _c(v, np.float32)
    v2 = v.reshape(-1, v.shape[-1])
    q = np.empty(v2.shape, dtype=np.uint8)
    s = np.empty(v2.shape[0], dtype=np.float32)
    lib().oracle_quantize_rows_fp8(P(v2), v2.shape[0], v2.shape[1], P(q), P(s))
    return q.reshape(v.shape), s.reshape(v.shape[:-1])


def quantize_tokens_fp8(x, inv_s, act_clip: float = 0.0):
    x = _c(x, np.float32)
    T, d = x.shape
    q = np.empty((T, d), dtype=np.uint8)
    sx = np.empty(T, dtype=np.float32)
    lib().oracle_quantize_tokens_fp8(P(x), P(_c(inv_s, np.float32)), T, d, float(act_clip), P(q), P(sx))
    return q, sx


def gemm_fp8(a, b) -> np.ndarray:
    a, b = _c(a, np.uint8), _c(b, np.uint8)
    M, K = a.shape
    N = b.shape[0]
    c = np.empty((M, N), dtype=np.float32)
    lib().oracle_gemm_fp8(P(a), P(b), M, N, K, P(c))
    return c


def swiglu_requant_fp8(acc_g, acc_u, sx: float, sw_g, sw_u):
    acc_g, acc_u = _c(acc_g, np.float32), _c(acc_u, np.float32)
    f = acc_g.size
    h = np.empty(f, dtype=np.float32)
    hq = np.empty(f, dtype=np.uint8)
    sh = np.empty(1, dtype=np.float32)
    lib().oracle_swiglu_requant_fp8(P(acc_g), P(acc_u), sx, P(_c(sw_g, np.float32)),
                                    P(_c(sw_u, np.float32)), f, P(h), P(hq), P(sh))
    return h, hq, float(sh[0])


def prepare_fp8(w_gate, w_up, w_down, calib_x, alpha: float, smooth: bool = True) -> Prepared:
    """As prepare(), with E4M3 weight codes (uint8) and amax/448 scales."""
    E, d, f = w_gate.shape
    ax = channel_absmax(calib_x)
    aw = gateup_input_absmax(w_gate, w_up)
    s, inv_s = smooth_scales(ax, aw, alpha) if smooth else (None, None)
    wq_gate = np.empty((E, f, d), dtype=np.uint8)
    wq_up = np.empty((E, f, d), dtype=np.uint8)
    sw_gate = np.empty((E, f), dtype=np.float32)
    sw_up = np.empty((E, f), dtype=np.float32)
    wq_down = np.empty((E, d, f), dtype=np.uint8)
    sw_down = np.empty((E, d), dtype=np.float32)
    L = lib()
    for e in range(E):
        for src, q, sw in ((w_gate[e], wq_gate[e], sw_gate[e]), (w_up[e], wq_up[e], sw_up[e])):
            src = _c(src, np.float32)
            L.oracle_quantize_gateup_expert_fp8(P(src), P(_c(s, np.float32)), d, f, P(q), P(sw))
        src = _c(w_down[e], np.float32)
        L.oracle_quantize_down_expert_fp8(P(src), f, d, P(wq_down[e]), P(sw_down[e]))
    if not smooth:
        s = np.ones(d, dtype=np.float32)
    return Prepared(ax, aw, s, inv_s, wq_gate, wq_up, sw_gate, sw_up, wq_down, sw_down)


def moe_tokens_fp8(x, prep: Prepared, rt: Routing, tokens=None, out_bf16=False, debug=True,
                   act_clip: float = 0.0):
    """Expert FFN + combine with E4M3 experts for the listed tokens (all by default)."""
    x = _c(x, np.float32)
    T, d = x.shape
    E, f, _ = prep.wq_gate.shape
    k = rt.idx.shape[1]
    tok = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = tok.size
    y = np.empty((n, d), dtype=np.float32)
    dbg = {}
    if debug:
        dbg = dict(xq=np.empty((n, d), np.uint8), sx=np.empty(n, np.float32),
                   acc1=np.zeros((n, k, 2 * f), np.float32), hq=np.zeros((n, k, f), np.uint8),
                   sh=np.zeros((n, k), np.float32), acc2=np.zeros((n, k, d), np.float32),
                   o=np.zeros((n, k, d), np.float32))
    g = dbg.get
    lib().oracle_moe_tokens_fp8(P(x), d, f, E, k, P(prep.wq_gate), P(prep.wq_up), P(prep.sw_gate),
                                P(prep.sw_up), P(prep.wq_down), P(prep.sw_down), P(prep.inv_s),
                                float(act_clip), P(rt.idx), P(rt.w), P(_c(rt.ts2row, np.int32)), P(tok), n,
                                1 if out_bf16 else 0, P(y), P(g("xq")), P(g("sx")), P(g("acc1")),
                                P(g("hq")), P(g("sh")), P(g("acc2")), P(g("o")))
    return y, dbg
