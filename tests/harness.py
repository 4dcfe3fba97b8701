"""Parity harness: the same seeded inputs through the CUDA library (C ABI via
the Python binding) and through the CPU oracle, compared stage by stage.

Used by the GPU tests, by ``__graft_entry__.smoke()`` and by ``bench.py``'s
CPU-baseline leg.  Nothing here computes any step of the layer itself.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

TOL = {False: 1e-3, True: 1e-2}   # max relative error: fp32 output, bf16 output


def max_rel_err(y, r) -> float:
    """max_i |y_i - r_i| / max(|r_i|, 1e-3 rms(r))."""
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    if r.size == 0:
        return 0.0
    floor = 1e-3 * np.sqrt(np.mean(r * r))
    den = np.maximum(np.abs(r), max(floor, 1e-30))
    return float(np.max(np.abs(y - r) / den))


# ------------------------------------------------------------------ device side

def torch_mod():
    import torch
    return torch


def to_dev(a, dtype=None):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def x_tensor(wl: synth.Workload, data: synth.LayerData):
    torch = torch_mod()
    if wl.in_bf16:
        return torch.from_numpy(data.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    return to_dev(data.x)


def gpu_layer_tensors(wl: synth.Workload, wts: synth.LayerWeights, capacity_factor=None, renormalize=True,
                      fmt=0, w_router=None):
    """The config and the device inputs of prepare: (cfg, w_gate, w_up, w_down,
    w_router, act_absmax), the calibration absmax measured through the C ABI."""
    import w8a8_quantized_moe_b200 as M
    torch = torch_mod()
    cfg = M.make_config(wl.d, wl.f, wl.E, wl.k, wl.alpha,
                        wl.capacity_factor if capacity_factor is None else capacity_factor,
                        renormalize, M.MOE_BF16 if wl.in_bf16 else M.MOE_F32,
                        M.MOE_BF16 if wl.in_bf16 else M.MOE_F32, fmt)
    calib = synth.f32_to_bf16_bits(wts.calib_x) if wl.in_bf16 else wts.calib_x
    if wl.in_bf16:
        cal = torch.from_numpy(calib.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        cal = to_dev(calib)
    ax = torch.zeros(wl.d, dtype=torch.float32, device="cuda")
    M.moe_w8a8_calibrate_absmax(cal, ax)
    if w_router is None:
        w_router = synth.normal(wl.data_seed, synth.TID_W_ROUTER, (wl.d, wl.E), std=wl.weight_std)
    return cfg, to_dev(wts.w_gate), to_dev(wts.w_up), to_dev(wts.w_down), to_dev(w_router), ax


def gpu_prepare(wl: synth.Workload, wts: synth.LayerWeights, capacity_factor=None, renormalize=True,
                fmt=0, w_router=None):
    """Calibration absmax + prepare through the C ABI (fmt: MOE_FMT_INT8 / MOE_FMT_E4M3)."""
    import w8a8_quantized_moe_b200 as M
    torch = torch_mod()
    cfg, wg, wu, wd, wr, ax = gpu_layer_tensors(wl, wts, capacity_factor, renormalize, fmt, w_router)
    W = M.moe_w8a8_prepare(cfg, wg, wu, wd, wr, ax)
    torch.cuda.synchronize()
    return W


DBG_ALL = ("logits", "topk_idx", "topk_w", "offsets", "row2ts", "ts2row", "xq", "sx", "acc1", "hq",
           "sh", "acc2", "o")
DBG_SMALL = ("logits", "topk_idx", "topk_w", "offsets", "row2ts", "ts2row", "xq", "sx", "hq", "sh")


def gpu_forward(W, wl: synth.Workload, data: synth.LayerData, debug=True, path=None, T=None,
                fields=DBG_ALL):
    """Run forward; returns (y as fp32 numpy, dict of debug numpy arrays)."""
    import w8a8_quantized_moe_b200 as M
    torch = torch_mod()
    T = data.x.shape[0] if T is None else T
    if path is not None:
        M.moe_w8a8_set_path(W, path)
    x = x_tensor(wl, data)
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    y = torch.empty((T, wl.d), dtype=odt, device="cuda")
    ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device="cuda")
    bias = to_dev(data.router_bias) if data.router_bias is not None else None
    logits = to_dev(data.router_logits) if data.router_logits is not None else None
    dbg = None
    if debug:
        tk = T * wl.k
        dev = "cuda"
        dbg = dict(logits=torch.empty((T, wl.E), dtype=torch.float32, device=dev),
                   topk_idx=torch.empty((T, wl.k), dtype=torch.int32, device=dev),
                   topk_w=torch.empty((T, wl.k), dtype=torch.float32, device=dev),
                   offsets=torch.empty(wl.E + 1, dtype=torch.int32, device=dev),
                   row2ts=torch.empty(tk, dtype=torch.int32, device=dev),
                   ts2row=torch.empty(tk, dtype=torch.int32, device=dev),
                   xq=torch.empty((T, wl.d), dtype=torch.int8, device=dev),
                   sx=torch.empty(T, dtype=torch.float32, device=dev),
                   acc1=torch.zeros((tk, 2 * wl.f), dtype=torch.int32, device=dev),
                   hq=torch.empty((tk, wl.f), dtype=torch.int8, device=dev),
                   sh=torch.empty(tk, dtype=torch.float32, device=dev),
                   acc2=torch.zeros((tk, wl.d), dtype=torch.int32, device=dev),
                   o=torch.empty((tk, wl.d), dtype=odt, device=dev))   # per-slot rows: output precision
        dbg = {k: v for k, v in dbg.items() if k in fields}
    M.moe_w8a8_forward(W, x, T, bias, logits, y, ws, dbg)
    M.moe_w8a8_check_status(W)
    out = {}
    if dbg:
        out = {k: (v.float() if v.dtype == torch.bfloat16 else v).cpu().numpy() for k, v in dbg.items()}
    return y.float().cpu().numpy(), out


# ------------------------------------------------------------------ oracle side

def oracle_prepare(wl: synth.Workload, wts: synth.LayerWeights, fmt=0) -> oracle.Prepared:
    if fmt == 1:
        return oracle.prepare_fp8(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
    return oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)


def oracle_route(wl: synth.Workload, data: synth.LayerData, capacity_factor=None,
                 renormalize=True) -> oracle.Routing:
    cf = wl.capacity_factor if capacity_factor is None else capacity_factor
    return oracle.route(data.x, wl.k, wl.E, w_router=data.w_router, logits=data.router_logits,
                        bias=data.router_bias, renormalize=renormalize, capacity_factor=cf)


# ------------------------------------------------------------------ comparisons

def compare_prepare(W, prep: oracle.Prepared):
    import w8a8_quantized_moe_b200 as M
    g = {k: v.cpu().numpy() for k, v in M.moe_w8a8_export_weights(W).items()}
    if prep.wq_gate.dtype == np.uint8:           # E4M3 codes travel in the same byte buffers
        g = {k: (v.view(np.uint8) if v.dtype == np.int8 else v) for k, v in g.items()}
    s = M.moe_w8a8_get_smooth_scales(W)
    assert np.array_equal(s, prep.s), "smoothing scales differ"
    assert np.array_equal(g["inv_s"], prep.inv_s), "inverse smoothing scales differ"
    for name in ("sw_gate", "sw_up", "sw_down"):
        assert np.array_equal(g[name], getattr(prep, name)), f"{name} differs"
    for name in ("wq_gate", "wq_up", "wq_down"):
        a, b = g[name], getattr(prep, name)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{name}: {len(bad)} codes differ, first at {bad[0].tolist()}")


def certified_router(wl: synth.Workload, T: int, renormalize: bool = True) -> bool:
    """Whether the library routes this batch with the certified tensor-core
    router (computed bf16 logits, renormalised gate, at least 1024 tokens and
    more than 2048 (token, slot) pairs)."""
    return (renormalize and wl.in_bf16 and not wl.logits_uniform and T >= 1024 and T * wl.k > 2048
            and wl.d % 64 == 0)


def compare_logits(wl, rt: oracle.Routing, got, bias=None, renormalize=True):
    """Router logits (+ bias): bit-exact, or, where the certified router ran,
    bit-exact for every selected expert and within 1e-4 of the row's largest
    logit elsewhere (those entries only chose the candidates)."""
    T = rt.idx.shape[0]
    ref_l = rt.logits if bias is None else (rt.logits + bias[None, :]).astype(np.float32)
    if not certified_router(wl, T, renormalize):
        assert np.array_equal(got, ref_l), "router logits differ"
        return
    sel = np.take_along_axis(got, rt.idx, axis=1)
    assert np.array_equal(sel, np.take_along_axis(ref_l, rt.idx, axis=1)), "selected logits differ"
    scale = np.abs(ref_l).max(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref_l) <= 1e-4 * scale), "approximate logits out of range"


def compare_stages(wl, rt: oracle.Routing, dbg: dict, y_gpu, y_ref, odbg: dict, tokens,
                   bias=None, renormalize=True):
    """Bit-exact integer stages, exact float intermediates, tolerance on y."""
    T = rt.idx.shape[0]
    k = wl.k
    tokens = np.asarray(tokens, np.int64)
    compare_logits(wl, rt, dbg["logits"], bias, renormalize)
    assert np.array_equal(dbg["topk_idx"], rt.idx), "top-k indices differ"
    assert np.array_equal(dbg["topk_w"], rt.w), "gate weights differ"
    assert np.array_equal(dbg["offsets"], rt.offsets), "expert offsets differ"
    R = int(rt.offsets[-1])
    assert np.array_equal(dbg["row2ts"][:R], rt.row2ts), "permutation differs"
    assert np.array_equal(dbg["ts2row"].reshape(T, k), rt.ts2row), "inverse permutation differs"
    assert np.array_equal(dbg["xq"][tokens], odbg["xq"]), "INT8 activations differ"
    assert np.array_equal(dbg["sx"][tokens], odbg["sx"]), "activation scales differ"
    for i, t in enumerate(tokens):
        for s in range(k):
            row = rt.ts2row[t, s]
            if row < 0:
                continue
            if "acc1" in dbg and dbg["acc1"] is not None:
                assert np.array_equal(dbg["acc1"][row], odbg["acc1"][i, s]), f"acc1 differs at t={t} s={s}"
            assert np.array_equal(dbg["hq"][row], odbg["hq"][i, s]), f"h codes differ at t={t} s={s}"
            assert dbg["sh"][row] == odbg["sh"][i, s], f"h scale differs at t={t} s={s}"
            if "acc2" in dbg and dbg["acc2"] is not None:
                assert np.array_equal(dbg["acc2"][row], odbg["acc2"][i, s]), f"acc2 differs at t={t} s={s}"
            if "o" in dbg:
                assert np.array_equal(dbg["o"][row], odbg["o"][i, s]), f"expert output differs at t={t} s={s}"
    err = max_rel_err(y_gpu[tokens], y_ref)
    assert err <= TOL[wl.in_bf16], f"output max relative error {err}"
    return err

