"""The C-ABI library without a GPU: it builds, loads, exports every entry
point the public header declares, and its host-side argument checks return
the documented statuses before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_w8a8.h")


@pytest.fixture(scope="module")
def M():
    from w8a8_quantized_moe_b200 import build
    build.build()
    import w8a8_quantized_moe_b200 as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports(M):
    assert declared_functions() == sorted(M.EXPORTS)


def declared_arg_counts():
    """Parameter count of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(moe_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(M):
    lib = M.lib()
    counts = declared_arg_counts()
    assert sorted(counts) == declared_functions()
    for name, n in counts.items():
        assert len(getattr(lib, name).argtypes) == n, name
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    kinds = {"size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32, "moe_status": ctypes.c_int32,
             "const char*": ctypes.c_char_p, "void": None}
    for m in re.finditer(r"^\s*([A-Za-z_][\w\s\*]*?)\s*\b(moe_\w+)\s*\(", text, flags=re.M):
        ret = " ".join(m.group(1).replace("*", " * ").split()).replace(" *", "*")
        assert ret in kinds, (m.group(2), ret)
        assert getattr(lib, m.group(2)).restype is kinds[ret], m.group(2)


def test_every_declared_symbol_is_exported(M):
    lib = M.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    nm = os.popen(f"nm -D --defined-only {M.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", nm), name


def test_status_strings(M):
    assert M.moe_status_string(M.MOE_OK) == "ok"
    assert M.moe_status_string(M.MOE_ERR_WORKSPACE_TOO_SMALL) == "workspace too small"
    assert M.moe_status_string(99) == "unknown status"


def test_host_side_argument_checks(M):
    L = M.lib()
    out = ctypes.c_void_p()
    cfg = M.make_config(4096, 1536, 64, 4)
    z = ctypes.c_void_p(16)   # never dereferenced: the checks fail first
    # null config / null output handle / bad enum / bad alpha / bad shapes
    assert L.moe_w8a8_prepare(None, z, z, z, z, z, None, ctypes.byref(out)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_prepare(ctypes.byref(cfg), z, z, z, z, z, None, None) == M.MOE_ERR_INVALID_ARG
    for field, value, status in [("alpha", -0.1, M.MOE_ERR_INVALID_ARG),
                                 ("alpha", 1.5, M.MOE_ERR_INVALID_ARG),
                                 ("in_dtype", 7, M.MOE_ERR_INVALID_ARG),
                                 ("renormalize", 2, M.MOE_ERR_INVALID_ARG),
                                 ("expert_format", 2, M.MOE_ERR_INVALID_ARG),
                                 ("expert_format", -1, M.MOE_ERR_INVALID_ARG),
                                 ("d", 4000, M.MOE_ERR_UNSUPPORTED_SHAPE),
                                 ("f", 100, M.MOE_ERR_UNSUPPORTED_SHAPE),
                                 ("n_experts", 300, M.MOE_ERR_UNSUPPORTED_SHAPE),
                                 ("top_k", 9, M.MOE_ERR_UNSUPPORTED_SHAPE),
                                 ("top_k", 0, M.MOE_ERR_UNSUPPORTED_SHAPE)]:
        c = M.make_config(4096, 1536, 64, 4)
        setattr(c, field, value)
        assert L.moe_w8a8_prepare(ctypes.byref(c), z, z, z, z, z, None, ctypes.byref(out)) == status, field
    c = M.make_config(256, 512, 4, 8)   # k > E
    assert L.moe_w8a8_prepare(ctypes.byref(c), z, z, z, z, z, None, ctypes.byref(out)) == \
        M.MOE_ERR_UNSUPPORTED_SHAPE
    # missing weight pointers
    assert L.moe_w8a8_prepare(ctypes.byref(cfg), None, z, z, z, z, None, ctypes.byref(out)) == \
        M.MOE_ERR_INVALID_ARG
    # handle-less calls
    assert L.moe_w8a8_workspace_size(None, 32) == 0
    assert L.moe_w8a8_forward(None, z, 32, None, None, z, z, 1 << 20, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_forward_host(None, z, 32, None, None, z, z, 1 << 20, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_set_path(None, 1) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_get_smooth_scales(None, z) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_check_status(None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_calibrate_absmax(z, 4, 16, 5, z, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_calibrate_absmax(z, -1, 16, 0, z, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_last_launch_count(None) == 0
    assert L.moe_w8a8_profile_start_stages(None, 4, 1 << M.STAGE_NAMES.index("gemm1")) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_set_act_clip(None, 1.0) == M.MOE_ERR_INVALID_ARG
    clip = ctypes.c_float(0.0)
    assert L.moe_w8a8_calibrate_act_clip(None, z, 4, 1, 99.9, ctypes.byref(clip), None) == M.MOE_ERR_INVALID_ARG
    L.moe_w8a8_destroy(None)


def test_expert_parallel_host_side_checks(M):
    L = M.lib()
    out = ctypes.c_void_p(123)
    cfg = M.make_config(4096, 1536, 64, 4)
    z = ctypes.c_void_p(16)   # never dereferenced: the checks fail first
    # shard range outside [0, E), empty shard, missing layer statistic
    for first, n in [(-1, 8), (60, 8), (0, 0), (0, 65)]:
        assert L.moe_w8a8_prepare_shard(ctypes.byref(cfg), first, n, z, z, z, z, z, z, None,
                                        ctypes.byref(out)) == M.MOE_ERR_INVALID_ARG, (first, n)
        assert out.value is None
    assert L.moe_w8a8_prepare_shard(ctypes.byref(cfg), 0, 8, z, z, z, z, z, None, None,
                                    ctypes.byref(out)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_prepare_shard(None, 0, 8, z, z, z, z, z, z, None, ctypes.byref(out)) == M.MOE_ERR_INVALID_ARG
    bad = M.make_config(4000, 1536, 64, 4)
    assert L.moe_w8a8_prepare_shard(ctypes.byref(bad), 0, 8, z, z, z, z, z, z, None,
                                    ctypes.byref(out)) == M.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_w8a8_gateup_absmax(ctypes.byref(cfg), 0, z, z, z, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_gateup_absmax(ctypes.byref(cfg), 65, z, z, z, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_gateup_absmax(ctypes.byref(cfg), 8, z, z, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_gateup_absmax(ctypes.byref(bad), 8, z, z, z, None) == M.MOE_ERR_UNSUPPORTED_SHAPE
    # handle-less calls
    assert L.moe_w8a8_ep_row_bytes(None) == 0
    assert L.moe_w8a8_ep_dispatch_workspace_size(None, 32) == 0
    assert L.moe_w8a8_ep_experts_workspace_size(None, 32) == 0
    assert L.moe_w8a8_ep_dispatch(None, z, 32, None, None, z, z, z, 1 << 20, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_ep_experts(None, z, 32, z, z, 1 << 20, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_ep_combine(None, z, 32, z, z, 1 << 20, None) == M.MOE_ERR_INVALID_ARG


def test_pointer_checks_come_before_the_handle(M):
    """Null and misaligned device pointers are refused with
    MOE_ERR_INVALID_ARG before the handle is looked at (so nothing is
    enqueued).  The handle here is a zeroed host buffer that is never read:
    the pointer checks fail first.  x, y, router_bias and router_logits are
    read with 16-byte vector accesses, so each must be 16-byte aligned."""
    L = M.lib()
    fake = ctypes.create_string_buffer(4096)
    h = ctypes.c_void_p(ctypes.addressof(fake))
    ok, odd = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    ws = ctypes.c_void_p(1 << 24)
    bad = M.MOE_ERR_INVALID_ARG
    fwd = L.moe_w8a8_forward
    assert fwd(h, odd, 32, None, None, ok, ws, 1 << 30, None, None) == bad           # x
    assert fwd(h, ok, 32, None, None, odd, ws, 1 << 30, None, None) == bad           # y
    assert fwd(h, ok, 32, odd, None, ok, ws, 1 << 30, None, None) == bad             # router_bias
    assert fwd(h, ok, 32, None, odd, ok, ws, 1 << 30, None, None) == bad             # router_logits
    assert fwd(h, ok, 32, None, None, ok, ctypes.c_void_p((1 << 24) + 16), 1 << 30, None, None) == bad
    assert fwd(h, None, 32, None, None, ok, ws, 1 << 30, None, None) == bad
    assert L.moe_w8a8_forward_noalloc(h, odd, 32, None, None, ok, None) == bad
    assert L.moe_w8a8_forward_noalloc(h, ok, 32, None, odd, ok, None) == bad
    assert L.moe_w8a8_ep_dispatch(h, odd, 32, None, None, ok, ok, ws, 1 << 30, None, None) == bad
    assert L.moe_w8a8_ep_dispatch(h, ok, 32, odd, None, ok, ok, ws, 1 << 30, None, None) == bad
    assert L.moe_w8a8_ep_experts(h, ok, 32, odd, ws, 1 << 30, None, None) == bad
    # the combine reads o_rows for every kept slot: NULL or misaligned is refused
    assert L.moe_w8a8_ep_combine(h, None, 32, ok, ws, 1 << 30, None) == bad
    assert L.moe_w8a8_ep_combine(h, odd, 32, ok, ws, 1 << 30, None) == bad
    assert L.moe_w8a8_ep_combine(h, ok, 32, odd, ws, 1 << 30, None) == bad


def test_capacity_factor_must_be_finite(M):
    L = M.lib()
    out = ctypes.c_void_p()
    z = ctypes.c_void_p(16)
    for cf in (float("inf"), float("-inf"), float("nan")):
        c = M.make_config(4096, 1536, 64, 4, capacity_factor=cf)
        assert L.moe_w8a8_prepare(ctypes.byref(c), z, z, z, z, z, None, ctypes.byref(out)) == \
            M.MOE_ERR_INVALID_ARG, cf


def test_binding_refuses_tensors_shorter_than_the_call(M):
    """The binding checks element counts before it hands pointers over, so a
    short tensor is an error, not an out-of-bounds device access."""
    import torch
    w = M.Weights(None, M.make_config(256, 512, 8, 2, in_dtype=M.MOE_F32, out_dtype=M.MOE_F32))
    T, d, E = 16, 256, 8
    x, y = torch.zeros(T * d), torch.zeros(T * d)
    ws = torch.zeros(16, dtype=torch.uint8)
    for args, name in [((torch.zeros(T * d - 1), T, None, None, y, ws), "x"),
                       ((x, T, None, None, torch.zeros(T * d - 4), ws), "y"),
                       ((x, T, None, torch.zeros(T * E - 1), y, ws), "router_logits"),
                       ((x, T, torch.zeros(E - 1), None, y, ws), "router_bias")]:
        with pytest.raises(ValueError, match=name):
            M.moe_w8a8_forward(w, *args)
    with pytest.raises(ValueError, match="x"):
        M.moe_w8a8_forward_noalloc(w, torch.zeros(5), T, None, None, y)
    import numpy as np
    with pytest.raises(ValueError, match="y_host"):
        M.moe_w8a8_forward_host(w, np.zeros(T * d, np.float32), T, None, None, np.zeros(3, np.float32), ws)


def test_product_path_does_not_touch_the_oracle():
    """The library sources and the binding never name the oracle."""
    pkg = os.path.join(ROOT, "w8a8_quantized_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in text.lower(), fn
