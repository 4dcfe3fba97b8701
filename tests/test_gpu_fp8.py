"""GPU parity of the FP8 (E4M3) expert path against the oracle.

Weights, token codes and scales are produced by single rounding steps and must
match bit for bit.  The tensor cores accumulate E4M3 products in fp32 in an
order of their own, so the accumulators are compared with the exact sum
(the oracle's) within an error bound, the h codes (which a last-bit difference
in h can move by one step) by agreement rate and step distance, and the
output: within the layer's tolerance of the down projection recomputed from
the GPU's own h codes, and within FP8_Y_TOL (normwise) of the oracle's y.

Bound used for an accumulator of K products p_j = a_j b_j:
    |acc_gpu - acc_exact| <= 2^-14 * sum_j |p_j|
i.e. a relative error of 2^-14 of the absolute sum.  fp32 accumulation with
round-to-nearest over the 128 MMA steps of K = 4096 stays below
(128 + 1) 2^-24 sum |p| ~ 2^-17 sum |p|; the bound leaves a factor 8 for
truncating adders.  A lost or duplicated k-block, a wrong scale or a swapped
operand moves an accumulator by orders of magnitude more.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

ACC_BOUND = 2.0 ** -14
# One E4M3 step of an h code is 1/16 to 1/8 of its value, so an h code that a
# last-bit difference moves changes y by up to that share of one term of the
# down projection; normwise, 1e-2 of max |y| covers a few such moves per row.
FP8_Y_TOL = 1e-2


@pytest.fixture(scope="module")
def M():
    from w8a8_quantized_moe_b200 import build
    build.build()
    import w8a8_quantized_moe_b200 as mod
    return mod


def _dec(q):
    return oracle.e4m3_decode(np.ascontiguousarray(q).view(np.uint8)).astype(np.float64)


def _check_acc(acc_gpu, a_codes, b_codes, what):
    """acc_gpu [n] vs the exact sums of a_codes [K] . b_codes [n][K]."""
    a = _dec(a_codes)
    b = _dec(b_codes)
    exact = b @ a
    absum = np.abs(b) @ np.abs(a)
    err = np.abs(acc_gpu.astype(np.float64) - exact)
    ok = err <= ACC_BOUND * absum + 1e-30
    assert ok.all(), f"{what}: {np.count_nonzero(~ok)} accumulators outside the bound"
    return float((err / np.maximum(absum, 1e-30)).max())


def _code_distance(a, b):
    """Steps between E4M3 codes of the same sign (codes are monotone in magnitude)."""
    a = np.asarray(a).view(np.uint8).astype(np.int32)
    b = np.asarray(b).view(np.uint8).astype(np.int32)
    same_sign = (a >> 7) == (b >> 7)
    mag = np.abs((a & 0x7f) - (b & 0x7f))
    zero_pair = ((a & 0x7f) == 0) & ((b & 0x7f) == 0)
    return np.where(same_sign | zero_pair, mag, (a & 0x7f) + (b & 0x7f))


def _bf16_round(v):
    b = np.ascontiguousarray(v, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _bf16_step(v):
    """Spacing of bf16 values at |v|, at the upper end of its binade (so that a
    value one step away in either direction is covered)."""
    a = np.abs(np.asarray(v, np.float64))
    m, e = np.frexp(a)
    e = np.where(a == 0.0, -125, np.maximum(e, -125))
    return np.ldexp(1.0, e - 7)


def compare_fp8(wl, prep, rt, dbg, y, y_ref, odbg, tokens, bias=None):
    """Routing and token codes exact; accumulators within ACC_BOUND of the
    exact sums of the GPU's own operands; h codes at most one step from the
    oracle's and rarely different; y equal (within the layer tolerance) to the
    down projection and combine recomputed from the GPU's h codes; and y within
    FP8_Y_TOL (normwise) of the oracle's end-to-end y."""
    T, k, f = rt.idx.shape[0], wl.k, wl.f
    ref_l = rt.logits if bias is None else (rt.logits + bias[None, :]).astype(np.float32)
    assert np.array_equal(dbg["logits"], ref_l)
    assert np.array_equal(dbg["topk_idx"], rt.idx)
    assert np.array_equal(dbg["topk_w"], rt.w)
    assert np.array_equal(dbg["offsets"], rt.offsets)
    assert np.array_equal(dbg["ts2row"].reshape(T, k), rt.ts2row)
    xq = dbg["xq"].view(np.uint8)
    assert np.array_equal(xq[tokens], odbg["xq"]), "E4M3 activation codes differ"
    assert np.array_equal(dbg["sx"][tokens], odbg["sx"]), "activation scales differ"
    worst = {"acc1": 0.0, "acc2": 0.0}
    n_h = n_hdiff = 0
    y_mid = np.zeros((len(tokens), wl.d), np.float32)
    # bf16 output: the per-slot rows are rounded to bf16 before the sum, and the
    # tensor cores' fp32 sums differ from the exact ones in the last bits, so a
    # row may round one bf16 step the other way; the bound is one step per
    # summed row plus one for the output
    steps = np.zeros((len(tokens), wl.d), np.float64)
    for i, t in enumerate(tokens):
        for s in range(k):
            row = rt.ts2row[t, s]
            if row < 0:
                continue
            e = rt.idx[t, s]
            acc1 = dbg["acc1"][row].view(np.float32)
            worst["acc1"] = max(worst["acc1"], _check_acc(acc1[:f], xq[t], prep.wq_gate[e], "gate"))
            worst["acc1"] = max(worst["acc1"], _check_acc(acc1[f:], xq[t], prep.wq_up[e], "up"))
            hq = dbg["hq"][row].view(np.uint8)
            dist = _code_distance(hq, odbg["hq"][i, s])
            assert dist.max() <= 1, "h codes more than one step apart"
            n_h += hq.size
            n_hdiff += int(np.count_nonzero(dist))
            sh = dbg["sh"][row]
            assert abs(float(sh) - float(odbg["sh"][i, s])) <= 1e-4 * float(odbg["sh"][i, s])
            acc2 = dbg["acc2"][row].view(np.float32)
            worst["acc2"] = max(worst["acc2"], _check_acc(acc2, hq, prep.wq_down[e], "down"))
            # the down epilogue and combine, from the GPU's own h codes and exact sums
            acc2_x = (_dec(prep.wq_down[e]) @ _dec(hq)).astype(np.float32)
            o = ((acc2_x * np.float32(sh)) * prep.sw_down[e]) * np.float32(rt.w[t, s])
            if wl.in_bf16:       # per-slot rows in the layer's output precision
                o = _bf16_round(o)
                steps[i] += _bf16_step(o)
            y_mid[i] = y_mid[i] + o
    if wl.in_bf16:
        y_mid = _bf16_round(y_mid)
        steps += _bf16_step(y_mid)
    assert n_hdiff <= max(2, n_h // 200), f"{n_hdiff} of {n_h} h codes differ"
    if wl.in_bf16:
        over = np.abs(y[tokens].astype(np.float64) - y_mid) - steps
        assert over.max() <= 0.0, f"y vs recomputed down projection: {over.max()} beyond the rounding bound"
    else:
        err_mid = H.max_rel_err(y[tokens], y_mid)
        assert err_mid <= H.TOL[wl.in_bf16], f"y vs recomputed down projection: {err_mid}"
    err = float(np.abs(y[tokens] - y_ref).max() / np.abs(y_ref).max())
    assert err <= FP8_Y_TOL, f"y vs oracle, normwise: {err}"
    return err, worst, n_hdiff, n_h


def run_fp8(M, wl, wts=None, data=None, W=None, prep=None, tokens=None):
    wts = synth.make_weights(wl) if wts is None else wts
    data = synth.make_data(wl) if data is None else data
    prep = H.oracle_prepare(wl, wts, fmt=1) if prep is None else prep
    if W is None:
        W = H.gpu_prepare(wl, wts, fmt=M.MOE_FMT_E4M3)
        H.compare_prepare(W, prep)
    rt = H.oracle_route(wl, data)
    y, dbg = H.gpu_forward(W, wl, data)
    T = data.x.shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    y_ref, odbg = oracle.moe_tokens_fp8(data.x, prep, rt, tokens=toks, out_bf16=wl.in_bf16)
    return compare_fp8(wl, prep, rt, dbg, y, y_ref, odbg, toks, bias=data.router_bias)


@pytest.mark.parametrize("T", [64, 1, 200, 300])
def test_fp8_tiny_layer(M, T):
    # T*k = 128, 2, 400 rows run the fused expert launch, 600 the separate ones
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=T, data_seed=400 + T)
    run_fp8(M, wl)


@pytest.fixture(scope="module")
def decode_fp8(M):
    wl = synth.WORKLOADS["decode"]
    wts = synth.make_weights(wl)
    prep = H.oracle_prepare(wl, wts, fmt=1)
    W = H.gpu_prepare(wl, wts, fmt=M.MOE_FMT_E4M3)
    return wl, wts, prep, W


def test_fp8_decode_prepare_bit_exact(M, decode_fp8):
    wl, wts, prep, W = decode_fp8
    H.compare_prepare(W, prep)


def test_fp8_decode_layer(M, decode_fp8):
    wl, wts, prep, W = decode_fp8
    err, worst, n_hdiff, n_h = run_fp8(M, wl, wts=wts, W=W, prep=prep)
    print(f"fp8 decode: y max rel err {err:.3e}; accumulator error / sum|p|: {worst}; "
          f"h codes differing: {n_hdiff} of {n_h}")


def test_fp8_refuses_the_streaming_path(M, decode_fp8):
    import torch
    wl, wts, prep, W = decode_fp8
    data = synth.make_data(wl)
    M.moe_w8a8_set_path(W, M.MOE_PATH_STREAM)
    try:
        x = H.x_tensor(wl, data)
        y = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(M.moe_w8a8_workspace_size(W, wl.T), dtype=torch.uint8, device="cuda")
        with pytest.raises(M.MoeError) as e:
            M.moe_w8a8_forward(W, x, wl.T, None, H.to_dev(data.router_logits), y, ws)
        assert e.value.status == M.MOE_ERR_UNSUPPORTED_SHAPE
    finally:
        M.moe_w8a8_set_path(W, M.MOE_PATH_AUTO)


def test_fp8_pair_gemms(M):
    """FP8 experts with the separate GEMM launches on SM pairs
    (tcgen05.mma.cta_group::2.kind::f8f6f4)."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1200, data_seed=610)   # also the large-batch quantiser
    wts = synth.make_weights(wl)
    W = H.gpu_prepare(wl, wts, fmt=M.MOE_FMT_E4M3)
    M.moe_w8a8_set_cta_pairs(W, 1)
    M.moe_w8a8_set_fused_threshold(W, 0)
    run_fp8(M, wl, wts=wts, W=W)
