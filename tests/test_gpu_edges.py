"""GPU parity at the edges: kernel variants and shapes the main parity cases do
not reach, each through the C ABI against the oracle on the same seeded
inputs, integer and fixed-order float stages bit for bit.

- the decode layer's shape with bf16 X and router logits computed by the layer
  (X W_router in the stated fp32 order) at the small and mid token counts of
  the token-count sweep, uniform and Zipf-skewed, alpha 0.5 and 0.7;
- bf16 X with E % 32 != 0 (E = 48 and E = 6), which take the other router
  kernels;
- more than 2048 (token, slot) pairs with given logits, with fp32 X, and with
  the softmax over all experts (the warp-per-token top-k and the two-kernel
  permutation);
- the gate softmax over all E experts (renormalize = 0) on both expert paths;
- tokens whose range is at the bottom of the fp32 range (the scale underflows
  to 0, is subnormal, or has an infinite reciprocal), on both expert paths and
  for fp32 and bf16 X;
- the degenerate shapes: one expert (a dense W8A8 SwiGLU FFN), k = E, and the
  smallest hidden and FFN sizes (d = f = 128).

"Day0 adaptation of ultra-large model inference", section 4: the top-k must
equal the reference's exactly, tie-break included; "MiniMax-M3 W8A8 on K100AI",
s3.2: per-token INT8 activations.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from w8a8_quantized_moe_b200 import build
    build.build()
    import w8a8_quantized_moe_b200 as mod
    return mod


def run(M, wl, W, prep, data, path=None, tokens=None, renormalize=True, fields=H.DBG_ALL):
    """Forward on the GPU and the oracle on the same data; every stage checked.
    Returns (routing, GPU debug buffers, GPU y)."""
    rt = H.oracle_route(wl, data, renormalize=renormalize)
    try:
        y, dbg = H.gpu_forward(W, wl, data, path=path, fields=fields)
    finally:
        M.moe_w8a8_set_path(W, M.MOE_PATH_AUTO)
    T = data.x.shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    y_ref, odbg = oracle.moe_tokens(data.x, prep, rt, tokens=toks, out_bf16=wl.in_bf16)
    H.compare_stages(wl, rt, dbg, y, y_ref, odbg, toks, bias=data.router_bias, renormalize=renormalize)
    assert np.array_equal(y[toks], y_ref)
    return rt, dbg, y


def layer(wl, renormalize=True):
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    W = H.gpu_prepare(wl, wts, renormalize=renormalize, w_router=data.w_router)
    prep = H.oracle_prepare(wl, wts)
    H.compare_prepare(W, prep)
    return wts, data, W, prep


def spread(T, n=24):
    return np.unique(np.linspace(0, T - 1, min(T, n)).astype(np.int64))


# ----------------------------------------------------------------- decode shape, computed bf16 logits

@pytest.fixture(scope="module")
def sweep_layer(M):
    """The decode layer's experts with the sweep's router (one W_g ~N(0, 0.02^2)
    for the whole sweep), prepared at each alpha on both sides."""
    base = synth.WORKLOADS["decode"]
    wts = synth.make_weights(base)
    w_router = synth.normal(base.weight_seed, synth.TID_W_ROUTER, (base.d, base.E), std=0.02)
    cache = {}

    def get(alpha):
        if alpha not in cache:
            wl = dataclasses.replace(base, alpha=alpha)
            cache[alpha] = (H.gpu_prepare(wl, wts, w_router=w_router), H.oracle_prepare(wl, wts))
        return cache[alpha]

    return w_router, get


SWEEP_POINTS = [(T, "unif", 0.5) for T in (1, 8, 32, 128, 512)] + [(32, "zipf", 0.7), (512, "zipf", 0.7)]


@pytest.mark.parametrize("T,skew,alpha", SWEEP_POINTS)
def test_sweep_points_with_computed_bf16_logits(M, sweep_layer, T, skew, alpha):
    """The token-count sweep's small and mid points on the decode layer's
    shape: bf16 X, logits computed by the layer (the wide bf16 router kernel,
    E = 64), the one-block routing front end, and the expert path AUTO picks
    (streaming up to 32 rows, the fused tcgen05 launch up to 512, separate
    launches above)."""
    w_router, get = sweep_layer
    wl = next(p for p in synth.sweep_workloads()
              if p.T == T and (p.zipf_s > 0) == (skew == "zipf") and p.alpha == alpha)
    W, prep = get(alpha)
    data = synth.make_data(wl)
    data.w_router = w_router
    run(M, wl, W, prep, data, tokens=spread(T), fields=H.DBG_SMALL + ("acc1", "acc2", "o"))


# ----------------------------------------------------------------- other router kernels

@pytest.mark.parametrize("E,k", [(48, 4), (6, 2)])
@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_bf16_router_with_expert_count_not_a_multiple_of_32(M, E, k, path):
    wl = synth.custom(f"bf16_E{E}", T=100, d=512, E=E, k=k, f=256, alpha=0.6, in_bf16=True,
                      weight_seed=50 + E, data_seed=60 + E, fixed_outliers=(3, 130, 257, 400),
                      outlier_factor=25.0)
    wts, data, W, prep = layer(wl)
    run(M, wl, W, prep, data, path=M.MOE_PATH_STREAM if path == "stream" else M.MOE_PATH_TENSOR)


def test_large_batch_with_given_logits_uses_warp_topk(M):
    """T k = 2200 > 2048 with given logits: warp-per-token top-k, then the
    histogram and scatter kernels (tensor path, separate launches)."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1100, data_seed=70, logits_uniform=True)
    wts, data, W, prep = layer(wl)
    rt, _, _ = run(M, wl, W, prep, data, tokens=spread(wl.T, 48))
    assert rt.offsets[-1] == wl.T * wl.k


def test_large_batch_fp32_x_computed_logits(M):
    """T k = 2400 with fp32 X and logits computed by the layer (fp32 router
    kernel), warp top-k and the two-kernel permutation."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1200, data_seed=71)
    wts, data, W, prep = layer(wl)
    run(M, wl, W, prep, data, tokens=spread(wl.T, 48))


def test_large_bf16_batch_with_full_softmax(M):
    """bf16 X with computed logits at T = 1100 would take the certified
    router, which needs the renormalised gate; with the softmax over all E the
    layer computes every logit in the stated order instead (T k = 4400)."""
    wl = synth.custom("bf16_full_softmax", T=1100, d=512, E=16, k=4, f=256, alpha=0.6, in_bf16=True,
                      weight_seed=72, data_seed=73, fixed_outliers=(1, 200, 333), outlier_factor=30.0)
    wts, data, W, prep = layer(wl, renormalize=False)
    rt, dbg, _ = run(M, wl, W, prep, data, tokens=spread(wl.T, 32), renormalize=False,
                     fields=H.DBG_SMALL)
    assert rt.w.sum(axis=1).max() < 1.0      # the k weights are part of a softmax over all 16


@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_gate_softmax_over_all_experts(M, path):
    """renormalize = 0: w = softmax over all E logits, taken at the k chosen
    experts (the one-block routing kernel), on both expert paths."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=48, data_seed=12, zipf_s=1.1)
    wts, data, W, prep = layer(wl, renormalize=False)
    rt, dbg, _ = run(M, wl, W, prep, data, renormalize=False,
                     path=M.MOE_PATH_STREAM if path == "stream" else M.MOE_PATH_TENSOR)
    s = rt.w.astype(np.float64).sum(axis=1)
    assert s.max() < 1.0 and s.min() > 0.0


# ----------------------------------------------------------------- bottom of the fp32 range

TINY_RANGES = (1.4e-45, 1e-44, 1e-40, 3e-39, 1e-37, 5e-37, 1e-36, 2e-35)


def _tiny_rows(wl, data, inv_s):
    """Scale rows 0.. of X so that the smoothed row's range max_j |x_j inv_s_j|
    is about each of TINY_RANGES (whatever it is exactly, both sides see the
    same inputs).  For bf16 layers the scaled values are rounded to bf16 and
    both the values and the bits are replaced."""
    for t, target in enumerate(TINY_RANGES):
        u = data.x[t].astype(np.float64)
        m = np.abs(u * inv_s.astype(np.float64)).max()
        row = (u * (target / m)).astype(np.float32)
        if wl.in_bf16:
            bits = synth.f32_to_bf16_bits(row)
            data.x_bits[t] = bits
            row = (bits.astype(np.uint32) << 16).view(np.float32)
        data.x[t] = row


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_tokens_at_the_bottom_of_the_fp32_range(M, bf16, path):
    """Token ranges from the smallest subnormal up: the scale amax/127
    underflows to 0 (codes 0), is subnormal with an infinite reciprocal (the
    quantiser forms the IEEE quotient), or is subnormal with a finite one.
    Codes, scales and everything after them match the oracle bit for bit."""
    wl = synth.custom("tiny_ranges", T=24, d=256, E=8, k=2, f=256, alpha=0.5, in_bf16=bf16,
                      weight_seed=80, data_seed=81)
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    prep = H.oracle_prepare(wl, wts)
    _tiny_rows(wl, data, prep.inv_s)
    W = H.gpu_prepare(wl, wts, w_router=data.w_router)
    H.compare_prepare(W, prep)
    rt, dbg, _ = run(M, wl, W, prep, data, path=M.MOE_PATH_STREAM if path == "stream" else M.MOE_PATH_TENSOR)
    n = len(TINY_RANGES)
    sx, xq = dbg["sx"][:n], dbg["xq"][:n].astype(np.int32)
    zero = sx == 0.0
    assert zero[:2].all() and not xq[zero].any()              # amax/127 underflows: codes 0
    assert np.abs(xq[~zero]).max(axis=1).min() >= 1
    assert np.any((sx > 0) & (sx < np.float32(2.0 ** -126)))   # subnormal scales
    with np.errstate(over="ignore", divide="ignore"):
        assert np.any(np.isinf(np.float32(1.0) / sx[~zero]))    # reciprocal overflows
        assert np.any(np.isfinite(np.float32(1.0) / sx[(sx > 0) & (sx < np.float32(2.0 ** -126))]))


# ----------------------------------------------------------------- degenerate shapes

@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_one_expert_is_a_dense_ffn(M, path):
    """E = 1, k = 1: every token goes to the one expert with weight 1; the
    layer is a dense W8A8 SwiGLU FFN."""
    wl = synth.custom("dense", T=40, d=256, E=1, k=1, f=512, weight_seed=90, data_seed=91)
    wts, data, W, prep = layer(wl)
    rt, dbg, _ = run(M, wl, W, prep, data, path=M.MOE_PATH_STREAM if path == "stream" else M.MOE_PATH_TENSOR)
    assert not rt.idx.any() and np.all(rt.w == 1.0)
    assert rt.offsets.tolist() == [0, wl.T]


@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_every_token_picks_every_expert(M, path):
    """k = E: every token uses all experts, in descending logit order."""
    wl = synth.custom("k_eq_E", T=50, d=256, E=4, k=4, f=256, weight_seed=92, data_seed=93)
    wts, data, W, prep = layer(wl)
    rt, dbg, _ = run(M, wl, W, prep, data, path=M.MOE_PATH_STREAM if path == "stream" else M.MOE_PATH_TENSOR)
    assert np.all(np.sort(rt.idx, axis=1) == np.arange(4)[None, :])
    assert np.diff(rt.offsets).tolist() == [wl.T] * 4


def test_smallest_hidden_and_ffn_sizes(M):
    """d = f = 128, the smallest accepted sizes: the streaming path runs it
    (AUTO picks it: the tcgen05 tiles need d % 256 == 0); asking for the
    tensor path is refused as an unsupported shape."""
    wl = synth.custom("d128", T=30, d=128, E=8, k=2, f=128, weight_seed=94, data_seed=95,
                      fixed_outliers=(0, 64))
    wts, data, W, prep = layer(wl)
    run(M, wl, W, prep, data)
    run(M, wl, W, prep, data, path=M.MOE_PATH_STREAM)
    M.moe_w8a8_set_path(W, M.MOE_PATH_TENSOR)
    try:
        with pytest.raises(M.MoeError) as e:
            H.gpu_forward(W, wl, data, debug=False)
        assert e.value.status == M.MOE_ERR_UNSUPPORTED_SHAPE
    finally:
        M.moe_w8a8_set_path(W, M.MOE_PATH_AUTO)


# ----------------------------------------------------------------- the fused expert launch behind the large-batch front end

def test_fused_launch_behind_the_two_kernel_permutation(M):
    """T k = 2200 > 2048 (warp top-k, histogram and scatter kernels, the scatter
    clearing the fused launch's counters) with GEMM1, requantisation and GEMM2
    as one launch; twice in a row, so the second forward relies on the
    counters being cleared again."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1100, data_seed=74, logits_uniform=True)
    wts, data, W, prep = layer(wl)
    M.moe_w8a8_set_fused_threshold(W, 1 << 20)
    try:
        for _ in range(2):
            run(M, wl, W, prep, data, path=M.MOE_PATH_TENSOR, tokens=spread(wl.T, 48))
    finally:
        M.moe_w8a8_set_fused_threshold(W, 512)


def test_fused_launch_behind_the_certified_router(M, sweep_layer):
    """The decode layer's shape at T = 2048 with computed bf16 logits (the
    certified tensor-core router, then the two-kernel permutation) and the
    fused expert launch over its 8192 rows."""
    w_router, get = sweep_layer
    wl = next(p for p in synth.sweep_workloads() if p.T == 2048 and p.zipf_s == 0 and p.alpha == 0.5)
    W, prep = get(0.5)
    data = synth.make_data(wl)
    data.w_router = w_router
    M.moe_w8a8_set_fused_threshold(W, 1 << 20)
    try:
        run(M, wl, W, prep, data, tokens=spread(wl.T, 16), fields=H.DBG_SMALL + ("acc1", "acc2", "o"))
    finally:
        M.moe_w8a8_set_fused_threshold(W, 512)


# ----------------------------------------------------------------- GEMMs on SM pairs (cta_group::2)

@pytest.mark.parametrize("T", [1000, 300])
def test_pair_gemms_tiny_layer(M, T):
    """The separate GEMM launches on SM pairs (256-row tiles, one 256-row MMA
    per K slice over two SMs): T = 1000 gives about 250 rows per expert, so
    pair tiles end half empty, T = 300 fewer rows than one pair tile per
    expert.  Accumulators, codes and outputs bit for bit."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=T, data_seed=500 + T)
    wts, data, W, prep = layer(wl)
    M.moe_w8a8_set_cta_pairs(W, 1)
    M.moe_w8a8_set_fused_threshold(W, 0)
    run(M, wl, W, prep, data, path=M.MOE_PATH_TENSOR, tokens=spread(wl.T, 64))


def test_pair_gemms_decode_shape_certified_router(M, sweep_layer):
    """The decode layer's shape at T = 4096 (the certified router; 256 rows per
    expert on average) with the GEMMs on SM pairs."""
    w_router, get = sweep_layer
    base = next(p for p in synth.sweep_workloads() if p.T == 2048 and p.zipf_s == 0 and p.alpha == 0.5)
    wl = dataclasses.replace(base, T=4096, data_seed=77)
    W, prep = get(0.5)
    data = synth.make_data(wl)
    data.w_router = w_router
    M.moe_w8a8_set_cta_pairs(W, 1)
    try:
        run(M, wl, W, prep, data, tokens=spread(wl.T, 16), fields=H.DBG_SMALL + ("acc1", "acc2", "o"))
    finally:
        M.moe_w8a8_set_cta_pairs(W, 2)


def test_large_batch_quantiser_with_activation_clip(M):
    """From 1024 tokens on the tensor path the quantisation runs one warp per
    token on bulk-copied X rows; with a saturating clip at the 99.9th
    percentile of the calibration activations every stage still matches."""
    import torch
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1100, data_seed=75, logits_uniform=True)
    wts, data, W, prep = layer(wl)
    cal = H.to_dev(wts.calib_x)
    clip = M.moe_w8a8_calibrate_act_clip(W, cal, 99.9)
    assert clip == oracle.act_clip_percentile(wts.calib_x, prep.inv_s, 99.9)
    M.moe_w8a8_set_act_clip(W, clip)
    rt = H.oracle_route(wl, data)
    y, dbg = H.gpu_forward(W, wl, data, path=M.MOE_PATH_TENSOR)
    toks = spread(wl.T, 48)
    y_ref, odbg = oracle.moe_tokens(data.x, prep, rt, tokens=toks, out_bf16=wl.in_bf16, act_clip=clip)
    H.compare_stages(wl, rt, dbg, y, y_ref, odbg, toks)
    assert np.array_equal(y[toks], y_ref)
    assert (dbg["sx"] == np.float32(clip) / np.float32(127.0)).sum() > 0
    del torch
