"""The large sparse layer (d=8192, 256 experts, top-8, f=2048, Zipf(1.1) router
bias, capacity factor 1.25 -> 160 rows per expert, overflow dropped in token
order) at full size, against the oracle on a sample of tokens.

Its fp32 weights are 51.5 GB, so they are generated and uploaded one expert at
a time; the oracle accumulates the smoothing statistic over the same stream
and quantises only the experts the sampled tokens use.  Every routing and
permutation entry is compared for all 4096 tokens."""
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


def _expert_weights(wl, e):
    per = wl.d * wl.f
    wg = synth.normal(wl.weight_seed, synth.TID_W_GATE, (wl.d, wl.f), std=wl.weight_std, start=e * per)
    wu = synth.normal(wl.weight_seed, synth.TID_W_UP, (wl.d, wl.f), std=wl.weight_std, start=e * per)
    wd = synth.normal(wl.weight_seed, synth.TID_W_DOWN, (wl.f, wl.d), std=wl.weight_std, start=e * per)
    return wg, wu, wd


def test_large_sparse_layer_sampled_tokens(M):
    import torch
    wl = synth.WORKLOADS["large"]
    E, d, f, k, T = wl.E, wl.d, wl.f, wl.k, wl.T
    dev = "cuda"
    g_dev = torch.empty((E, d, f), dtype=torch.float32, device=dev)
    u_dev = torch.empty((E, d, f), dtype=torch.float32, device=dev)
    d_dev = torch.empty((E, f, d), dtype=torch.float32, device=dev)
    aw = np.zeros(d, dtype=np.float32)
    for e in range(E):
        wg, wu, wd = _expert_weights(wl, e)
        oracle.gateup_input_absmax(wg[None], wu[None], aw)
        g_dev[e].copy_(torch.from_numpy(wg))
        u_dev[e].copy_(torch.from_numpy(wu))
        d_dev[e].copy_(torch.from_numpy(wd))
    calib, _ = synth.activations(wl.weight_seed + synth.CALIB_SEED_OFFSET, synth.CALIB_TOKENS, d,
                                 wl.outlier_channels(), wl.outlier_factor, True)
    ax = oracle.channel_absmax(calib)
    s, inv_s = oracle.smooth_scales(ax, aw, wl.alpha)

    cfg = M.make_config(d, f, E, k, wl.alpha, wl.capacity_factor, True, M.MOE_BF16, M.MOE_BF16)
    cal = torch.from_numpy(synth.f32_to_bf16_bits(calib).view(np.int16)).view(torch.bfloat16).to(dev)
    axd = torch.zeros(d, dtype=torch.float32, device=dev)
    M.moe_w8a8_calibrate_absmax(cal, axd)
    data = synth.make_data(wl)
    W = M.moe_w8a8_prepare(cfg, g_dev, u_dev, d_dev, H.to_dev(data.w_router), axd)
    del g_dev, u_dev, d_dev
    torch.cuda.empty_cache()
    assert np.array_equal(M.moe_w8a8_get_smooth_scales(W), s)

    # full routing on both sides; expert FFN on a spread sample of tokens
    rt = H.oracle_route(wl, data)
    y, dbg = H.gpu_forward(W, wl, data, fields=H.DBG_SMALL)
    assert np.diff(rt.offsets).max() == oracle.capacity(wl.capacity_factor, T, k, E) == 160
    assert (rt.ts2row < 0).sum() > 0           # the Zipf skew overflows the hot experts
    toks = np.array([0, 1, T // 2, T - 1], dtype=np.int64)
    used = sorted(set(rt.idx[toks].reshape(-1).tolist()))
    remap = {e: i for i, e in enumerate(used)}
    n = len(used)
    wq_gate = np.empty((n, f, d), np.int8)
    wq_up = np.empty((n, f, d), np.int8)
    wq_down = np.empty((n, d, f), np.int8)
    sw_gate = np.empty((n, f), np.float32)
    sw_up = np.empty((n, f), np.float32)
    sw_down = np.empty((n, d), np.float32)
    for e in used:
        i = remap[e]
        wg, wu, wd = _expert_weights(wl, e)
        wq_gate[i], sw_gate[i] = oracle.quantize_gateup_expert(wg, s)
        wq_up[i], sw_up[i] = oracle.quantize_gateup_expert(wu, s)
        wq_down[i], sw_down[i] = oracle.quantize_down_expert(wd)
    prep = oracle.Prepared(ax, aw, s, inv_s, wq_gate, wq_up, sw_gate, sw_up, wq_down, sw_down)
    idx_c = np.vectorize(lambda e: remap.get(int(e), 0))(rt.idx).astype(np.int32)
    rt_c = oracle.Routing(rt.logits, idx_c, rt.w, rt.cap, rt.offsets, rt.row2ts, rt.ts2row)
    y_ref, odbg = oracle.moe_tokens(data.x, prep, rt_c, tokens=toks, out_bf16=True)
    H.compare_stages(wl, rt, dbg, y, y_ref, odbg, toks, bias=data.router_bias)
    assert np.array_equal(y[toks], y_ref)
