"""The certified tensor-core router against the oracle.

Batches of at least 1024 bf16 tokens with computed router logits are routed by
approximate tensor-core logits that only pick candidate experts (every expert
within twice a stated error bound of the k-th approximate logit), whose logits
are then computed in the stated fp32 order.  Top-k, gate weights and the whole
layer must match the oracle, which computes every logit in that order, bit for
bit -- including exact ties between the k-th and the (k+1)-th expert, which
must still go to the lower index.
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


def _run(M, wl, w_router):
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    data.w_router = np.ascontiguousarray(w_router, dtype=np.float32)
    W = H.gpu_prepare(wl, wts, w_router=data.w_router)
    prep = H.oracle_prepare(wl, wts)
    rt = H.oracle_route(wl, data)
    y, dbg = H.gpu_forward(W, wl, data)
    y_ref, odbg = oracle.moe_tokens(data.x, prep, rt, out_bf16=wl.in_bf16)
    assert H.certified_router(wl, wl.T)
    H.compare_stages(wl, rt, dbg, y, y_ref, odbg, np.arange(wl.T), bias=data.router_bias)
    assert np.array_equal(y, y_ref)
    return rt, dbg


@pytest.mark.parametrize("E,k", [(8, 2), (64, 4)])
def test_certified_router_with_exact_ties(M, E, k):
    """Experts 5 and 7 (and, with 64 experts, 40) have the same router column
    as expert 3, so every token has exact ties among them."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1200, E=E, k=k, in_bf16=True, data_seed=500 + E)
    wr = synth.normal(wl.data_seed, synth.TID_W_ROUTER, (wl.d, E), std=wl.weight_std)
    dup = [5, 7] + ([40] if E > 40 else [])
    for e in dup:
        wr[:, e] = wr[:, 3]
    rt, dbg = _run(M, wl, wr)
    tie_group = [3] + dup
    picked = np.isin(rt.idx, tie_group)
    # whenever the group is cut by the top-k boundary, the lower indices win
    for t in range(wl.T):
        chosen = sorted(set(rt.idx[t]) & set(tie_group))
        if 0 < len(chosen) < len(tie_group):
            assert chosen == tie_group[:len(chosen)], (t, chosen)
    assert picked.any()


def test_certified_router_skewed_bias(M):
    """Zipf router bias (a log-prior added to every logit) and capacity drops."""
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=1500, E=64, k=4, in_bf16=True, zipf_s=1.1,
                             capacity_factor=1.25, data_seed=601)
    wr = synth.normal(wl.data_seed, synth.TID_W_ROUTER, (wl.d, wl.E), std=wl.weight_std)
    rt, _ = _run(M, wl, wr)
    assert (rt.ts2row < 0).sum() > 0
