"""The failure path of the fused expert launch, made to happen on purpose
without faulting or hanging the GPU: a testing switch on the handle makes the
launch withhold the release of one expert's h codes, so the down-projection
tiles that need them wait until the handle's wait budget (10 ms here) runs
out.  The launch must then end by itself, report MOE_ERR_TIMEOUT with the
place it gave up, and leave the GPU usable: the next forward on the same
handle matches the oracle bit for bit.  ("One night of MoE inference
optimisation", s6.4: a watchdog that turns a stuck step into an error.)"""
import dataclasses
import time

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


def _forward_raw(M, W, wl, data):
    """Enqueue one forward and wait for it, without reading the status."""
    import torch
    T = wl.T
    x = H.x_tensor(wl, data)
    y = torch.empty((T, wl.d), dtype=torch.bfloat16 if wl.in_bf16 else torch.float32, device="cuda")
    ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device="cuda")
    logits = H.to_dev(data.router_logits) if data.router_logits is not None else None
    M.moe_w8a8_forward(W, x, T, None, logits, y, ws)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T", [64, 32], ids=["128-row plan", "swapped-operand plan"])
def test_withheld_release_times_out_and_the_gpu_stays_usable(M, T):
    # 64 tokens x top-2 = 128 rows: the fused launch with 128-row MMAs; 32 tokens: its
    # swapped-operand plan (at most 32 rows per expert)
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], T=T)
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    W = H.gpu_prepare(wl, wts, w_router=data.w_router)
    prep = H.oracle_prepare(wl, wts)
    rt = H.oracle_route(wl, data)
    assert len(np.unique(rt.idx)) == wl.E    # one m-tile per expert, tiles 0..7
    M.moe_w8a8_set_path(W, M.MOE_PATH_TENSOR)
    M.moe_w8a8_set_wait_budget(W, 10_000_000)
    M.moe_w8a8_test_withhold_release(W, 3)
    t0 = time.time()
    _forward_raw(M, W, wl, data)
    seconds = time.time() - t0
    words = M.moe_w8a8_status_words(W, 5)
    assert words[0] == M.MOE_ERR_TIMEOUT
    # a down-projection producer (site 6) or epilogue (site 16), waiting for m-tile 3
    assert words[1] in (6, 16) and words[4] == 3, words
    assert 0 <= words[2] < 1024
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_check_status(W)
    assert e.value.status == M.MOE_ERR_TIMEOUT
    assert seconds < 5.0
    M.moe_w8a8_check_status(W)               # the check cleared the words

    # the switch off again: the same handle, the same GPU, a correct result
    M.moe_w8a8_test_withhold_release(W, -1)
    M.moe_w8a8_set_wait_budget(W, 2_000_000_000)
    y, dbg = H.gpu_forward(W, wl, data)
    y_ref, odbg = oracle.moe_tokens(data.x, prep, rt, out_bf16=wl.in_bf16)
    H.compare_stages(wl, rt, dbg, y, y_ref, odbg, np.arange(wl.T))
    assert np.array_equal(y, y_ref)


def test_withhold_switch_is_ignored_by_the_other_launches(M):
    """The streaming path has no cross-block waits: the switch changes nothing."""
    wl = synth.WORKLOADS["tiny"]
    wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    W = H.gpu_prepare(wl, wts, w_router=data.w_router)
    M.moe_w8a8_test_withhold_release(W, 0)
    M.moe_w8a8_set_wait_budget(W, 10_000_000)
    y, _ = H.gpu_forward(W, wl, data, path=M.MOE_PATH_STREAM, debug=False)
    prep = H.oracle_prepare(wl, wts)
    y_ref, _ = oracle.moe_tokens(data.x, prep, H.oracle_route(wl, data), out_bf16=wl.in_bf16)
    assert np.array_equal(y, y_ref)


def test_wait_budget_bounds(M):
    wl = synth.WORKLOADS["tiny"]
    W = H.gpu_prepare(wl, synth.make_weights(wl))
    for bad in (0, 999_999, 61_000_000_000):
        with pytest.raises(M.MoeError) as e:
            M.moe_w8a8_set_wait_budget(W, bad)
        assert e.value.status == M.MOE_ERR_INVALID_ARG
    with pytest.raises(M.MoeError):
        M.moe_w8a8_test_withhold_release(W, -2)
