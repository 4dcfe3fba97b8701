"""The per-stage event pairs (measurement aid) through the C ABI.

moe_w8a8_profile_start brackets every stage of the next forwards with a CUDA
event pair; moe_w8a8_profile_start_stages brackets only the stages of a mask.
The test checks that recording leaves the output unchanged (bit for bit
against a forward without events), that a masked run reads 0 for the stages
it left out and a positive time for the one it kept, that the number of
recorded forwards stops at max_forwards, and that an empty or out-of-range
mask is refused.
"""
import ctypes

import numpy as np
import pytest

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from w8a8_quantized_moe_b200 import build
    build.build()
    import w8a8_quantized_moe_b200 as mod
    return mod


@pytest.fixture(scope="module")
def tiny(M):
    wl = synth.WORKLOADS["tiny"]
    return wl, H.gpu_prepare(wl, synth.make_weights(wl)), synth.make_data(wl)


def _forward(M, W, wl, data, n):
    import torch
    T = wl.T
    x = H.x_tensor(wl, data)
    bias = H.to_dev(data.router_bias) if data.router_bias is not None else None
    logits = H.to_dev(data.router_logits) if data.router_logits is not None else None
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, wl.d), dtype=odt, device="cuda")
    for _ in range(n):
        M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
    M.moe_w8a8_check_status(W)
    return y.float().cpu().numpy()


def test_all_stages_and_masked_stage(M, tiny):
    wl, W, data = tiny
    ref = _forward(M, W, wl, data, 1)

    M.moe_w8a8_profile_start(W, 3)
    got = _forward(M, W, wl, data, 5)     # only the first 3 are recorded
    st = M.moe_w8a8_profile_read(W, 8)
    M.moe_w8a8_profile_stop(W)
    assert np.array_equal(got, ref)
    assert st.shape == (3, M.MOE_N_STAGES)
    assert np.all(st >= 0.0)
    gi = M.STAGE_NAMES.index("gemm1")
    assert np.all(st[:, gi] > 0.0)

    M.moe_w8a8_profile_start_stages(W, 4, [gi])
    got = _forward(M, W, wl, data, 4)
    st = M.moe_w8a8_profile_read(W, 4)
    M.moe_w8a8_profile_stop(W)
    assert np.array_equal(got, ref)
    assert st.shape == (4, M.MOE_N_STAGES)
    assert np.all(st[:, gi] > 0.0)
    others = [i for i in range(M.MOE_N_STAGES) if i != gi]
    assert np.all(st[:, others] == 0.0)


def test_bad_masks_are_refused(M, tiny):
    wl, W, data = tiny
    L = M.lib()
    assert L.moe_w8a8_profile_start_stages(W.handle, 4, 0) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_profile_start_stages(W.handle, 4, 1 << M.MOE_N_STAGES) == M.MOE_ERR_INVALID_ARG
    assert L.moe_w8a8_profile_start_stages(W.handle, 0, 1) == M.MOE_ERR_INVALID_ARG
    # nothing was started: a forward runs without events and reading reports no events
    _forward(M, W, wl, data, 1)
    out = np.zeros((1, M.MOE_N_STAGES), dtype=np.float32)
    assert L.moe_w8a8_profile_read(W.handle, ctypes.c_void_p(out.ctypes.data), 1) == -1
