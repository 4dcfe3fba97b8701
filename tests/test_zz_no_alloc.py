"""The forward variant for callers that cannot allocate device memory.

Some callers may not call cudaMalloc on their request path (a serving
process that plans all device memory at start-up, a plugin whose host
framework owns the allocator).  moe_w8a8_forward_noalloc takes only inputs
and outputs and uses the library's fixed device scratch array.  This test
calls it through the C ABI twice in a row and checks both outputs against the
workspace-taking moe_w8a8_forward on the same inputs, within the tolerance
the parity tests use (they are in fact identical), and checks that a token
count whose scratch does not fit is refused before anything runs.  It runs
last in the suite (file name) and also passes on its own in a fresh process.
"""
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


def _check_against_workspace_forward(M, W, wl, data, T):
    """moe_w8a8_forward_noalloc, twice in a row, against moe_w8a8_forward on
    the same inputs."""
    import torch
    x = H.x_tensor(wl, data)
    bias = H.to_dev(data.router_bias) if data.router_bias is not None else None
    logits = H.to_dev(data.router_logits) if data.router_logits is not None else None
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    assert M.moe_w8a8_workspace_size(W, T) <= M.MOE_NOALLOC_SCRATCH_BYTES

    y_ref = torch.empty((T, wl.d), dtype=odt, device="cuda")
    ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device="cuda")
    M.moe_w8a8_forward(W, x, T, bias, logits, y_ref, ws)
    ref = y_ref.float().cpu().numpy()

    for _ in range(2):   # two calls in a row share (and reuse) the same scratch
        y = torch.full((T, wl.d), float("nan"), dtype=odt, device="cuda")
        M.moe_w8a8_forward_noalloc(W, x, T, bias, logits, y)
        M.moe_w8a8_check_status(W)
        got = y.float().cpu().numpy()
        assert H.max_rel_err(got, ref) <= H.TOL[wl.in_bf16]
        assert np.array_equal(got, ref)


@pytest.fixture(scope="module")
def decode_handle(M):
    wl = synth.WORKLOADS["decode"]
    return wl, H.gpu_prepare(wl, synth.make_weights(wl))


@pytest.mark.parametrize("path", ["auto", "stream", "tensor"])
def test_noalloc_forward_matches_workspace_forward_tiny(M, path):
    """The tiny layer on each expert path: the streaming path's scratch
    layout (INT32 accumulators, token codes) and the tensor path's (sorted
    rows, h, fused-launch counters) both live in the shared array."""
    wl = synth.WORKLOADS["tiny"]
    W = H.gpu_prepare(wl, synth.make_weights(wl))
    M.moe_w8a8_set_path(W, {"auto": M.MOE_PATH_AUTO, "stream": M.MOE_PATH_STREAM,
                            "tensor": M.MOE_PATH_TENSOR}[path])
    _check_against_workspace_forward(M, W, wl, synth.make_data(wl), wl.T)


def test_noalloc_forward_matches_workspace_forward_decode(M, decode_handle):
    wl, W = decode_handle
    _check_against_workspace_forward(M, W, wl, synth.make_data(wl), wl.T)


def test_noalloc_largest_decode_batch_and_the_first_refused(M, decode_handle):
    """The decode layer's largest batch that fits the array (82 tokens, as the
    header states) runs and matches; one more token does not fit and is
    refused before anything runs."""
    import torch
    wl, W = decode_handle
    t_max = 1
    while M.moe_w8a8_workspace_size(W, t_max + 1) <= M.MOE_NOALLOC_SCRATCH_BYTES:
        t_max += 1
    assert t_max == 82, f"the header states 82 tokens for this layer; the array now fits {t_max}"
    _check_against_workspace_forward(M, W, wl, synth.make_data(wl, T=t_max), t_max)
    T = t_max + 1
    data = synth.make_data(wl, T=T)
    y = torch.zeros((T, wl.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_forward_noalloc(W, H.x_tensor(wl, data), T, None, H.to_dev(data.router_logits), y)
    assert e.value.status == M.MOE_ERR_WORKSPACE_TOO_SMALL


def test_noalloc_refuses_token_counts_beyond_the_scratch(M):
    import torch
    wl = synth.WORKLOADS["tiny"]
    W = H.gpu_prepare(wl, synth.make_weights(wl))
    M.moe_w8a8_set_path(W, M.MOE_PATH_STREAM)
    T = 1
    while M.moe_w8a8_workspace_size(W, T) <= M.MOE_NOALLOC_SCRATCH_BYTES:
        T *= 2
    x = torch.zeros((T, wl.d), dtype=torch.float32, device="cuda")
    y = torch.zeros((T, wl.d), dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_forward_noalloc(W, x, T, None, None, y)
    assert e.value.status == M.MOE_ERR_WORKSPACE_TOO_SMALL
