"""Expert parallelism on one GPU.

G ranks are emulated in one process: each "rank" has its own shard handle and
its own tokens, and the two All-to-All exchanges are done by the host with
tensor copies between the library calls (no kernel waits on another).  The
output of every rank must equal, bit for bit, the single-GPU forward of a
handle holding all experts on that rank's tokens: the INT8 expert arithmetic
is per row and exact, and the combine sums the same fp32 rows in slot order.
The last test runs the real driver (``ExpertParallelMoE``) on a one-rank NCCL
group.
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


def _torch():
    import torch
    return torch


_WEIGHTS = {}


def _weights(wl):
    """Host weights per workload, generated once for the module."""
    key = (wl.name, wl.weight_seed, wl.d, wl.E, wl.f)
    if key not in _WEIGHTS:
        _WEIGHTS[key] = synth.make_weights(wl)
    return _WEIGHTS[key]


class Layer:
    """A layer's device weights, its all-experts handle and G shard handles."""

    def __init__(self, M, wl, G, fmt=0, capacity_factor=None):
        from w8a8_quantized_moe_b200.ep import equal_expert_ranges
        torch = _torch()
        self.wl, self.G = wl, G
        self.wts = _weights(wl)
        cfg, wg, wu, wd, wr, ax = H.gpu_layer_tensors(wl, self.wts, capacity_factor, fmt=fmt)
        self.cfg = cfg
        self.full = M.moe_w8a8_prepare(cfg, wg, wu, wd, wr, ax)
        self.ranges = equal_expert_ranges(wl.E, G)
        # each rank's maximum, then the all-reduce (MAX) every rank would run
        aws = []
        for first, n in self.ranges:
            aw = torch.empty(wl.d, dtype=torch.float32, device="cuda")
            M.moe_w8a8_gateup_absmax(cfg, wg[first:first + n], wu[first:first + n], aw)
            aws.append(aw)
        aw = torch.stack(aws).amax(0).contiguous()
        self.shards = [M.moe_w8a8_prepare_shard(cfg, first, wg[first:first + n], wu[first:first + n],
                                                wd[first:first + n], wr, ax, aw)
                       for first, n in self.ranges]
        torch.cuda.synchronize()

    def rank_data(self, g, T, step=0):
        wl = dataclasses.replace(self.wl, T=T, data_seed=self.wl.data_seed + 101 * g + 7919 * step)
        return synth.make_data(wl)


def _inputs(wl, data):
    x = H.x_tensor(wl, data)
    logits = H.to_dev(data.router_logits) if data.router_logits is not None else None
    bias = H.to_dev(data.router_bias) if data.router_bias is not None else None
    return x, logits, bias


def run_emulated(M, L, datas, Ts):
    """One expert-parallel layer over G emulated ranks; returns (y per rank,
    rows received per rank)."""
    torch = _torch()
    wl, G = L.wl, L.G
    k, E, d = wl.k, wl.E, wl.d
    rb = M.moe_w8a8_ep_row_bytes(L.shards[0])
    assert rb == d + 16
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    sends, offs, wss = [], [], []
    for g in range(G):
        T = Ts[g]
        x, logits, bias = _inputs(wl, datas[g])
        send = torch.empty(max(T * k * rb, 16), dtype=torch.uint8, device="cuda")
        off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        ws = torch.empty(M.moe_w8a8_ep_dispatch_workspace_size(L.shards[g], T), dtype=torch.uint8, device="cuda")
        M.moe_w8a8_ep_dispatch(L.shards[g], x[:T], T, bias, logits[:T] if logits is not None else None,
                               send, off, ws)
        sends.append(send)
        offs.append(off)
        wss.append(ws)
    offs_h = [o.cpu().numpy() for o in offs]
    for g in range(G):
        assert offs_h[g][0] == 0 and np.all(np.diff(offs_h[g]) >= 0)
    # the dispatch exchange: destination h receives, source by source, the rows of its experts
    count = np.zeros((G, G), np.int64)   # [source][destination]
    recvs = []
    for h, (first, n) in enumerate(L.ranges):
        parts = []
        for g in range(G):
            a, b = int(offs_h[g][first]), int(offs_h[g][first + n])
            parts.append(sends[g][a * rb:b * rb])
            count[g, h] = b - a
        recvs.append(torch.cat(parts).contiguous())
    o_recv = []
    for h in range(G):
        R = int(count[:, h].sum())
        o = torch.full((max(R, 1), d), float("nan"), dtype=torch.float32, device="cuda")[:R]
        ws = torch.empty(M.moe_w8a8_ep_experts_workspace_size(L.shards[h], R), dtype=torch.uint8, device="cuda")
        M.moe_w8a8_ep_experts(L.shards[h], recvs[h], R, o, ws)
        o_recv.append(o)
    # the return exchange: every output row back to its source, in send order
    ys = []
    for g in range(G):
        parts = []
        for h in range(G):
            start = int(count[:g, h].sum())
            parts.append(o_recv[h][start:start + count[g, h]])
        o_back = torch.cat(parts).contiguous()
        assert o_back.shape[0] == offs_h[g][E]
        y = torch.empty((Ts[g], d), dtype=odt, device="cuda")
        M.moe_w8a8_ep_combine(L.shards[g], o_back, Ts[g], y, wss[g])
        ys.append(y)
    for s in L.shards:
        M.moe_w8a8_check_status(s)
    return ys, count.sum(axis=0)


def run_emulated_blocked(M, L, datas, Ts, B):
    """The fixed-block exchange over G emulated ranks: every block travels
    whole (the host copies blocks, it never reads a count); returns y per rank
    and the number of rows each rank's experts saw (from their debug offsets)."""
    torch = _torch()
    wl, G = L.wl, L.G
    k, E, d = wl.k, wl.E, wl.d
    rb = M.moe_w8a8_ep_row_bytes(L.shards[0])
    nb = M.moe_w8a8_ep_block_rows(L.shards[0], B)
    assert nb == B * k + 1
    rank_first = [first for first, _ in L.ranges] + [E]
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    blocks, wss = [], []
    for g in range(G):
        T = Ts[g]
        x, logits, bias = _inputs(wl, datas[g])
        send = torch.empty(B * k * rb, dtype=torch.uint8, device="cuda")
        off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        ws = torch.empty(M.moe_w8a8_ep_dispatch_workspace_size(L.shards[g], B), dtype=torch.uint8, device="cuda")
        M.moe_w8a8_ep_dispatch(L.shards[g], x[:T], T, bias, logits[:T] if logits is not None else None,
                               send, off, ws)
        blk = torch.full((G * nb * rb,), 0x5A, dtype=torch.uint8, device="cuda")   # junk in unused rows
        M.moe_w8a8_ep_pack(L.shards[g], send, off, rank_first, B, blk)
        blocks.append(blk.view(G, nb * rb))
        wss.append(ws)
    o_blocks, seen = [], []
    for h in range(G):
        recv = torch.cat([blocks[g][h] for g in range(G)]).contiguous()   # block h of every source
        o = torch.full((G * nb, d), float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(M.moe_w8a8_ep_experts_blocked_workspace_size(L.shards[h], G, B), dtype=torch.uint8,
                         device="cuda")
        offs = torch.empty(L.ranges[h][1] + 1, dtype=torch.int32, device="cuda")
        M.moe_w8a8_ep_experts_blocked(L.shards[h], recv, G, B, o, ws, {"offsets": offs})
        o_blocks.append(o.view(G, nb * d))
        seen.append(int(offs[-1].item()))
    ys = []
    for g in range(G):
        o_back = torch.cat([o_blocks[h][g] for h in range(G)]).contiguous()   # block g of every destination
        y = torch.empty((Ts[g], d), dtype=odt, device="cuda")
        M.moe_w8a8_ep_combine_blocked(L.shards[g], o_back, Ts[g], rank_first, B, y, wss[g])
        ys.append(y)
    for s in L.shards:
        M.moe_w8a8_check_status(s)
    return ys, np.array(seen)


def full_forward(M, L, data, T):
    torch = _torch()
    wl = L.wl
    x, logits, bias = _inputs(wl, data)
    odt = torch.bfloat16 if wl.in_bf16 else torch.float32
    y = torch.empty((T, wl.d), dtype=odt, device="cuda")
    ws = torch.empty(M.moe_w8a8_workspace_size(L.full, T), dtype=torch.uint8, device="cuda")
    M.moe_w8a8_forward(L.full, x[:T], T, bias, logits[:T] if logits is not None else None, y, ws)
    M.moe_w8a8_check_status(L.full)
    return y


def check_layer(M, L, Ts, steps=1, block_tokens=None):
    recv_rows = None
    for step in range(steps):
        datas = [L.rank_data(g, max(Ts[g], 1), step) for g in range(L.G)]
        if block_tokens is None:
            ys, recv_rows = run_emulated(M, L, datas, Ts)
        else:
            ys, recv_rows = run_emulated_blocked(M, L, datas, Ts, block_tokens)
        for g in range(L.G):
            if Ts[g] == 0:
                continue
            ref = full_forward(M, L, datas[g], Ts[g])
            assert _torch().equal(ys[g], ref), f"rank {g}: expert-parallel output differs from the forward"
    return recv_rows


def test_shards_quantise_like_the_whole_layer(M):
    L = Layer(M, synth.WORKLOADS["tiny"], 4)
    full = {k: v.cpu().numpy() for k, v in M.moe_w8a8_export_weights(L.full).items()}
    for (first, n), s in zip(L.ranges, L.shards):
        part = {k: v.cpu().numpy() for k, v in M.moe_w8a8_export_weights(s).items()}
        for name in ("wq_gate", "wq_up", "sw_gate", "sw_up", "wq_down", "sw_down"):
            assert np.array_equal(part[name], full[name][first:first + n]), name
        assert np.array_equal(part["inv_s"], full["inv_s"])
        assert np.array_equal(M.moe_w8a8_get_smooth_scales(s), M.moe_w8a8_get_smooth_scales(L.full))


@pytest.mark.parametrize("G", [2, 4])
def test_tiny_layer(M, G):
    L = Layer(M, synth.WORKLOADS["tiny"], G)
    rows = check_layer(M, L, [64] * G, steps=2)
    assert rows.sum() == 64 * 2 * G


def test_tiny_layer_against_the_oracle(M):
    # the same emulated layer, checked against the oracle directly
    wl = synth.WORKLOADS["tiny"]
    L = Layer(M, wl, 2)
    prep = H.oracle_prepare(wl, L.wts)
    datas = [L.rank_data(g, wl.T) for g in range(2)]
    ys, _ = run_emulated(M, L, datas, [wl.T, wl.T])
    for g in range(2):
        w_router = synth.normal(wl.data_seed, synth.TID_W_ROUTER, (wl.d, wl.E), std=wl.weight_std)
        rt = oracle.route(datas[g].x, wl.k, wl.E, w_router=w_router, logits=datas[g].router_logits,
                          bias=datas[g].router_bias)
        y_ref, _ = oracle.moe_tokens(datas[g].x, prep, rt, debug=False)
        err = H.max_rel_err(ys[g].float().cpu().numpy(), y_ref)
        assert err <= H.TOL[wl.in_bf16], err


def test_skewed_routing_with_capacity(M):
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], zipf_s=1.5, capacity_factor=1.0)
    L = Layer(M, wl, 4)
    rows = check_layer(M, L, [64, 64, 64, 64])
    assert rows.sum() < 4 * 64 * 2 and len(set(rows.tolist())) > 1


def test_few_rows_streaming_expert_path(M):
    # 8 tokens x top-4 per rank: the experts of each rank see at most 32 rows
    L = Layer(M, synth.WORKLOADS["decode"], 2)
    rows = check_layer(M, L, [4, 4])
    assert rows.max() <= 32


def test_decode_layer_four_ranks(M):
    L = Layer(M, synth.WORKLOADS["decode"], 4)
    check_layer(M, L, [32, 32, 32, 32], steps=2)


def test_rank_without_tokens_and_separate_expert_launches(M):
    # rank 1 sends nothing; rank 0's 512 tokens x top-4 give each rank's
    # experts about 1024 rows (above 512 rows: the separate GEMM launches)
    L = Layer(M, synth.WORKLOADS["decode"], 2)
    rows = check_layer(M, L, [512, 0])
    assert rows.sum() == 2048 and rows.min() > 800


@pytest.mark.parametrize("G", [2, 4])
def test_blocked_exchange_decode(M, G):
    # fixed blocks of 32 tokens (129 rows per peer), each rank's experts take
    # their row counts from the block headers on the device
    L = Layer(M, synth.WORKLOADS["decode"], G)
    rows = check_layer(M, L, [32] * G, steps=2, block_tokens=32)
    assert rows.sum() == 32 * 4 * G


def test_blocked_exchange_short_batches_skew_and_idle_rank(M):
    # batches at and below the block (T = 20, 7, 0, 32 under B = 32), Zipf
    # skew and capacity, on the tiny layer (fp32 in and out)
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], zipf_s=1.5, capacity_factor=1.0)
    L = Layer(M, wl, 4)
    check_layer(M, L, [20, 7, 0, 32], block_tokens=32)


def test_blocked_exchange_streaming_expert_path(M):
    # 1 token per rank: 2 x (4 + 1) rows per rank's experts, the streaming path
    L = Layer(M, synth.WORKLOADS["decode"], 2)
    check_layer(M, L, [1, 1], block_tokens=1)


def test_block_count_out_of_range_is_reported(M):
    torch = _torch()
    wl = synth.WORKLOADS["tiny"]
    L = Layer(M, wl, 2)
    B = 2
    nb = M.moe_w8a8_ep_block_rows(L.shards[0], B)
    rb = wl.d + 16
    blk = torch.zeros((2, nb, rb), dtype=torch.uint8)
    blk[1, 0, :4] = torch.from_numpy(np.array([nb], np.int32).view(np.uint8))   # one more than fits
    o = torch.empty((2 * nb, wl.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_w8a8_ep_experts_blocked_workspace_size(L.shards[0], 2, B), dtype=torch.uint8,
                     device="cuda")
    M.moe_w8a8_ep_experts_blocked(L.shards[0], blk.cuda().reshape(-1), 2, B, o, ws)
    words = M.moe_w8a8_status_words(L.shards[0], 4)
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_check_status(L.shards[0])
    assert e.value.status == M.MOE_ERR_INVALID_ARG
    assert words[1] == 15 and words[2] == 1 and words[3] == nb
    assert torch.count_nonzero(o).item() == 0     # every row left out: zeros
    with pytest.raises(M.MoeError):
        M.moe_w8a8_ep_pack(L.shards[0], torch.empty(64, dtype=torch.uint8, device="cuda"),
                           torch.zeros(wl.E + 1, dtype=torch.int32, device="cuda"), [0, 3, 2, wl.E], B,
                           torch.empty(3 * nb * rb, dtype=torch.uint8, device="cuda"))


def test_fp8_experts(M):
    wl = synth.WORKLOADS["decode"]
    L = Layer(M, wl, 2, fmt=M.MOE_FMT_E4M3)
    datas = [L.rank_data(g, 32) for g in range(2)]
    ys, _ = run_emulated(M, L, datas, [32, 32])
    for g in range(2):
        ref = full_forward(M, L, datas[g], 32).float()
        y = ys[g].float()
        err = float((y - ref).abs().max() / ref.abs().max())
        assert err <= 1e-2, err


def test_row_for_a_foreign_expert_is_reported(M):
    torch = _torch()
    wl = synth.WORKLOADS["tiny"]
    L = Layer(M, wl, 2)
    rb = wl.d + 16
    rows = torch.zeros((4, rb), dtype=torch.uint8)
    meta = np.array([[1.0, 0.5]] * 4, np.float32).view(np.uint8)
    ids = np.array([[0, 0], [1, 1], [6, 2], [3, 3]], np.int32).view(np.uint8)   # expert 6 is rank 1's
    rows[:, wl.d:wl.d + 8] = torch.from_numpy(meta)
    rows[:, wl.d + 8:] = torch.from_numpy(ids)
    recv = rows.cuda().reshape(-1)
    o = torch.empty((4, wl.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_w8a8_ep_experts_workspace_size(L.shards[0], 4), dtype=torch.uint8, device="cuda")
    M.moe_w8a8_ep_experts(L.shards[0], recv, 4, o, ws)
    words = M.moe_w8a8_status_words(L.shards[0], 4)
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_check_status(L.shards[0])
    assert e.value.status == M.MOE_ERR_INVALID_ARG
    assert words[1] == 14 and words[2] == 2 and words[3] == 6
    M.moe_w8a8_check_status(L.shards[0])   # cleared


def test_shard_handle_refuses_the_single_gpu_forward(M):
    torch = _torch()
    wl = synth.WORKLOADS["tiny"]
    L = Layer(M, wl, 2)
    data = L.rank_data(0, wl.T)
    x = H.x_tensor(wl, data)
    y = torch.empty((wl.T, wl.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_w8a8_workspace_size(L.full, wl.T), dtype=torch.uint8, device="cuda")
    with pytest.raises(M.MoeError) as e:
        M.moe_w8a8_forward(L.shards[0], x, wl.T, None, None, y, ws)
    assert e.value.status == M.MOE_ERR_INVALID_ARG


def test_driver_on_a_one_rank_nccl_group(M):
    import datetime
    import os
    import socket

    import torch.distributed as dist

    from w8a8_quantized_moe_b200.ep import ExpertParallelMoE, LibraryStages, prepare_expert_shard
    torch = _torch()
    wl = synth.WORKLOADS["decode"]
    cfg, wg, wu, wd, wr, ax = H.gpu_layer_tensors(wl, _weights(wl))
    full = M.moe_w8a8_prepare(cfg, wg, wu, wd, wr, ax)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        shard = prepare_expert_shard(cfg, 0, wg, wu, wd, wr, ax)
        layer = ExpertParallelMoE(LibraryStages(shard))
        for step in range(2):
            data = synth.make_data(dataclasses.replace(wl, data_seed=wl.data_seed + 11 * step))
            x, logits, bias = _inputs(wl, data)
            y = layer.forward(x, wl.T, bias, logits)
            ref = torch.empty_like(y)
            ws = torch.empty(M.moe_w8a8_workspace_size(full, wl.T), dtype=torch.uint8, device="cuda")
            M.moe_w8a8_forward(full, x, wl.T, bias, logits, ref, ws)
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
            assert layer.last_rows == (wl.T * wl.k, wl.T * wl.k)
        # the fixed-block exchange through the same group: no count reaches the host
        blocked = ExpertParallelMoE(LibraryStages(shard), block_tokens=wl.T)
        for step in range(2):
            data = synth.make_data(dataclasses.replace(wl, data_seed=wl.data_seed + 13 * step))
            x, logits, bias = _inputs(wl, data)
            y = blocked.forward(x, wl.T, bias, logits)
            ref = torch.empty_like(y)
            ws = torch.empty(M.moe_w8a8_workspace_size(full, wl.T), dtype=torch.uint8, device="cuda")
            M.moe_w8a8_forward(full, x, wl.T, bias, logits, ref, ws)
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
    finally:
        dist.destroy_process_group()
