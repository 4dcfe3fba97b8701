"""Expert-parallel exchange on CPU.

gloo ranks run ``ExpertParallelMoE`` (the same driver the GPU ranks run) with
stand-ins for the library's three compute steps written on the oracle: the
dispatch writes the routed, quantised rows in the library's row layout, the
expert step evaluates each received row with the oracle's GEMMs and
epilogues, and the combine sums slots in slot order.  Every rank's output
must equal the oracle's single-process layer on that rank's tokens bit for
bit, which holds only if every row reaches the rank holding its expert and
every output row comes back to the position it left from.
"""
import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleStages:
    """One rank's compute steps on the oracle (experts [first, first + n))."""

    def __init__(self, wl, prep, first, n):
        import torch
        self.wl, self.prep, self.first, self.n = wl, prep, first, n
        self.d, self.k, self.E = wl.d, wl.k, wl.E
        self.row_bytes = wl.d + 16
        self.device = torch.device("cpu")
        self.out_dtype = torch.float32
        self.ts2row = None
        self.seen_experts = set()

    def dispatch_workspace(self, T):
        return 16

    def experts_workspace(self, R):
        return 16

    def dispatch(self, data, T, bias, logits, send, offsets, ws):
        import torch

        import oracle
        d, k, E, rb = self.d, self.k, self.E, self.row_bytes
        if T == 0:
            offsets.zero_()
            self.ts2row = np.zeros((0, k), np.int32)
            return
        rt = oracle.route(data.x, k, E, w_router=data.w_router, logits=data.router_logits, bias=data.router_bias,
                          capacity_factor=self.wl.capacity_factor)
        xq, sx = oracle.quantize_tokens(data.x, self.prep.inv_s)
        R = int(rt.offsets[E])
        rows = np.zeros((T * k, rb), np.uint8)
        for r in range(R):
            ts = int(rt.row2ts[r])
            t, sl = divmod(ts, k)
            rows[r, :d] = xq[t].view(np.uint8)
            rows[r, d:d + 8] = np.array([sx[t], rt.w[t, sl]], np.float32).view(np.uint8)
            rows[r, d + 8:] = np.array([rt.idx[t, sl], ts], np.int32).view(np.uint8)
        send[:rows.size].copy_(torch.from_numpy(rows.reshape(-1)))
        offsets.copy_(torch.from_numpy(rt.offsets.astype(np.int32)))
        self.ts2row = rt.ts2row

    def _expert_row(self, row):
        import oracle
        d, p = self.d, self.prep
        codes = row[:d].view(np.int8)
        sx, w = row[d:d + 8].view(np.float32)
        e, _ts = row[d + 8:].view(np.int32)
        assert self.first <= e < self.first + self.n, f"row for expert {e} on the wrong rank"
        self.seen_experts.add(int(e))
        acc_g = oracle.gemm_i8(codes[None], p.wq_gate[e])[0]
        acc_u = oracle.gemm_i8(codes[None], p.wq_up[e])[0]
        _h, hq, sh = oracle.swiglu_requant(acc_g, acc_u, float(sx), p.sw_gate[e], p.sw_up[e])
        acc2 = oracle.gemm_i8(hq[None], p.wq_down[e])[0]
        o = oracle.down_epilogue(acc2, sh, p.sw_down[e], float(w))
        if self.wl.in_bf16:          # per-slot rows in the layer's output precision
            o = oracle.round_bf16(o)
        return o

    def experts(self, recv, R, o_rows, ws):
        import torch
        rows = recv.numpy().reshape(R, self.row_bytes)
        for r in range(R):
            o_rows[r] = torch.from_numpy(self._expert_row(rows[r]))

    # fixed-block exchange: the library's block layout (header row with the
    # count, then the rows; unused rows filled with junk that must be ignored)
    def block_rows(self, B):
        return B * self.k + 1

    def pack(self, send, offsets, rank_first, B, blocks):
        rb, nb = self.row_bytes, self.block_rows(B)
        src = send.numpy().reshape(-1, rb)
        off = offsets.numpy()
        out = blocks.numpy().reshape(len(rank_first) - 1, nb, rb)
        out[:] = 0xA5
        for g in range(len(rank_first) - 1):
            lo, hi = int(off[rank_first[g]]), int(off[rank_first[g + 1]])
            out[g, 0] = 0
            out[g, 0, :4] = np.array([hi - lo], np.int32).view(np.uint8)
            out[g, 1:1 + hi - lo] = src[lo:hi]
        self.offsets_host = off.copy()

    def experts_blocked_workspace(self, world, B):
        return 16

    def experts_blocked(self, blocks, world, B, o_blocks, ws):
        import torch
        nb = self.block_rows(B)
        b = blocks.numpy().reshape(world, nb, self.row_bytes)
        o = o_blocks.view(world, nb, self.d)
        o.zero_()
        for g in range(world):
            n = int(b[g, 0, :4].view(np.int32)[0])
            assert 0 <= n <= nb - 1
            for i in range(1, n + 1):
                o[g, i] = torch.from_numpy(self._expert_row(b[g, i]))
            self.blocked_recv = getattr(self, "blocked_recv", 0) + n

    def combine_blocked(self, o_back, T, rank_first, B, y, ws):
        import torch
        nb = self.block_rows(B)
        o = o_back.numpy().reshape(-1, self.d)
        off = self.offsets_host
        acc = np.zeros((T, self.d), np.float32)
        for sl in range(self.k):
            for t in range(T):
                r = int(self.ts2row[t, sl])
                if r < 0:
                    continue
                g = max(h for h in range(len(rank_first) - 1) if off[rank_first[h]] <= r)
                acc[t] = acc[t] + o[g * nb + 1 + r - int(off[rank_first[g]])]
        y.copy_(torch.from_numpy(acc))

    def combine(self, o_rows, T, y, ws):
        import torch
        o = o_rows.numpy()
        acc = np.zeros((T, self.d), np.float32)
        for sl in range(self.k):
            rows = self.ts2row[:, sl]
            m = rows >= 0
            acc[m] = acc[m] + o[rows[m]]
        y.copy_(torch.from_numpy(acc))


def _rank_main(rank, world, port, out_dir, case):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import json

    import torch.distributed as dist

    import oracle
    import synth
    from w8a8_quantized_moe_b200.ep import ExpertParallelMoE, equal_expert_ranges

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        wl = dataclasses.replace(synth.WORKLOADS["tiny"], **case.get("wl", {}))
        T = case.get("T", [wl.T] * world)[rank]
        wts = synth.make_weights(wl)
        prep = oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
        ranges = case.get("ranges") or equal_expert_ranges(wl.E, world)
        first, n = ranges[rank]
        stages = OracleStages(wl, prep, first, n)
        layer = ExpertParallelMoE(stages, ranges=ranges, block_tokens=case.get("block_tokens"))
        bad = []
        for r in ([(0, wl.E)], [(1, wl.E - 1)] + [(0, 1)] * (world - 1),
                  [(0, 2), (3, wl.E - 3)] + [(wl.E, 0)] * (world - 2)):
            try:
                ExpertParallelMoE(stages, ranges=r)
                bad.append(r)
            except ValueError:
                pass
        out = {"rows": None, "equal": True, "T": T, "accepted_bad_ranges": len(bad)}
        for step in range(2):   # two layers' worth of traffic through the same buffers
            wl_r = dataclasses.replace(wl, T=max(T, 1), data_seed=wl.data_seed + 37 * rank + 1000 * step)
            data = synth.make_data(wl_r)
            y = layer.forward(data, T).numpy()
            if T:
                rt = oracle.route(data.x, wl.k, wl.E, w_router=data.w_router, logits=data.router_logits,
                                  bias=data.router_bias, capacity_factor=wl.capacity_factor)
                y_ref, _ = oracle.moe_tokens(data.x, prep, rt, debug=False)
                out["equal"] &= bool(np.array_equal(y, y_ref))
            out["rows"] = list(layer.last_rows)
        out["seen"] = sorted(stages.seen_experts)
        out["blocked_recv"] = getattr(stages, "blocked_recv", 0)
        out["range"] = [first, n]
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
            json.dump(out, fh)
    finally:
        dist.destroy_process_group()


def _run(tmp_path, world, case):
    import json
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), case), nprocs=world,
                       start_method="spawn", join=True)
    return [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]


def test_ep_two_ranks_uniform(tmp_path):
    r = _run(tmp_path, 2, {})
    assert all(x["equal"] for x in r)
    sent = sum(x["rows"][0] for x in r)
    assert sent == sum(x["rows"][1] for x in r) == 2 * 64 * 2   # no capacity: every slot travels
    for x in r:
        first, n = x["range"]
        assert x["seen"] and all(first <= e < first + n for e in x["seen"])


def test_ep_four_ranks_skewed_with_capacity(tmp_path):
    # Zipf router bias piles tokens on a few experts; capacity 1.0 drops the
    # late arrivals on the sending rank, so ranks send and receive unequal counts
    r = _run(tmp_path, 4, {"wl": {"zipf_s": 1.5, "capacity_factor": 1.0}})
    assert all(x["equal"] for x in r)
    sent = [x["rows"][0] for x in r]
    recv = [x["rows"][1] for x in r]
    assert sum(sent) == sum(recv) < 4 * 64 * 2
    assert len(set(recv)) > 1


def test_ep_rank_without_tokens(tmp_path):
    # rank 1 routes no tokens this step but still serves its experts
    r = _run(tmp_path, 2, {"T": [64, 0]})
    assert r[0]["equal"] and r[1]["T"] == 0
    assert r[1]["rows"][0] == 0 and r[1]["rows"][1] > 0


def test_ep_eight_ranks_one_expert_each(tmp_path):
    # one expert per rank and a skewed router: many peer pairs exchange no rows
    r = _run(tmp_path, 8, {"wl": {"zipf_s": 2.0}, "T": [16] * 8})
    assert all(x["equal"] for x in r)
    assert sum(x["rows"][0] for x in r) == sum(x["rows"][1] for x in r) == 8 * 16 * 2
    assert min(x["rows"][1] for x in r) < 16 < max(x["rows"][1] for x in r)


def test_ep_uneven_expert_ranges(tmp_path):
    # 3 experts on rank 0, 5 on rank 1; malformed range lists are refused
    r = _run(tmp_path, 2, {"ranges": [(0, 3), (3, 5)]})
    assert all(x["equal"] for x in r)
    assert r[0]["range"] == [0, 3] and r[1]["range"] == [3, 5]
    assert all(x["accepted_bad_ranges"] == 0 for x in r)


def test_expert_ranges_host_checks():
    sys.path.insert(0, ROOT)
    from w8a8_quantized_moe_b200.ep import equal_expert_ranges
    assert equal_expert_ranges(64, 8) == [(8 * g, 8) for g in range(8)]
    with pytest.raises(ValueError):
        equal_expert_ranges(10, 4)


def _leave_main(rank, world, port, out_dir):
    """Rank 1 leaves between two layer steps (after its first step completes,
    with nothing in flight); rank 0 starts the next step, and its first
    exchange must end with an error within the process group's timeout
    instead of waiting for good."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import json
    import time

    import torch.distributed as dist

    import oracle
    import synth
    from w8a8_quantized_moe_b200.ep import ExpertParallelMoE, equal_expert_ranges

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    wl = synth.WORKLOADS["tiny"]
    wts = synth.make_weights(wl)
    prep = oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
    first, n = equal_expert_ranges(wl.E, world)[rank]
    layer = ExpertParallelMoE(OracleStages(wl, prep, first, n))
    out = {"first_step": False, "error": None, "seconds": None}
    data = synth.make_data(dataclasses.replace(wl, data_seed=wl.data_seed + 37 * rank))
    layer.forward(data, wl.T)
    out["first_step"] = True
    dist.barrier()
    if rank == 1:
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
            json.dump(out, fh)
        os._exit(0)          # leaves between steps: no collective of its own in flight
    time.sleep(0.5)
    t0 = time.time()
    try:
        layer.forward(data, wl.T)
    except Exception as exc:   # the exchange with the departed rank fails
        out["error"] = type(exc).__name__ + ": " + str(exc).splitlines()[0][:200]
    out["seconds"] = time.time() - t0
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
        json.dump(out, fh)
    os._exit(0)


def test_ep_rank_leaving_between_steps_is_an_error_not_a_hang(tmp_path):
    import json
    mp.start_processes(_leave_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn",
                       join=True)
    r0, r1 = (json.load(open(tmp_path / f"r{i}.json")) for i in range(2))
    assert r0["first_step"] and r1["first_step"]
    assert r0["error"] is not None
    assert r0["seconds"] < 30.0     # the group timeout is 5 s; the peer's closed socket may end it sooner


def test_ep_blocked_two_ranks(tmp_path):
    # fixed blocks of 64 tokens (129 rows per peer): no row count reaches the host
    r = _run(tmp_path, 2, {"block_tokens": 64})
    assert all(x["equal"] for x in r)
    assert sum(x["blocked_recv"] for x in r) == 2 * 2 * 64 * 2   # two steps, every slot travels once
    for x in r:
        first, n = x["range"]
        assert x["seen"] and all(first <= e < first + n for e in x["seen"])


def test_ep_blocked_skew_capacity_and_short_batches(tmp_path):
    # blocks larger than the batches (T = 40, 64, 17, 0 under B = 64), Zipf skew
    # and capacity: unequal counts per peer, empty blocks, an idle sender
    r = _run(tmp_path, 4, {"wl": {"zipf_s": 1.5, "capacity_factor": 1.0}, "T": [40, 64, 17, 0],
                           "block_tokens": 64})
    assert all(x["equal"] for x in r)
    assert r[3]["T"] == 0 and r[3]["blocked_recv"] > 0


def test_ep_blocked_eight_ranks_one_expert_each(tmp_path):
    r = _run(tmp_path, 8, {"wl": {"zipf_s": 2.0}, "T": [16] * 8, "block_tokens": 16})
    assert all(x["equal"] for x in r)
    assert sum(x["blocked_recv"] for x in r) == 2 * 8 * 16 * 2
