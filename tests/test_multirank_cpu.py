"""Multi-GPU plumbing of bench.py on CPU: two gloo ranks (no GPU) exercise the
max-over-ranks timing, the barrier, the per-rank replica batches and the
reference arm's rank-0-only rule."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import json

    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(1.0 + 2.5 * rank, world)
        bench.barrier(world)
        wl = bench.replica_workload(synth.WORKLOADS["decode"], rank)

        class Args:
            workload = "decode"
        ref = bench.run_reference(Args(), world, rank) if rank else "rank0-skipped"
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
            json.dump({"slowest": slowest, "seed": wl.data_seed, "wseed": wl.weight_seed,
                       "ref": ref}, fh)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import json
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    assert r[0]["slowest"] == r[1]["slowest"] == 3.5          # max over ranks, seen by every rank
    assert r[0]["wseed"] == r[1]["wseed"]                     # same layer weights
    assert r[0]["seed"] != r[1]["seed"]                       # a different batch per replica
    assert r[1]["ref"] is None                                # only rank 0 runs the reference arm


def test_threaded_oracle_step_equals_the_serial_oracle():
    """The all-cores CPU baseline runs the unchanged oracle on token subsets in
    threads; its output must be the serial oracle's, bit for bit."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import oracle
    import synth
    wl = synth.WORKLOADS["tiny"]
    wts = synth.make_weights(wl)
    prep = oracle.prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
    data = synth.make_data(wl)
    rt = oracle.route(data.x, wl.k, wl.E, w_router=data.w_router, logits=data.router_logits,
                      bias=data.router_bias, capacity_factor=wl.capacity_factor)
    y_ref, _ = oracle.moe_tokens(data.x, prep, rt, out_bf16=wl.in_bf16, debug=False)
    for threads in (1, 3, 8):
        _, y = bench.oracle_step_threads(wl, prep, data, threads)
        assert np.array_equal(y, y_ref), threads
