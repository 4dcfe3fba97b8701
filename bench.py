#!/usr/bin/env python
"""Benchmark of the B200 W8A8 MoE layer: tokens/s and roofline fraction.

One step = one forward of the whole layer (router/top-k, permute, smoothed
per-token quantisation, grouped expert GEMMs with their epilogues, combine)
over one batch of synthetic tokens already resident in HBM.  The prepared
INT8 weights are made once, untimed (the offline preparation step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|tiny|large]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm
    python bench.py --ep [--gpus N] ...    # the expert-parallel layer

Multi-GPU runs (torchrun, one process per GPU) are independent replicas of
the layer on different token batches; value = all ranks' tokens / the
slowest rank's device time.  With --ep the ranks instead split the experts
(E/N each), every rank routes its own batch, and rows cross between ranks
with one All-to-All each way per layer (on one GPU: a one-rank NCCL group).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W8A8 MoE layer tokens/s at T=32 and T=16384; % of HBM / INT8 TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0   # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernels, recorded from ncu captures into profiles/dram_traffic.md (--record-traffic) with a
# hash of the CUDA sources; a figure whose hash no longer matches the sources is not used.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.md")


def sources_hash() -> str:
    """First 16 hex digits of a SHA-256 over the library's CUDA sources and headers."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w8a8_quantized_moe_b200", "csrc")
    for fn in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")) +
                     glob.glob(os.path.join(csrc, "*.h"))):
        h.update(os.path.basename(fn).encode())
        with open(fn, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def norm_kernel(name: str) -> str:
    """A kernel's name as the traffic table keys it: no namespaces or parameters, and of
    its template arguments only the first ("tc_pair_gemm_kernel<0, 0>" -> "tc_pair_gemm_kernel<0>")."""
    import re
    name = re.sub(r"\(anonymous namespace\)::|<unnamed>::|unnamed>::", "", name).split("(")[0].strip()
    name = name.split()[-1].split("::")[-1] if "<" not in name else name.split("<")[0].split()[-1].split("::")[-1] + \
        "<" + name.split("<", 1)[1].split(",")[0].rstrip(">").strip() + ">"
    return name


def load_traffic() -> dict:
    """{(workload, T, kernel): bytes per launch} for the current sources."""
    out = {}
    if not os.path.exists(TRAFFIC_FILE):
        return out
    cur = sources_hash()
    for line in open(TRAFFIC_FILE):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) != 8 or not cells[1].isdigit():
            continue
        wl, T, kernel, launches, rd, wr, per_launch, sha = cells
        if sha == cur:
            out[(wl, int(T), kernel)] = float(per_launch)
    return out


def record_traffic(csv_path: str, workload: str, T: int, scale: float = 1.0):
    """Parse an ncu CSV (--metrics dram__bytes_read.sum,dram__bytes_write.sum --csv) and
    write the per-launch DRAM bytes of each kernel to profiles/dram_traffic.md (mean over
    its captured launches, times `scale` when a smaller case stands in for the workload),
    replacing the rows of this workload and T."""
    import csv
    import re
    unit = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    per = {}
    with open(csv_path) as fh:
        rows = [r for r in csv.reader(l for l in fh if l.startswith('"'))]
    hdr = rows[0]
    col = {n: hdr.index(n) for n in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    for r in rows[1:]:
        name = norm_kernel(r[col["Kernel Name"]])
        m = r[col["Metric Name"]]
        if m not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        v = float(r[col["Metric Value"]].replace(",", "")) * unit.get(r[col["Metric Unit"]], 1.0)
        d = per.setdefault(name, {}).setdefault(r[col["ID"]], {})
        d[m] = v
    keep = []
    if os.path.exists(TRAFFIC_FILE):
        for line in open(TRAFFIC_FILE):
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) == 8 and cells[1].isdigit() and (cells[0], int(cells[1])) == (workload, T):
                continue
            keep.append(line.rstrip("\n"))
    if not keep:
        keep = ["# DRAM traffic per launch of the dominant kernels (ncu)", "",
                "Written by `python bench.py --record-traffic <ncu csv> --workload <w> [--tokens T]` from",
                "`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none --csv` of the",
                "same bench command; bench.py uses a row only while the sources hash still matches.", "",
                "| workload | T | kernel | launches | read bytes | write bytes | bytes per launch | sources |",
                "|---|---|---|---|---|---|---|---|"]
    sha = sources_hash()
    for name, launches in sorted(per.items()):
        rd = sum(x.get("dram__bytes_read.sum", 0.0) for x in launches.values()) / len(launches)
        wr = sum(x.get("dram__bytes_write.sum", 0.0) for x in launches.values()) / len(launches)
        keep.append(f"| {workload} | {T} | {name} | {len(launches)} | {rd * scale:.0f} | {wr * scale:.0f} | "
                    f"{(rd + wr) * scale:.0f} | {sha} |")
    with open(TRAFFIC_FILE, "w") as fh:
        fh.write("\n".join(keep) + "\n")

FUSED_MAX_ROWS = 512   # the library's default: T*k up to which GEMM1 + requant + GEMM2 are one launch


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="decode", choices=sorted(synth.WORKLOADS))
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="CPU work budget of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-stage-events", action="store_true")
    p.add_argument("--path", choices=["auto", "stream", "tensor"], default="auto",
                   help="expert GEMM path: weight streaming, tcgen05 grouped GEMM, or automatic")
    p.add_argument("--sweep", action="store_true",
                   help="token-count x skew x alpha sweep on the decode layer's shape: one JSON line "
                        "per point and expert path (not the headline line)")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's token count T (same layer, same seeds)")
    p.add_argument("--format", choices=["int8", "e4m3"], default="int8",
                   help="expert number format: INT8 (the pages' W8A8) or FP8 E4M3")
    p.add_argument("--act-clip", type=float, default=0.0, metavar="PERCENT",
                   help="saturating activation clip at this percentile of the smoothed calibration "
                        "activations (0: off)")
    p.add_argument("--ep", action="store_true",
                   help="time the expert-parallel layer (experts split over the ranks) instead")
    p.add_argument("--no-prefill", action="store_true",
                   help="skip the extra prefill-layer measurement of the decode run")
    p.add_argument("--record-traffic", metavar="NCU_CSV", default="",
                   help="write the per-launch DRAM bytes of an ncu CSV (dram__bytes_read.sum, "
                        "dram__bytes_write.sum) for --workload / --tokens to profiles/dram_traffic.md and exit")
    p.add_argument("--traffic-scale", type=float, default=1.0,
                   help="with --record-traffic: factor from the captured case to the workload's launch")
    p.add_argument("--no-large", action="store_true",
                   help="skip the extra large-sparse-layer measurement of the decode run")
    p.add_argument("--fused-max-rows", type=int, default=-1,
                   help="rows (T*k) up to which the tensor path runs GEMM1 + requant + GEMM2 as one launch "
                        "(-1: the library's default)")
    p.add_argument("--cta-pairs", type=int, default=-1, choices=[-1, 0, 1, 2],
                   help="separate GEMM launches on SM pairs: 0 never, 1 always, 2 by rows per expert "
                        "(-1: the library's default)")
    p.add_argument("--no-tensor-peak", action="store_true",
                   help="skip the 8-bit tensor-core rate loop (the tensor-bound roofline then divides by "
                        "2 x the bf16 peak)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def describe(wl: synth.Workload) -> str:
    router = "uniform random router logits" if wl.logits_uniform else "router W_g ~N(0,0.02)"
    if wl.zipf_s:
        router += f" + Zipf({wl.zipf_s}) expert bias"
    cap = f", capacity factor {wl.capacity_factor}" if wl.capacity_factor > 0 else ""
    return (f"{wl.name}: T={wl.T} tokens, d={wl.d}, E={wl.E} experts, top-{wl.k}, SwiGLU f={wl.f}, "
            f"{'bf16' if wl.in_bf16 else 'fp32'} X with {wl.n_outliers} outlier channels x"
            f"{wl.outlier_factor:g}, INT8 per-channel weights ~N(0,0.02), alpha {wl.alpha}, "
            f"{router}{cap}, weight seed {wl.weight_seed}, data seed {wl.data_seed}")


# ------------------------------------------------------------------ clocks (NVML, read only)

class ClockSampler:
    """Samples SM clock and clock-event reasons during the timed region."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev: int):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_dev)
            try:
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report that, keep going
            self.nv = None
            self.err = str(exc)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ measured 8-bit tensor peak

NOMINAL_INT8_TOPS = 4500.0   # NVIDIA's dense INT8 / FP8 figure for B200 (context only)


def measure_tensor_peak(local: int, fmt: int) -> dict:
    """The dense 8-bit tensor-core rate of this GPU with the library's own
    tcgen05 MMA loop (operands resident in shared memory, one block per SM):
    a burst (~20 ms, the rate a kernel timed alone sees) and a sustained run
    (~0.5-1 s, under the power cap), each with the SM clocks sampled during
    it."""
    import torch

    import w8a8_quantized_moe_b200 as M
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    M.moe_w8a8_tensor_peak_loop(fmt, 1 << 14)
    torch.cuda.synchronize(dev)
    out = {}
    for name, n in (("burst", 1 << 18), ("sustained", 1 << 23)):
        clocks = ClockSampler(local)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.start()
        e0.record(stream)
        ops = M.moe_w8a8_tensor_peak_loop(fmt, n)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        clocks.stop()
        ms = e0.elapsed_time(e1)
        out[name] = {"tops": ops / (ms / 1e3) / 1e12, "ms": ms, "mma_per_sm": n, "clocks": clocks.summary()}
    out["kernel"] = "tc_peak_kernel (tcgen05.mma %s, M=128 N=256 K=32, operands in shared memory)" % (
        "kind::f8f6f4 E4M3" if fmt == 1 else "kind::i8")
    out["nominal_tops"] = NOMINAL_INT8_TOPS
    return out


# ------------------------------------------------------------------ byte / op model

def algorithmic(wl: synth.Workload, n_active: int, R: int, tensor: bool = False):
    """Per-step algorithmic bytes and INT8 ops.  Layer: active experts' INT8
    weights (3 d f bytes each) and their fp32 scales, X in, Y out, router input;
    intermediates excluded.  Per GEMM launch: the weights of the active experts
    plus that launch's own inputs and outputs (streaming path: A rows and the
    INT32 accumulators; tensor path: sorted A rows, fp32 h + partial maxima for
    GEMM1, h codes and the per-slot output rows (in the output dtype) for GEMM2;
    the fused launch: the sum of the two)."""
    in_b = 2 if wl.in_bf16 else 4
    w_bytes = n_active * 3 * wl.d * wl.f
    scales = n_active * (2 * wl.f + wl.d) * 4
    router = wl.T * wl.E * 4 if wl.logits_uniform else wl.d * wl.E * 4
    layer = w_bytes + scales + wl.T * wl.d * in_b * 2 + router
    if tensor:
        gemm1 = n_active * 2 * wl.f * wl.d + R * wl.d + R * wl.f * 4 + R * (wl.f // 64) * 4
    else:
        gemm1 = n_active * 2 * wl.f * wl.d + wl.T * wl.d + R * 2 * wl.f * 4
    gemm2 = n_active * wl.d * wl.f + R * wl.f + R * wl.d * in_b + n_active * wl.d * 4   # O rows: output dtype
    ops = 2 * R * 3 * wl.d * wl.f
    # the fused launch (GEMM1 + requantisation + GEMM2): both GEMMs' bytes
    return dict(layer_bytes=layer, gemm1_bytes=gemm1, gemm2_bytes=gemm2, fused_bytes=gemm1 + gemm2,
                int8_ops=ops)


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time (every rank gets it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_workload(base: synth.Workload, rank: int) -> synth.Workload:
    """Replicas: the same layer weights on every rank, a different token batch
    (data seed) per rank."""
    import dataclasses
    return dataclasses.replace(base, data_seed=base.data_seed + 1000 * rank) if rank else base


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ oracle timing

def oracle_step(wl, prep, data):
    """One oracle step on the tokens of `data`: routing of those tokens, the
    expert FFNs and the combine.  Returns the seconds it took."""
    import oracle
    t0 = time.perf_counter()
    rt = oracle.route(data.x, wl.k, wl.E, w_router=data.w_router, logits=data.router_logits,
                      bias=data.router_bias, capacity_factor=wl.capacity_factor)
    if prep.wq_gate.dtype == np.uint8:     # E4M3 experts
        oracle.moe_tokens_fp8(data.x, prep, rt, out_bf16=wl.in_bf16, debug=False)
    else:
        oracle.moe_tokens(data.x, prep, rt, out_bf16=wl.in_bf16, debug=False)
    return time.perf_counter() - t0


def oracle_step_threads(wl, prep, data, threads: int):
    """The same oracle step with the expert FFNs and combine of its tokens
    split over `threads` host threads (the oracle's C calls release the GIL;
    each thread runs the unchanged per-token code on its own tokens).  Returns
    (seconds, y)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    oracle.expf(np.zeros(1, np.float32))   # one-time constant set-up, before the threads
    fp8 = prep.wq_gate.dtype == np.uint8
    run = oracle.moe_tokens_fp8 if fp8 else oracle.moe_tokens
    T = data.x.shape[0]
    chunks = [c for c in np.array_split(np.arange(T, dtype=np.int64), threads) if c.size]
    t0 = time.perf_counter()
    rt = oracle.route(data.x, wl.k, wl.E, w_router=data.w_router, logits=data.router_logits,
                      bias=data.router_bias, capacity_factor=wl.capacity_factor)
    with ThreadPoolExecutor(len(chunks)) as ex:
        parts = list(ex.map(lambda tok: run(data.x, prep, rt, tokens=tok, out_bf16=wl.in_bf16, debug=False)[0],
                            chunks))
    secs = time.perf_counter() - t0
    return secs, np.concatenate(parts, axis=0)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample_size(wl, prep, budget_s: float, steps: int) -> int:
    """Tokens per oracle step so that `steps` steps take about budget_s."""
    probe = synth.make_data(wl, T=1)
    per_token = max(oracle_step(wl, prep, probe), 1e-4)
    return int(max(1, min(wl.T, budget_s / (steps * per_token))))


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores.
    Each step is a bounded sample (the first n tokens of the workload's
    batch, n sized so that warm-up + timed steps take about two minutes)."""
    if rank != 0:
        return
    import oracle
    wl = synth.WORKLOADS[args.workload]
    wts = synth.make_weights(wl)
    prepare = oracle.prepare_fp8 if args.format == "e4m3" else oracle.prepare
    prep = prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
    n_tok = oracle_sample_size(wl, prep, 120.0, args.steps + args.warmup)
    data = synth.make_data(wl, T=n_tok)
    for _ in range(args.warmup):
        oracle_step(wl, prep, data)
    secs = sum(oracle_step(wl, prep, data) for _ in range(args.steps))
    value = n_tok * args.steps / secs
    sample = (f"{args.steps} steps of the first {n_tok} of the {wl.T} tokens of the {wl.name} "
              f"workload (routing of the sampled tokens, expert FFNs, combine); preparation untimed")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.format == "e4m3" else "int8", "data": "synthetic",
            "config": {"workload": describe(wl), "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f,
                       "alpha": wl.alpha, "parallelism": "single CPU thread"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def measure(args, wl, world, rank, local, e2e_on=True, wts=None):
    """Prepare the layer (untimed), then time K forwards on resident inputs,
    with per-stage CUDA events, clock samples and an end-to-end leg."""
    import torch

    import w8a8_quantized_moe_b200 as M

    dev = torch.device("cuda", local)
    streamed = wts is None and 3 * wl.E * wl.d * wl.f * 4 > 8e9
    if wts is None and not streamed:
        wts = synth.make_weights(wl)
    data = synth.make_data(wl)
    fp8 = getattr(args, "format", "int8") == "e4m3"
    cfg = M.make_config(wl.d, wl.f, wl.E, wl.k, wl.alpha, wl.capacity_factor, True,
                        M.MOE_BF16 if wl.in_bf16 else M.MOE_F32,
                        M.MOE_BF16 if wl.in_bf16 else M.MOE_F32,
                        M.MOE_FMT_E4M3 if fp8 else M.MOE_FMT_INT8)
    act = torch.bfloat16 if wl.in_bf16 else torch.float32

    def to_act(v32):
        if wl.in_bf16:
            return torch.from_numpy(synth.f32_to_bf16_bits(v32).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(v32)

    if streamed:
        # fp32 weights too large for host memory: generate and upload one expert at a time
        per = wl.d * wl.f
        wg = torch.empty((wl.E, wl.d, wl.f), dtype=torch.float32, device=dev)
        wu = torch.empty((wl.E, wl.d, wl.f), dtype=torch.float32, device=dev)
        wd = torch.empty((wl.E, wl.f, wl.d), dtype=torch.float32, device=dev)
        for e in range(wl.E):
            for dst, tid, shape in ((wg, synth.TID_W_GATE, (wl.d, wl.f)), (wu, synth.TID_W_UP, (wl.d, wl.f)),
                                    (wd, synth.TID_W_DOWN, (wl.f, wl.d))):
                dst[e].copy_(torch.from_numpy(synth.normal(wl.weight_seed, tid, shape, std=wl.weight_std,
                                                           start=e * per)))
        calib_x, _ = synth.activations(wl.weight_seed + synth.CALIB_SEED_OFFSET, synth.CALIB_TOKENS, wl.d,
                                       wl.outlier_channels(), wl.outlier_factor, wl.in_bf16)
    else:
        calib_x = wts.calib_x
        wg, wu, wd = (torch.from_numpy(a).to(dev) for a in (wts.w_gate, wts.w_up, wts.w_down))
    cal = to_act(calib_x).to(dev)
    ax = torch.zeros(wl.d, dtype=torch.float32, device=dev)
    M.moe_w8a8_calibrate_absmax(cal, ax)
    wr = torch.from_numpy(data.w_router).to(dev)
    W = M.moe_w8a8_prepare(cfg, wg, wu, wd, wr, ax)
    M.moe_w8a8_set_path(W, {"auto": M.MOE_PATH_AUTO, "stream": M.MOE_PATH_STREAM,
                            "tensor": M.MOE_PATH_TENSOR}[args.path])
    if getattr(args, "fused_max_rows", -1) >= 0:
        M.moe_w8a8_set_fused_threshold(W, args.fused_max_rows)
    if getattr(args, "cta_pairs", -1) >= 0:
        M.moe_w8a8_set_cta_pairs(W, args.cta_pairs)
    clip = 0.0
    if getattr(args, "act_clip", 0.0) > 0.0:
        clip = M.moe_w8a8_calibrate_act_clip(W, cal, args.act_clip)
        M.moe_w8a8_set_act_clip(W, clip)
    del wg, wu, wd, cal
    torch.cuda.empty_cache()

    T = wl.T
    x = torch.from_numpy(data.x_bits.view(np.int16)).view(torch.bfloat16).to(dev) if wl.in_bf16 \
        else torch.from_numpy(data.x).to(dev)
    logits = torch.from_numpy(data.router_logits).to(dev) if data.router_logits is not None else None
    bias = torch.from_numpy(data.router_bias).to(dev) if data.router_bias is not None else None
    y = torch.empty((T, wl.d), dtype=act, device=dev)
    ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device=dev)

    # routing statistics of this batch (for the byte / op model): one debug forward
    offs = torch.empty(wl.E + 1, dtype=torch.int32, device=dev)
    M.moe_w8a8_forward(W, x, T, bias, logits, y, ws, {"offsets": offs})
    counts = np.diff(offs.cpu().numpy())
    n_active, R = int((counts > 0).sum()), int(counts.sum())
    tensor = args.path == "tensor" or (args.path == "auto" and (fp8 or T * wl.k > 32))
    fmax = args.fused_max_rows if getattr(args, "fused_max_rows", -1) >= 0 else FUSED_MAX_ROWS
    fused = tensor and T * wl.k <= fmax
    alg = algorithmic(wl, n_active, R, tensor)

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
    torch.cuda.synchronize(dev)

    K = args.steps
    # timed region: K forwards, nothing else on the stream
    clocks = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0.record(stream)
    for _ in range(K):
        M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(world)
    launches = M.moe_w8a8_last_launch_count(W) * K
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    M.moe_w8a8_check_status(W)

    # a second region of K forwards with a CUDA event pair around every stage
    # (the events add about 1.5 us per record, so the per-step time above is
    # taken without them); the roofline uses these per-launch stage times
    stages = None
    if not args.no_stage_events:
        M.moe_w8a8_profile_start(W, K)
        barrier(world)
        for _ in range(K):
            M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
        st = M.moe_w8a8_profile_read(W, K)
        M.moe_w8a8_profile_stop(W)
        barrier(world)
        stages = {M.STAGE_NAMES[i]: float(st[:, i].mean()) for i in range(M.MOE_N_STAGES)}
        # a third region of K forwards with an event pair around the dominant
        # expert stage only: the roofline's per-launch time, with no events at
        # the other stages' boundaries
        dom = max(("gemm1", "gemm2"), key=lambda k: stages[k])
        di = M.STAGE_NAMES.index(dom)
        M.moe_w8a8_profile_start_stages(W, K, [di])
        barrier(world)
        for _ in range(K):
            M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
        st = M.moe_w8a8_profile_read(W, K)
        M.moe_w8a8_profile_stop(W)
        barrier(world)
        dom_only_ms = max_over_ranks(float(st[:, di].mean()), world)

    e2e = None
    if e2e_on and not args.no_e2e:
        if wl.in_bf16:
            xh = torch.from_numpy(data.x_bits.view(np.int16)).pin_memory()
            yh = torch.empty((T, wl.d), dtype=torch.int16).pin_memory()
        else:
            xh = torch.from_numpy(data.x).pin_memory()
            yh = torch.empty((T, wl.d), dtype=torch.float32).pin_memory()
        lh = torch.from_numpy(data.router_logits).pin_memory() if data.router_logits is not None else None
        bh = torch.from_numpy(data.router_bias).pin_memory() if data.router_bias is not None else None
        for _ in range(max(3, args.warmup)):
            M.moe_w8a8_forward_host(W, xh, T, bh, lh, yh, ws)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0.record(stream)
        for _ in range(K):
            M.moe_w8a8_forward_host(W, xh, T, bh, lh, yh, ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world)
        h2d = xh.numel() * xh.element_size() + (lh.numel() * 4 if lh is not None else 0) + \
            (bh.numel() * 4 if bh is not None else 0)
        e2e = {"value": world * T * K / (ms_e2e / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(yh.numel() * yh.element_size())}

    peaks, peak_src = load_peaks()
    tpk = getattr(args, "tensor_peak", None)
    if tpk:
        int8_peak = tpk["burst"]["tops"]
        int8_src = (f"burst rate of the library's own tcgen05 8-bit MMA loop on this GPU "
                    f"({tpk['burst']['ms']:.1f} ms); sustained {tpk['sustained']['tops']:.0f} TOPS")
    else:
        int8_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * INT8_PER_BF16
        int8_src = f"2 x bf16_tflops_sustained of {peak_src} (INT8 dense = 2 x bf16, nominal)"
    roof = None
    if stages:
        dom_ms = dom_only_ms
        # the library's rule for SM pairs (a cta_pairs setting of 2 or the default)
        cp = getattr(args, "cta_pairs", -1)
        pairs = cp == 1 or (cp in (-1, 2) and wl.T * wl.k >= 256 * wl.E)
        kernel = (f"tc_{'pair_' if pairs else ''}gemm_kernel<{0 if dom == 'gemm1' else 1}>" if tensor else
                  ("stream_gateup_kernel" if dom == "gemm1" else "stream_down_kernel"))
        ops = 2 * R * (2 * wl.f if dom == "gemm1" else wl.f) * wl.d
        nbytes = alg[f"{dom}_bytes"]
        if fused:
            kernel, ops, nbytes = f"tc_ffn_fused_kernel<{1 if fp8 else 0}>", alg["int8_ops"], alg["fused_bytes"]
        timing = (f"mean of {K} CUDA event pairs around this stage alone on the forward's stream "
                  f"({stages[dom]:.4f} ms with event pairs around every stage)")
        # the bound is whichever of the byte time and the INT8 op time is larger
        if ops / (int8_peak * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9):
            achieved = ops / (dom_ms / 1e3) / 1e12
            roof = {"bound": "tensor", "kernel": f"{dom} ({kernel})", "achieved": achieved,
                    "peak": int8_peak, "unit": "TFLOP/s", "frac": achieved / int8_peak,
                    "traffic": load_traffic().get((wl.name, wl.T, norm_kernel(kernel))),
                    "peak_source": int8_src,
                    "int8_ops_per_launch": ops, "launch_ms": dom_ms, "launch_timing": timing,
                    "frac_of_nominal_4500": achieved / NOMINAL_INT8_TOPS}
            if tpk:
                roof["frac_of_sustained"] = achieved / tpk["sustained"]["tops"]
        else:
            achieved = nbytes / (dom_ms / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": f"{dom} ({kernel})", "achieved": achieved,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                    "traffic": load_traffic().get((wl.name, wl.T, norm_kernel(kernel))),
                    "peak_source": f"hbm_gbs of {peak_src}",
                    "algorithmic_bytes_per_launch": nbytes, "launch_ms": dom_ms, "launch_timing": timing}
    step_s = ms_total / K / 1e3
    layer_gbs = alg["layer_bytes"] / step_s / 1e9
    layer_tops = alg["int8_ops"] / step_s / 1e12
    if roof is not None:
        # the whole layer step against the same bound (roofline.frac is the dominant kernel's)
        if roof["bound"] == "hbm":
            roof["layer"] = {"achieved": layer_gbs, "frac": layer_gbs / peaks["hbm_gbs"], "unit": "GB/s",
                             "algorithmic_bytes_per_step": alg["layer_bytes"]}
        else:
            roof["layer"] = {"achieved": layer_tops, "frac": layer_tops / int8_peak, "unit": "TOPS",
                             "int8_ops_per_step": alg["int8_ops"]}
    out = {
        "value": world * T * K / (ms_total / 1e3), "ms_per_step": ms_total / K,
        "config": {"workload": describe(wl), "T": T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f,
                   "alpha": wl.alpha, "active_experts": n_active, "rows": R,
                   "expert_path": "tcgen05 grouped GEMM" if tensor else "weight streaming",
                   "l2": (f"inputs larger than L2: {alg['layer_bytes'] / 1e9:.2f} GB of algorithmic "
                          f"bytes per step (INT8 weights of the active experts, X, Y) vs 126 MB L2; "
                          f"no flush"),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "layer_bytes_per_step": alg["layer_bytes"], "layer_gbs": layer_gbs,
                   "layer_hbm_frac": layer_gbs / peaks["hbm_gbs"],
                   "int8_ops_per_step": alg["int8_ops"], "layer_int8_tops": layer_tops,
                   "layer_int8_frac": layer_tops / int8_peak,
                   "layer_int8_frac_of_nominal_4500": layer_tops / NOMINAL_INT8_TOPS},
        "roofline": roof, "stages_ms": stages, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if clip > 0.0:
        out["config"]["act_clip"] = {"percentile": args.act_clip, "value": clip}
    return out, wts, W


def run_sweep(args, local):
    """T in {1 .. 16384} x {uniform, Zipf(1.1) skew} x alpha in {0.5, 0.7} on the
    decode layer's shape and weights (seeds 10..41): tokens/s per point for the
    weight-streaming and the tcgen05 expert paths, with the roofline fraction of
    the bound that applies (HBM below the machine balance, INT8 tensor above)."""
    import torch

    import w8a8_quantized_moe_b200 as M

    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    tpk = measure_tensor_peak(local, 0)
    int8_peak = tpk["burst"]["tops"]
    points = synth.sweep_workloads()
    base = synth.WORKLOADS["decode"]
    wts = synth.make_weights(base)
    handles = {}
    for wl in points:
        if wl.alpha not in handles:
            cfg = M.make_config(wl.d, wl.f, wl.E, wl.k, wl.alpha, 0.0, True, M.MOE_BF16, M.MOE_BF16)
            cal = torch.from_numpy(synth.f32_to_bf16_bits(wts.calib_x).view(np.int16)).view(torch.bfloat16).to(dev)
            ax = torch.zeros(wl.d, dtype=torch.float32, device=dev)
            M.moe_w8a8_calibrate_absmax(cal, ax)
            wg, wu, wd = (torch.from_numpy(a).to(dev) for a in (wts.w_gate, wts.w_up, wts.w_down))
            # one router W_g ~N(0, 0.02^2) for the whole sweep (part of the layer's weights)
            wr = torch.from_numpy(synth.normal(base.weight_seed, synth.TID_W_ROUTER, (wl.d, wl.E),
                                               std=0.02)).to(dev)
            handles[wl.alpha] = M.moe_w8a8_prepare(cfg, wg, wu, wd, wr, ax)
            del wg, wu, wd
            torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)
    for wl in points:
        W = handles[wl.alpha]
        data = synth.make_data(wl)
        T = wl.T
        x = torch.from_numpy(data.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        bias = torch.from_numpy(data.router_bias).to(dev) if data.router_bias is not None else None
        logits = None   # the layer's router computes X W_router (timed)
        y = torch.empty((T, wl.d), dtype=torch.bfloat16, device=dev)
        for path_name, path in (("stream", M.MOE_PATH_STREAM), ("tensor", M.MOE_PATH_TENSOR)):
            M.moe_w8a8_set_path(W, path)
            ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device=dev)
            offs = torch.empty(wl.E + 1, dtype=torch.int32, device=dev)
            M.moe_w8a8_forward(W, x, T, bias, logits, y, ws, {"offsets": offs})
            counts = np.diff(offs.cpu().numpy())
            n_active, R = int((counts > 0).sum()), int(counts.sum())
            alg = algorithmic(wl, n_active, R, path_name == "tensor")
            steps = max(3, min(args.steps, int(2e5 / max(T, 1))))
            for _ in range(3):
                M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for _ in range(steps):
                M.moe_w8a8_forward(W, x, T, bias, logits, y, ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            M.moe_w8a8_check_status(W)
            step_s = e0.elapsed_time(e1) / steps / 1e3
            t_hbm = alg["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)
            t_tc = alg["int8_ops"] / (int8_peak * 1e12)
            bound = "hbm" if t_hbm >= t_tc else "tensor"
            print(json.dumps({"sweep_point": wl.name, "T": T, "skew": "zipf1.1" if wl.zipf_s else "uniform",
                              "alpha": wl.alpha, "seed": wl.data_seed, "path": path_name,
                              "tokens_per_s": T / step_s, "ms_per_step": step_s * 1e3,
                              "active_experts": n_active, "rows": R, "bound": bound,
                              "roofline_frac": max(t_hbm, t_tc) / step_s,
                              "peak_source": f"hbm_gbs of {peak_src}; 8-bit tensor burst rate of the "
                                             f"library's MMA loop on this GPU ({int8_peak:.0f} TOPS)"}),
                  flush=True)
            del ws
        M.moe_w8a8_set_path(W, M.MOE_PATH_AUTO)


def run_ours(args, world, rank, local):
    import torch

    import w8a8_quantized_moe_b200 as M
    from w8a8_quantized_moe_b200 import build as B

    if not os.path.exists(M.LIB_PATH):
        B.build()
    torch.cuda.set_device(local)
    if args.sweep:
        if rank == 0:
            run_sweep(args, local)
        return
    import dataclasses
    base = synth.WORKLOADS[args.workload]
    if args.tokens > 0:
        base = dataclasses.replace(base, T=args.tokens)
    wl = replica_workload(base, rank)
    args.tensor_peak = measure_tensor_peak(local, 1 if args.format == "e4m3" else 0) \
        if not args.no_tensor_peak else None
    res, wts, W = measure(args, wl, world, rank, local)
    del W

    extra = None
    if args.workload == "decode" and not args.no_prefill:
        pw = replica_workload(synth.WORKLOADS["prefill"], rank)
        # the prefill layer reuses the decode layer's expert weights
        pres, _, PW = measure(args, pw, world, rank, local, e2e_on=False, wts=wts)
        del PW
        torch.cuda.empty_cache()
        extra = {"metric": "prefill layer tokens/s (T=16384)", "unit": "tokens/s", **pres}
    large = None
    if args.workload == "decode" and not args.no_large:
        lw = replica_workload(synth.WORKLOADS["large"], rank)
        # its fp32 weights (51.5 GB) are generated and uploaded expert by expert, untimed
        lres, _, LW = measure(args, lw, world, rank, local, e2e_on=False)
        del LW
        torch.cuda.empty_cache()
        large = {"metric": "large sparse layer tokens/s (T=4096, d=8192, E=256, top-8, capacity 1.25)",
                 "unit": "tokens/s", **lres,
                 "cpu_baseline": {"value": None, "unit": "tokens/s", "cores": 0, "kind": "oracle",
                                  "sample": "not run for this layer: its smoothing statistic needs all 256 "
                                            "experts' fp32 weights on the host"}}

    if rank != 0:
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline and wts is None:
        cpu = {"value": None, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": "not run: this workload's fp32 weights (over 8 GB) are generated on the "
                         "device expert by expert, and the oracle would need all of them on the host"}
    elif world == 1 and not args.no_cpu_baseline:
        import oracle
        prepare = oracle.prepare_fp8 if args.format == "e4m3" else oracle.prepare
        prep = prepare(wts.w_gate, wts.w_up, wts.w_down, wts.calib_x, wl.alpha)
        n_tok = min(wl.T, 32)
        sdata = synth.make_data(wl, T=n_tok)
        secs, n = 0.0, 0
        while n == 0 or secs < args.cpu_seconds:
            secs += oracle_step(wl, prep, sdata)
            n += 1
        cpu = {"value": n * n_tok / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} steps of the first {n_tok} of the {wl.T} tokens of the {wl.name} workload "
                         f"({secs:.1f} s of single-thread CPU time; preparation untimed)"}
        # the same oracle code with the sample's tokens split over all host cores
        cores = min(host_cores(), n_tok)
        psecs, pn = 0.0, 0
        while pn == 0 or psecs < args.cpu_seconds / 2:
            psecs += oracle_step_threads(wl, prep, sdata, cores)[0]
            pn += 1
        cpu["all_cores"] = {"value": pn * n_tok / psecs, "unit": "tokens/s", "cores": cores,
                            "sample": f"{pn} steps of the same {n_tok} tokens, split over {cores} host threads "
                                      f"({psecs:.1f} s wall time)"}

    line = {"metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if args.format == "e4m3" else "int8",
            "data": "synthetic", "config": res["config"], "roofline": res["roofline"],
            "stages_ms": res["stages_ms"], "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
            "clocks": res["clocks"], "cpu_baseline": cpu}
    if extra is not None:
        line["prefill"] = extra
    if large is not None:
        line["large"] = large
    if args.tensor_peak:
        line["tensor_peak"] = args.tensor_peak
    print(json.dumps(line), flush=True)


def run_ep(args, world, rank, local):
    """The expert-parallel layer: rank g holds experts [g E/N, (g+1) E/N) (only
    those are generated and prepared), routes its own batch of T tokens, and
    exchanges rows with the other ranks (one All-to-All each way).  Times K
    layer steps with CUDA events on the current stream (the host's reads of
    the row counts are inside the timed region); max over ranks.  On one rank
    it also times the single-GPU forward on the same handle."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    import w8a8_quantized_moe_b200 as M
    from w8a8_quantized_moe_b200 import build as B
    from w8a8_quantized_moe_b200.ep import ExpertParallelMoE, LibraryStages, equal_expert_ranges, \
        prepare_expert_shard

    if not os.path.exists(M.LIB_PATH):
        B.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    own_group = world == 1
    if own_group:
        with socket.socket() as sock:
            sock.bind(("127.0.0.1", 0))
            port = sock.getsockname()[1]
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    try:
        wl = replica_workload(synth.WORKLOADS[args.workload], rank)
        first, n = equal_expert_ranges(wl.E, world)[rank]
        per = wl.d * wl.f
        wg = torch.empty((n, wl.d, wl.f), dtype=torch.float32, device=dev)
        wu = torch.empty((n, wl.d, wl.f), dtype=torch.float32, device=dev)
        wd = torch.empty((n, wl.f, wl.d), dtype=torch.float32, device=dev)
        for i in range(n):
            e = first + i
            for dst, tid, shape in ((wg, synth.TID_W_GATE, (wl.d, wl.f)), (wu, synth.TID_W_UP, (wl.d, wl.f)),
                                    (wd, synth.TID_W_DOWN, (wl.f, wl.d))):
                dst[i].copy_(torch.from_numpy(synth.normal(wl.weight_seed, tid, shape, std=wl.weight_std,
                                                           start=e * per)))
        calib_x, _ = synth.activations(wl.weight_seed + synth.CALIB_SEED_OFFSET, synth.CALIB_TOKENS, wl.d,
                                       wl.outlier_channels(), wl.outlier_factor, wl.in_bf16)
        if wl.in_bf16:
            cal = torch.from_numpy(synth.f32_to_bf16_bits(calib_x).view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            cal = torch.from_numpy(calib_x).to(dev)
        ax = torch.zeros(wl.d, dtype=torch.float32, device=dev)
        M.moe_w8a8_calibrate_absmax(cal, ax)
        data = synth.make_data(wl)
        wr = torch.from_numpy(data.w_router).to(dev)
        cfg = M.make_config(wl.d, wl.f, wl.E, wl.k, wl.alpha, wl.capacity_factor, True,
                            M.MOE_BF16 if wl.in_bf16 else M.MOE_F32, M.MOE_BF16 if wl.in_bf16 else M.MOE_F32,
                            M.MOE_FMT_E4M3 if args.format == "e4m3" else M.MOE_FMT_INT8)
        W = prepare_expert_shard(cfg, first, wg, wu, wd, wr, ax)
        del wg, wu, wd, cal
        torch.cuda.empty_cache()
        layer = ExpertParallelMoE(LibraryStages(W))
        T = wl.T
        x = torch.from_numpy(data.x_bits.view(np.int16)).view(torch.bfloat16).to(dev) if wl.in_bf16 \
            else torch.from_numpy(data.x).to(dev)
        logits = torch.from_numpy(data.router_logits).to(dev) if data.router_logits is not None else None
        bias = torch.from_numpy(data.router_bias).to(dev) if data.router_bias is not None else None
        y = torch.empty((T, wl.d), dtype=torch.bfloat16 if wl.in_bf16 else torch.float32, device=dev)
        stream = torch.cuda.current_stream(dev)

        def timed(step):
            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(world)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            return e0.elapsed_time(e1) / args.steps

        clocks = ClockSampler(local)
        clocks.start()
        ms_ep = max_over_ranks(timed(lambda: layer.forward(x, T, bias, logits, y)), world)
        clocks.stop()
        M.moe_w8a8_check_status(W)
        sent, received = layer.last_rows
        # the fixed-block exchange: equal All-to-All parts, no host read of a count
        blocked = ExpertParallelMoE(LibraryStages(W), block_tokens=T)
        yb = torch.empty_like(y)
        ms_blocked = max_over_ranks(timed(lambda: blocked.forward(x, T, bias, logits, yb)), world)
        M.moe_w8a8_check_status(W)
        torch.cuda.synchronize(dev)
        assert torch.equal(y, yb), "fixed-block exchange output differs from the counted one"
        ms_fwd = None
        if world == 1:
            ws = torch.empty(M.moe_w8a8_workspace_size(W, T), dtype=torch.uint8, device=dev)
            yf = torch.empty_like(y)
            ms_fwd = timed(lambda: M.moe_w8a8_forward(W, x, T, bias, logits, yf, ws))
            torch.cuda.synchronize(dev)
            assert torch.equal(y, yf), "expert-parallel output differs from the forward"
        if rank == 0:
            line = {"metric": "expert-parallel W8A8 MoE layer tokens/s", "value": world * T / ms_ep * 1e3,
                    "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": ms_ep, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                    "dtype": "e4m3" if args.format == "e4m3" else "int8", "data": "synthetic",
                    "config": {"workload": describe(wl) + f"; expert-parallel over {world} rank(s), "
                                                          f"{n} experts per rank, {T} tokens per rank",
                               "parallelism": f"ep{world}", "experts_per_rank": n,
                               "rank0_rows_sent": sent, "rank0_rows_received": received,
                               "exchange": "torch.distributed all_to_all_single (NCCL), host reads the "
                                           "row counts each step",
                               "l2": "weights larger than L2; no flush"},
                    "single_gpu_forward_ms": ms_fwd, "clocks": clocks.summary(),
                    "blocked_exchange": {"ms_per_step": ms_blocked, "value": world * T / ms_blocked * 1e3,
                                         "unit": "tokens/s", "block_tokens": T,
                                         "exchange": "all_to_all_single of fixed blocks (T k + 1 rows per "
                                                     "peer, count in a header row read on the device); no "
                                                     "host read"}}
            print(json.dumps(line), flush=True)
    finally:
        if own_group:
            dist.destroy_process_group()


def main():
    args = parse()
    if args.record_traffic:
        wl = synth.WORKLOADS[args.workload]
        record_traffic(args.record_traffic, args.workload, args.tokens or wl.T, args.traffic_scale)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.ep:
            run_ep(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
