"""The bench's algorithmic byte / op model (the numerators of the roofline
fractions), checked against figures worked out by hand from the layer's shapes:
an active expert carries 3 d f INT8 weight bytes and (2f + d) fp32 scales, a
token d input and d output elements, and a kept row 2 * 3 d f INT8 ops."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    return bench, synth


def test_decode_layer_bytes_and_ops():
    bench, synth = _bench()
    wl = synth.WORKLOADS["decode"]          # T=32, d=4096, E=64, k=4, f=1536, bf16, given logits
    a = bench.algorithmic(wl, n_active=56, R=128, tensor=True)
    # 56 * 3 * 4096 * 1536 weight bytes          = 1,056,964,608
    # 56 * (2 * 1536 + 4096) * 4 scale bytes     =     1,605,632
    # 32 tokens * 4096 * 2 bytes, in and out     =       524,288
    # given router logits 32 * 64 * 4            =         8,192
    assert a["layer_bytes"] == 1_059_102_720
    assert a["int8_ops"] == 4_831_838_208     # 2 * 128 * 3 * 4096 * 1536
    # the fused launch reads both GEMMs' weights once: at least the weight bytes
    assert a["fused_bytes"] >= 1_056_964_608


def test_prefill_ops():
    bench, synth = _bench()
    wl = synth.WORKLOADS["prefill"]         # T=16384, top-4: 65,536 rows
    a = bench.algorithmic(wl, n_active=64, R=65536, tensor=True)
    assert a["int8_ops"] == 2_473_901_162_496
    # GEMM1 is two thirds of the ops: 2 * 65536 * 3072 * 4096
    assert 2 * 65536 * 2 * 1536 * 4096 == 1_649_267_441_664


def test_layer_bytes_count_only_active_experts():
    bench, synth = _bench()
    wl = synth.WORKLOADS["decode"]
    a40 = bench.algorithmic(wl, n_active=40, R=128)
    a41 = bench.algorithmic(wl, n_active=41, R=128)
    assert a41["layer_bytes"] - a40["layer_bytes"] == 3 * 4096 * 1536 + (2 * 1536 + 4096) * 4


def test_gemm2_bytes_count_per_slot_rows_in_the_output_dtype():
    bench, synth = _bench()
    wl = synth.WORKLOADS["decode"]           # bf16 output: 2-byte per-slot rows
    a = bench.algorithmic(wl, n_active=56, R=128, tensor=True)
    # 56 * 4096 * 1536 weights + 128 * 1536 h codes + 128 * 4096 * 2 rows + 56 * 4096 * 4 scales
    assert a["gemm2_bytes"] == 352_321_536 + 196_608 + 1_048_576 + 917_504


def test_traffic_record_and_lookup(tmp_path, monkeypatch):
    """An ncu CSV's per-kernel DRAM bytes become a table row stamped with the
    sources hash; the lookup uses it only while the hash matches."""
    bench, synth = _bench()
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "dram_traffic.md"))
    hdr = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
           '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    rows = []
    for i, (rd, wr) in enumerate([(1000.0, 10.0), (1002.0, 12.0)]):
        for m, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr)):
            rows.append(f'"{i}","1","python","h","void moe::(anonymous namespace)::tc_ffn_fused_kernel<0>'
                        f'(CUtensorMap_st, TcParams)","1","7","(352, 1, 1)","(148, 1, 1)","0","10.0",'
                        f'"Command line profiler metrics","{m}","Mbyte","{v}"\n')
    csv_path = tmp_path / "l.csv"
    csv_path.write_text("==PROF== noise\n" + hdr + "".join(rows))
    bench.record_traffic(str(csv_path), "decode", 32)
    t = bench.load_traffic()
    # keyed by the name without namespaces or parameters and its first template argument
    assert abs(t[("decode", 32, "tc_ffn_fused_kernel<0>")] - 1012e6) < 1.0
    assert bench.norm_kernel("void moe::<unnamed>::tc_pair_gemm_kernel<1, 0>(CUtensorMap_st)") == \
        "tc_pair_gemm_kernel<1>"
    assert bench.norm_kernel("moe::<unnamed>::router_select_kernel(const unsigned short *)") == \
        "router_select_kernel"
    # a different sources hash: the row is ignored
    monkeypatch.setattr(bench, "sources_hash", lambda: "0" * 16)
    assert bench.load_traffic() == {}


def test_reference_arm_line_keeps_the_contract():
    """`bench.py --impl reference` (the CPU oracle as the reference arm) prints one JSON line
    with the contract's keys; it needs no GPU."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root, check=True).stdout
    lines = [json.loads(x) for x in out.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (2, 1, 1)
    assert all(k in d["config"] for k in ("workload", "T", "d", "E", "k", "f"))
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
