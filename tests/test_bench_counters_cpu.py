"""bench.py's reading of an ncu --csv log into the per-launch counters it
reports (DRAM bytes, warp and thread instructions), on CPU."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


CSV = '''==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","4.26"
"0","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","1,024"
"0","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","usecond","12.10"
"0","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","smsp__inst_executed.sum","inst","5,780,000"
"0","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","smsp__thread_inst_executed.sum","inst","160,000,000"
"1","1","python","h","trellis_gemv_kernel","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","9.99"
'''


def test_record_counters_reads_the_first_launch(tmp_path, monkeypatch):
    bench = _bench()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "_source_hash", lambda kind: "h-" + kind)
    log = tmp_path / "c.csv"
    log.write_text(CSV)
    bench.record_counters(str(log), "gemv_attn4096_b1", "profiles/x.md")
    d = json.load(open(tmp_path / "profiles" / "counters.json"))
    e = d["gemv_attn4096_b1"]
    assert e["dram_bytes"] == 4.26e6 + 1024
    assert e["warp_inst"] == 5.78e6 and e["thread_inst"] == 1.6e8
    assert abs(e["duration_us_ncu"] - 12.10) < 1e-9
    assert e["source_hash"] == "h-gemv"
    assert bench._counters("gemv_attn4096_b1")["warp_inst"] == 5.78e6
    monkeypatch.setattr(bench, "_source_hash", lambda kind: "changed")
    assert bench._counters("gemv_attn4096_b1") is None


def test_nanosecond_durations_are_read():
    bench = _bench()
    assert bench._UNITS["ns"] == 1e-9 and bench._UNITS["us"] == 1e-6 and bench._UNITS["ms"] == 1e-3


def test_roofline_takes_the_burst_peak_for_short_loops_only():
    bench = _bench()
    import workloads as wl
    sp = wl.WORKLOADS["halftcq"]
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    short = bench.roofline(sp, 256, 40e-6, pk, "measured", 1965.0, 148, "t", burst_gemm=True, chain_s=45e-6)
    long_ = bench.roofline(sp, 256, 40e-6, pk, "measured", 1965.0, 148, "t", burst_gemm=False)
    flops = 2.0 * sp.m * sp.n * 256
    assert short["bound"] == "tensor" and abs(short["achieved"] - flops / 40e-6 / 1e12) < 1e-9
    assert short["peak"] == 1600.0 and long_["peak"] == 1400.0
    assert abs(short["frac"] * 1600.0 - long_["frac"] * 1400.0) < 1e-9
    assert abs(short["kernel_us_in_forward"] - 45.0) < 1e-9 and "kernel_us_in_forward" not in long_
    gemv = bench.roofline(wl.WORKLOADS["attn4096"], 1, 8e-6, pk, "measured", 1965.0, 148, "t", burst_gemm=True)
    alg = wl.WORKLOADS["attn4096"].stream_bytes + 4096 * 2 + 4096 * 4
    assert gemv["bound"] == "hbm" and abs(gemv["achieved"] - alg / 8e-6 / 1e9) < 1e-6
