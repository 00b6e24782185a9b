#!/usr/bin/env python
"""Throughput of the trellis-coded quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--batch B]

A step is one forward y = W x of the layer (input random-sign Hadamard
transform, fused trellis decode + contraction, output transform) over one
batch of synthetic inputs.  The default workload is the 2-bit 4096 x 4096
3INST layer at batch 1.  Steps rotate through enough independent layer
instances that their code words (4 MiB each) exceed the 126 MB L2 four times
over, so every step streams its weights from HBM; the rotation is replayed
from a CUDA graph.  One JSON line goes to stdout (rank 0).

N > 1: one process per GPU (torchrun, NCCL process group for the barrier and
the max-over-ranks timing only); each rank runs its own independent layer
instances (weak scaling, no collective on the data path).

--impl reference runs the float64 CPU oracle as the reference arm on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "quantized-linear tokens/s and compressed-weight HBM GB/s (% of B200 peak)"
L2_BYTES = 126 * 1024 * 1024
GEMV_MAX_BATCH = 8  # the library runs batch <= 8 on the decode-GEMV, larger batches on the tensor-core GEMM
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50000)
    p.add_argument("--warmup", type=int, default=500)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="attn4096", choices=sorted(wl.WORKLOADS))
    p.add_argument("--batch", type=int, default=None)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="skip the per-configuration measurements of every benchmark (workload, batch) pair")
    p.add_argument("--encode", action="store_true",
                   help="time the trellis-coded quantizer (qlinear_encode, k = 2, 3INST) on an N(0,1) "
                        "source instead of the forward")
    p.add_argument("--encode-L", type=int, default=16, help="state bits of the --encode run (at most 16)")
    p.add_argument("--encode-blocks", type=int, default=148 * 8,
                   help="source blocks of 256 values per --encode step (a smaller count for profiler captures)")
    p.add_argument("--record-counters", nargs=3, metavar=("NCU_CSV", "KEY", "CAPTURE"),
                   help="store the counters of an ncu --csv log in profiles/counters.json under KEY (e.g. "
                        "gemv_attn4096_b1) and exit; CAPTURE names the profile that gives the command")
    p.add_argument("--instances", type=int, default=None,
                   help="layer instances to rotate through (default: enough code words for 4x L2); a smaller "
                        "count is for profiler captures only, and the line then says its inputs may sit in L2")
    a = p.parse_args()
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def config_dict(sp, batch, n_inst, extra=None):
    d = {"workload": f"{sp.name}: m={sp.m} n={sp.n} bits/weight={sp.bits_per_weight:g} L={sp.L} V={sp.V} "
                     f"code={wl.CODE_NAMES[sp.code]}" + (f" Q={sp.Q}" if sp.Q else ""),
         "global_batch": batch, "seq_len": 1, "parallelism": "independent layer instances per GPU",
         "l2": (f"inputs larger than L2: rotating {n_inst} layer instances "
                f"({n_inst * sp.stream_bytes / 2**20:.0f} MiB of code words)")
               if n_inst * sp.stream_bytes >= 4 * L2_BYTES else
               f"PROFILING CASE, not a benchmark: {n_inst} layer instances "
               f"({n_inst * sp.stream_bytes / 2**20:.0f} MiB of code words) may stay in L2"}
    if extra:
        d.update(extra)
    return d


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.12)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ oracle arms
def _oracle_chunked(sp, batch, blocks_per_step, steps, deadline=None):
    """Run the oracle forward in steps of `blocks_per_step` 256-column blocks of
    W_hat (row-major order): the first step of every forward also applies the
    input transform, the step that completes z the output transform.
    Returns (seconds, blocks processed)."""
    from oracle import hadamard, qlinear
    layer = qlinear.Layer.from_inputs(wl.make_layer(sp))
    x = wl.make_x(sp, batch)
    nb = sp.n // 256
    total = sp.m * nb
    z = np.zeros((batch, sp.m))
    xp = None
    pos = 0
    done = 0
    t0 = time.perf_counter()
    for _ in range(steps):
        if pos == 0:
            xp = layer.input_transform(x)
            z[:] = 0.0
        left = blocks_per_step
        while left > 0:
            r, j0 = divmod(pos, nb)
            j1 = min(nb, j0 + left)
            W = layer.decode_rows([r], np.arange(j0, j1))
            z[:, r] += qlinear.contract(W, xp[:, j0 * 256:j1 * 256])[:, 0]
            left -= j1 - j0
            pos += j1 - j0
            done += j1 - j0
            if pos == total:
                y = layer.alpha * layer.s_out * hadamard.apply_blockwise(z, layer.B_m)
                assert np.all(np.isfinite(y))
                pos = 0
                break
        if deadline is not None and time.perf_counter() - t0 > deadline:
            break
    return time.perf_counter() - t0, done


def cpu_baseline(sp, batch, budget_s=15.0):
    nb = sp.n // 256
    secs, blocks = _oracle_chunked(sp, batch, 16 * nb, steps=10**9, deadline=budget_s)
    fwd = blocks / (sp.m * nb)
    return {"value": batch * fwd / secs, "unit": "tokens/s", "cores": 1, "cpu_model": _cpu_model(), "kind": "oracle",
            "sample": f"{blocks // nb} of {sp.m} rows of W_hat ({fwd:.3f} forwards) of {sp.name} at batch {batch}: "
                      f"float64 trellis walk, code evaluation, dense Hadamard blocks, matrix product; "
                      f"{secs:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sp = wl.WORKLOADS[args.workload]
    batch = args.batch or sp.batches[0]
    # calibrate: blocks per step so that warmup + steps fit in about two minutes
    nb = sp.n // 256
    t_row, _ = _oracle_chunked(sp, batch, nb, 1)
    per_block = t_row / nb
    budget = 120.0
    bps = int(max(1, min(sp.m * nb, budget / max(1, args.steps + args.warmup) / per_block)))
    _oracle_chunked(sp, batch, bps, args.warmup)
    secs, done = _oracle_chunked(sp, batch, bps, args.steps)
    value = batch * (done / (sp.m * nb)) / secs
    rows = bps / nb
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(sp, batch, 1, {"l2": "CPU oracle: no GPU caches involved",
                                                 "step": f"{bps} blocks of 256 columns of W_hat per step "
                                                         f"(1/{sp.m * nb / bps:g} of a forward)"}),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "cpu_model": _cpu_model(), "kind": "oracle",
                             "sample": f"{done} blocks of 256 columns of W_hat in {args.steps} steps of {bps}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ranks
def max_over_ranks(values, device):
    """Each value's maximum over all ranks (the values unchanged on one rank).
    Every rank must call this with the same number of values."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(world, steps, batch, secs):
    """Whole-job throughput: every rank ran `steps` forwards of `batch` tokens
    (weak scaling), timed as the slowest rank's `secs`."""
    return world * steps * batch / secs


# ------------------------------------------------------------------ CUDA arm
# the sources each profiled kernel is built from (its DRAM-traffic capture is
# valid while these are unchanged)
KERNEL_SOURCES = {
    "gemv": ("gemv.cu", "codes.cuh", "layout.cuh", "fwht.cuh", "xstep.cuh", "internal.h"),
    "gemm": ("gemm_tc.cu", "codes.cuh", "layout.cuh", "tc_ptx.cuh", "internal.h"),
}


def _source_hash(kind):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "trellis_coded_matmul_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


_UNITS = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "inst": 1, "": 1, "nsecond": 1e-9, "ns": 1e-9,
          "us": 1e-6, "ms": 1e-3,
          "usecond": 1e-6, "msecond": 1e-3}
_COUNTER_METRICS = {"dram__bytes_read.sum": "dram_read", "dram__bytes_write.sum": "dram_write",
                    "smsp__inst_executed.sum": "warp_inst", "smsp__thread_inst_executed.sum": "thread_inst",
                    "gpu__time_duration.sum": "duration_s"}


def record_counters(csv_path, key, capture):
    """Store the counters of the first kernel launch in an ncu --csv log under
    `key` in profiles/counters.json, stamped with the hash of that kernel's
    sources (bench.py reports them only while the sources are unchanged)."""
    import csv
    rows = list(csv.reader(l for l in open(csv_path) if l.startswith('"')))
    head = rows[0]
    iid, iname, iunit, ival = (head.index(c) for c in ("ID", "Metric Name", "Metric Unit", "Metric Value"))
    first = rows[1][iid]
    vals = {}
    for r in rows[1:]:
        if r[iid] != first or r[iname] not in _COUNTER_METRICS:
            continue
        vals[_COUNTER_METRICS[r[iname]]] = float(r[ival].replace(",", "")) * _UNITS[r[iunit]]
    entry = {"dram_bytes": vals.get("dram_read", 0) + vals.get("dram_write", 0),
             "warp_inst": vals.get("warp_inst"), "thread_inst": vals.get("thread_inst"),
             "duration_us_ncu": vals.get("duration_s", 0) * 1e6,
             "source_hash": _source_hash(key.split("_")[0]), "capture": capture}
    path = os.path.join(ROOT, "profiles", "counters.json")
    d = json.load(open(path)) if os.path.exists(path) else {
        "_note": "per-launch counters of one ncu capture per kernel and workload (dram bytes read + written, warp "
                 "and thread instructions executed); bench.py uses an entry only while the kernel's sources hash "
                 "to its source_hash"}
    d[key] = entry
    json.dump(d, open(path, "w"), indent=1, sort_keys=True)
    print(json.dumps({key: entry}))


def run_encode(args):
    """The GPU trellis-coded quantizer on an i.i.d. N(0,1) source: blocks of 256
    values, L = --encode-L (16 by default), k = 2, V = 1, 3INST; each step is one
    qlinear_encode call (scratch allocation and the stream synchronisation
    included).

    Roofline: the search is plain fp32 ALU work.  Per block it updates 2^L
    states at each of the T = 256 / V steps of both passes, and a state update
    is 3V + (C - 1) / C operations (V subtractions, V multiplications, V - 1
    additions over the values, one addition to the path cost, and one C-way
    minimum per group of C = 2^kV states).  The peak is the SM array's fp32
    lane rate at the highest SM clock seen (128 lanes per SM per clock)."""
    import torch
    import trellis_coded_matmul_b200 as tcm
    L, k, V, code = args.encode_L, 2, 1, wl.CODE_3INST
    blocks = args.encode_blocks
    x = torch.randn((blocks, 256), generator=torch.Generator().manual_seed(7)).cuda()
    for _ in range(args.warmup):
        tcm.qlinear_encode(code, L, k, V, x)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        _, err = tcm.qlinear_encode(code, L, k, V, x, with_error=True)
    end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    secs = start.elapsed_time(end) * 1e-3
    C = 1 << (k * V)
    ops_per_block = 2 * (256 // V) * (1 << L) * (3 * V + (C - 1) / C)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    max_mhz = clk["sm_max_mhz"] if clk else 1965.0
    peak = sms * 128 * max_mhz * 1e6 / 1e12
    achieved = ops_per_block * blocks * args.steps / secs / 1e12
    line = {"metric": "trellis-coded quantization (two-pass tail-biting Viterbi) source weights/s",
            "value": blocks * 256 * args.steps / secs, "unit": "weights/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"encode: {blocks} blocks of 256 N(0,1) values, L={L} k={k} V={V} code=3INST",
                       "mse": float(err.sum()) / (blocks * 256)},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Top/s", "frac": achieved / peak,
                         "traffic": None, "ops_per_block": ops_per_block,
                         "peak_kind": f"derived: {sms} SMs x 128 fp32 lanes x {max_mhz:.0f} MHz"},
            "gpu_launches": args.steps, "clocks": clk}
    if not args.no_cpu_baseline:
        from oracle import encode as oenc
        xs = x[:4].cpu().numpy()
        t0 = time.perf_counter()
        done = 0
        for blk in xs:
            oenc.encode_two_pass(blk.reshape(-1, V), L, k, V, code)
            done += 1
            if time.perf_counter() - t0 > 20.0:
                break
        cs = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": done * 256 / cs, "unit": "weights/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"{done} blocks of 256 values: oracle.encode.encode_two_pass (numpy "
                                          f"element-wise, one thread; float32 costs), {cs:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


# The (workload, batch) pairs the layer shapes are benchmarked at: the five
# layer configurations of the workload list with their batches.
PER_CONFIG = [("tiny", 1), ("attn4096", 1), ("mlp_up", 1), ("mlp_up", 4), ("mlp_up", 8), ("mlp_down", 1),
              ("mlp_down", 4), ("mlp_down", 8), ("large", 1), ("large", 4), ("large", 16), ("halftcq", 64),
              ("halftcq", 256)]


def _counters(key):
    """Per-launch counters of the kernel `key` from the committed ncu summary
    (profiles/counters.json), if they were taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "counters.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(key)
    if not d or d.get("source_hash") != _source_hash(key.split("_")[0]):
        return None
    return d


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def make_handle(tcm, torch, li):
    sp_ = li.spec
    codes = torch.from_numpy(li.codes.view(np.int32).copy()).cuda()
    s_in = torch.from_numpy(li.s_in.copy()).cuda()
    s_out = torch.from_numpy(li.s_out.copy()).cuda()
    lut = torch.from_numpy(li.lut.copy()).cuda() if li.lut is not None else None
    if sp_.fractional:  # a half-integer bitwidth: parts given as bits per trellis step
        return tcm.qlinear_create_kv(sp_.m, sp_.n, [r for _, r, _ in sp_.row_parts()], sp_.part_kv(), sp_.L,
                                     sp_.V, sp_.code, codes, s_in, s_out, sp_.alpha, Q=sp_.Q, lut=lut)
    if sp_.row_split is not None:
        return tcm.qlinear_create_parts(sp_.m, sp_.n, [r for r, _ in sp_.row_split], [k for _, k in sp_.row_split],
                                        sp_.L, sp_.V, sp_.code, codes, s_in, s_out, sp_.alpha, Q=sp_.Q, lut=lut)
    if sp_.mixed:
        return tcm.qlinear_create_mixed(sp_.m, sp_.n, sp_.m_top, sp_.k_top, sp_.k_bot, sp_.L, sp_.V, sp_.code,
                                        codes, s_in, s_out, sp_.alpha, Q=sp_.Q, lut=lut)
    return tcm.qlinear_create(sp_.m, sp_.n, sp_.k, sp_.L, sp_.V, sp_.code, codes, s_in, s_out, sp_.alpha,
                              Q=sp_.Q, lut=lut)


class Runner:
    """Times forwards of one workload at one batch on this rank's GPU: steps
    rotate through enough independent layer instances that their code words
    exceed four times the L2 (replayed from CUDA graphs), and a separate replay
    with CUDA events around the layer's main kernel gives its duration."""

    def __init__(self, torch, tcm, dist, world, rank, stream, sp, batch, n_inst):
        self.torch, self.tcm, self.dist, self.world = torch, tcm, dist, world
        self.stream, self.sp, self.batch, self.n_inst = stream, sp, batch, n_inst
        self.handles = [make_handle(tcm, torch, wl.make_layer(sp, instance=1 + rank * 4096 + i)) for i in range(n_inst)]
        self.xs = [torch.from_numpy(wl.make_x(sp, batch, instance=i)).cuda() for i in range(n_inst)]
        self.ys = [torch.empty((batch, sp.m), dtype=torch.float32, device="cuda") for _ in range(n_inst)]
        self.graphs = []
        with torch.cuda.stream(stream):
            self.run_steps(n_inst)  # allocate per-handle scratch before capture
        torch.cuda.synchronize()

    def run_steps(self, count, start=0):
        for s in range(start, start + count):
            i = s % self.n_inst
            self.tcm.qlinear_forward(self.handles[i], self.xs[i], self.ys[i])

    def capture(self, count):
        if count == 0:
            return None
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, stream=self.stream):
            self.run_steps(count)
        self.graphs.append(g)
        return g

    def replay(self, steps, full, tail):
        for _ in range(steps // self.n_inst):
            full.replay()
        if steps % self.n_inst:
            tail.replay()

    def timed(self, fn):
        torch, dist = self.torch, self.dist
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            start.record(self.stream)
            fn()
            end.record(self.stream)
        torch.cuda.synchronize()
        if self.world > 1:
            dist.barrier()
        return start.elapsed_time(end) * 1e-3

    def throughput(self, steps, warmup):
        """Seconds for `steps` forwards after `warmup` untimed ones."""
        g_full, g_tail, g_warm = self.capture(self.n_inst), self.capture(steps % self.n_inst), \
            self.capture(warmup % self.n_inst)
        with self.torch.cuda.stream(self.stream):
            self.replay(warmup, g_full, g_warm)
        return self.timed(lambda: self.replay(steps, g_full, g_tail))

    def kernel_seconds(self, steps):
        """Average duration of the main kernel (decode-GEMV or tensor-core GEMM):
        the same steps again from a graph whose forwards carry CUDA events
        around that kernel (events between programmatically dependent launches
        serialise them, so this pass is separate from the throughput one)."""
        tcm = self.tcm
        for h in self.handles:
            tcm.qlinear_profile_enable(h, 1)
        prof_steps = min(steps, 4 * self.n_inst)
        g_prof, g_tail = self.capture(self.n_inst), self.capture(prof_steps % self.n_inst)
        with self.torch.cuda.stream(self.stream):
            g_prof.replay()
        prof_secs = self.timed(lambda: self.replay(prof_steps, g_prof, g_tail))
        ms, n = 0.0, 0
        for h in self.handles:
            a, b = tcm.qlinear_profile_read(h)
            ms += a
            n += b
            tcm.qlinear_profile_enable(h, 0)
        return ms * 1e-3 / max(1, n), prof_steps, prof_secs

    def main_kernel_seconds(self, steps):
        """Average duration of the main kernel (decode-GEMV or tensor-core GEMM)
        launched alone, back to back: every handle first runs one forward with
        this batch (its scratch then holds x'), then a graph of one
        main-kernel launch per instance (rotating, so the code words come from
        HBM as in the forwards) is replayed with CUDA events around the
        replays on the launching stream.  A last forward per handle leaves the
        accumulators clean."""
        torch, tcm = self.torch, self.tcm
        with torch.cuda.stream(self.stream):
            self.run_steps(self.n_inst)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(self.n_inst):
                tcm.qlinear_launch_main_kernel(self.handles[i], self.batch, self.xs[i], self.ys[i], stream=self.stream)
        self.graphs.append(g)
        with torch.cuda.stream(self.stream):
            g.replay()
        # a timed warm-up replay sizes the measured loop: at most `steps`
        # launches and about a quarter of a second (a kernel timed in isolation
        # for a short while, the condition of the burst peak)
        one = self.timed(lambda: g.replay())
        reps = max(2, min(-(-steps // self.n_inst), int(0.25 / max(one, 1e-9)) + 1))
        # the GPU idles for half a second first, as before the burst peak's own
        # short measurement (a long loop just before holds the power-capped clock)
        time.sleep(0.5)

        def body():
            for _ in range(reps):
                g.replay()
        secs = self.timed(body)
        with torch.cuda.stream(self.stream):
            self.run_steps(self.n_inst)
        torch.cuda.synchronize()
        return secs / (reps * self.n_inst), reps * self.n_inst, secs

    def e2e(self, steps):
        """Seconds for `steps` forwards through qlinear_forward_host (pinned host
        x in, host y out, copies and the stream synchronisation in every step)."""
        torch, tcm, sp, batch = self.torch, self.tcm, self.sp, self.batch
        x_h = [torch.from_numpy(wl.make_x(sp, batch, instance=i)).pin_memory() for i in range(4)]
        y_h = [torch.empty((batch, sp.m), dtype=torch.float32).pin_memory() for _ in range(4)]
        with torch.cuda.stream(self.stream):
            for s in range(8):
                tcm.qlinear_forward_host(self.handles[s % self.n_inst], x_h[s % 4], y_h[s % 4], stream=self.stream)

        def body():
            for s in range(steps):
                tcm.qlinear_forward_host(self.handles[s % self.n_inst], x_h[s % 4], y_h[s % 4], stream=self.stream)
        return self.timed(body)

    def cold_call_us(self):
        """Latency of one forward whose code words are not in L2 (a buffer of
        twice the L2 size is written first), median of 3; None if it fails."""
        torch = self.torch
        try:
            flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            out = []
            with torch.cuda.stream(self.stream):
                for i in range(3):
                    flush.zero_()
                    ev0.record(self.stream)
                    j = i % self.n_inst
                    self.tcm.qlinear_forward(self.handles[j], self.xs[j], self.ys[j])
                    ev1.record(self.stream)
                    torch.cuda.synchronize()
                    out.append(ev0.elapsed_time(ev1) * 1e3)
            del flush
            return statistics.median(out)
        except Exception:
            return None

    def close(self):
        for h in self.handles:
            self.tcm.qlinear_destroy(h)
        self.handles = []
        self.graphs = []


def n_instances(sp, override=None):
    n = int(min(512, max(1, math.ceil(4 * L2_BYTES / sp.stream_bytes))))
    return max(1, min(n, override)) if override else n


MAIN_TIMING = ("the main kernel alone (qlinear_launch_main_kernel), {} launches back to back over the rotating "
               "instances ({:.2f} s, after a 0.5 s idle pause), CUDA events on the launching stream around the graph "
               "replays")


def roofline(sp, batch, kern_s, pk, pk_kind, clk_mhz, sms, timing, burst_gemm, chain_s=None):
    """The main kernel's roofline: HBM on the algorithmic bytes (decode-GEMV,
    batch <= 8) or the dense tensor rate (tensor-core GEMM), plus the issue
    fraction from the committed instruction counters when they are current."""
    weights = sp.m * sp.n
    if batch <= GEMV_MAX_BATCH:
        key = f"gemv_{sp.name}_b{batch}"
        alg_bytes = sp.stream_bytes + batch * sp.n * 2 + batch * sp.m * 4
        achieved = alg_bytes / kern_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "kernel": "trellis_gemv_kernel (fused trellis decode + MMA)",
                "peak_kind": pk_kind + " hbm_gbs (copy)", "alg_bytes_per_launch": alg_bytes}
    else:
        key = f"gemm_{sp.name}_b{batch}"
        flops = 2.0 * sp.m * sp.n * batch
        achieved = flops / kern_s / 1e12
        peak = pk["bf16_tflops"] if burst_gemm else pk["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "kernel": "trellis_gemm_kernel (trellis decode into tensor memory + tcgen05 MMA, fp16 in, "
                          "fp32 accumulate)",
                "peak_kind": pk_kind + (" bf16_tflops (burst: the kernel is timed in a loop of under a second)"
                                        if burst_gemm else " bf16_tflops_sustained (a loop of a second or more)")
                + "; the fp16 dense rate equals the bf16 one",
                "alg_flops_per_launch": flops}
    c = _counters(key)
    roof["traffic"] = c["dram_bytes"] if c else None
    roof["kernel_us"] = kern_s * 1e6
    roof["timing"] = timing
    if chain_s is not None:
        roof["kernel_us_in_forward"] = chain_s * 1e6
        roof["in_forward_note"] = ("CUDA events around the kernel inside the forwards (a separate graph replay); "
                                   "they serialise its programmatically dependent launch, so this includes the "
                                   "launch gap: an upper bound")
    if c and c.get("warp_inst"):
        roof["warp_inst_per_launch"] = c["warp_inst"]
        roof["lane_inst_per_weight"] = c["thread_inst"] / weights
        roof["issue_frac"] = c["warp_inst"] / kern_s / (sms * 4 * clk_mhz * 1e6)
        roof["issue_note"] = (f"warp instructions per launch (ncu) / kernel time / ({sms} SMs x 4 issue slots x "
                              f"{clk_mhz:.0f} MHz sampled)")
    else:
        roof["issue_frac"] = None
    return roof


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch N>1 with torch.distributed.run")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    import trellis_coded_matmul_b200 as tcm

    sms = torch.cuda.get_device_properties(local).multi_processor_count
    stream = torch.cuda.Stream()
    pk, pk_kind = peaks()
    sp = wl.WORKLOADS[args.workload]
    batch = args.batch or sp.batches[0]
    n_inst = n_instances(sp, args.instances)
    r = Runner(torch, tcm, dist, world, rank, stream, sp, batch, n_inst)

    clocks = ClockSampler(local)
    secs = r.throughput(args.steps, args.warmup)
    clk = clocks.stop()
    launches_per_step = tcm.qlinear_info(r.handles[0])["last_launches"]
    # The main kernel's duration: launched alone, back to back (the roofline's
    # denominator); and CUDA events around it inside the forwards (an upper
    # bound: they serialise its programmatically dependent launch).
    kern_chain_s, prof_steps, prof_secs = r.kernel_seconds(args.steps)
    kern_s, kern_launches, kern_total = r.main_kernel_seconds(args.steps)
    if world > 1:
        secs, kern_s, kern_chain_s = max_over_ranks([secs, kern_s, kern_chain_s], "cuda")
    e2e = None
    if not args.no_e2e:
        e2e_steps = min(args.steps, 2000)
        e2e_s = r.e2e(e2e_steps)
        if world > 1:
            e2e_s = max_over_ranks([e2e_s], "cuda")[0]
        e2e = {"value": job_tokens_per_s(world, e2e_steps, batch, e2e_s), "unit": "tokens/s",
               "h2d_bytes_per_step": batch * sp.n * 2, "d2h_bytes_per_step": batch * sp.m * 4,
               "steps": e2e_steps}
    cold = r.cold_call_us() if rank == 0 else None  # rank 0 only, no collective inside
    r.close()
    clk_mhz = (clk or {}).get("sm_mhz") or 1965.0

    # every benchmark configuration, each on its own rotating instances
    per_config = None
    if not args.no_per_config and not args.instances:
        per_config = []
        clocks_pc = ClockSampler(local)
        for name, b in PER_CONFIG:
            spc = wl.WORKLOADS[name]
            ni = n_instances(spc)
            rc = Runner(torch, tcm, dist, world, rank, stream, spc, b, ni)
            steps_c = max(args.steps, 2 * ni, 200)
            s_c = rc.throughput(steps_c, max(args.warmup, ni))
            launches_c = tcm.qlinear_info(rc.handles[0])["last_launches"]
            kc_chain, ps, pss = rc.kernel_seconds(steps_c)
            k_c, kl, k_total = rc.main_kernel_seconds(steps_c)
            timing_c = MAIN_TIMING.format(kl, k_total)
            if world > 1:
                s_c, k_c, kc_chain = max_over_ranks([s_c, k_c, kc_chain], "cuda")
            rc.close()
            per_config.append({"workload": name, "batch": b, "steps": steps_c, "instances": ni,
                               "ms_per_step": s_c / steps_c * 1e3,
                               "tokens_per_s": job_tokens_per_s(world, steps_c, b, s_c),
                               "stream_gbs_step": spc.stream_bytes * steps_c * world / s_c / 1e9,
                               "launches_per_step": launches_c,
                               "roofline": roofline(spc, b, k_c, pk, pk_kind, clk_mhz, sms, timing_c,
                                                    burst_gemm=k_total < 1.0, chain_s=kc_chain)})
        clk_pc = clocks_pc.stop()
        per_config.append({"clocks": clk_pc, "note": f"issue fractions use the headline run's median SM clock "
                                                      f"({clk_mhz:.0f} MHz)"})

    line = None
    if rank == 0:
        value = job_tokens_per_s(world, args.steps, batch, secs)
        timing = MAIN_TIMING.format(kern_launches, kern_total)
        roof = roofline(sp, batch, kern_s, pk, pk_kind, clk_mhz, sms, timing, burst_gemm=kern_total < 1.0,
                        chain_s=kern_chain_s)
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
                "config": config_dict(sp, batch, n_inst),
                "hbm_gbs_step": sp.stream_bytes * args.steps * world / secs / 1e9,
                "cold_call_us": cold,
                "roofline": roof,
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clk, "e2e": e2e, "per_config": per_config}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(sp, batch)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.record_counters:
        record_counters(*args.record_counters)
        return 0
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", "29517", __file__] + sys.argv[1:]
        return subprocess.call(cmd)
    if args.impl == "reference":
        return run_reference(args)
    if args.encode:
        return run_encode(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
