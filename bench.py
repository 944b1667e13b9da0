"""Benchmark of the Q4_K / Q8_0 dequant GEMV on B200 (one JSON line on stdout, rank 0).

Headline (value): effective HBM GB/s of one Q4_K GEMV y = dequant(W) . x at B = 1 on the FFN gate
shape N=17408, K=5120 of a 27B-class hybrid decoder (weight + x + y bytes / time).  A step is one
such call; the weights rotate over enough distinct device copies that every step reads them from
HBM (the copies together exceed 4x the L2).  Steps are replayed from CUDA graphs and timed with
CUDA events on the launching stream.  The same line carries B = 8 on the same tensor, every other
workload of the suite (per call: us, GB/s, fraction of the measured HBM copy bandwidth), the
end-to-end number through the Python API with host buffers, the roofline of the kernel, clocks
sampled during the timed region, and the CPU oracle's throughput on a bounded sample.

--impl reference times the CPU oracle (the plain C dequant + fp64 dot) instead, on the same
metric and workload, each step a bounded sample of rows.

Multi-GPU: the GEMV does not shard across GPUs here (replicas only): each rank runs its own copy
of the workload, the timed region is bracketed by barriers, its time is the max over ranks and
value = all ranks' bytes / that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from quant_dequant_gemv_q4_b200 import synth  # noqa: E402

METRIC = "Q4_K GEMV effective HBM GB/s and % of B200 HBM roofline (\u00b5s/call), B=1 and B=8"
UNIT = "GB/s"
HEADLINE = synth.Gemv("ffn_gate", synth.Q4_K, 17408, 5120, 1, 0)
HEADLINE_B8 = synth.Gemv("ffn_gate_b8", synth.Q4_K, 17408, 5120, 8, 0)
HEADLINE_B16 = synth.Gemv("ffn_gate_b16", synth.Q4_K, 17408, 5120, 16, 0)
HEADLINE_SEED = 4  # the batched-verify workload's seed
FALLBACK_HBM_GBS = 6650.0


# The sources the headline's CUDA-core kernel (rows_gemv_kernel) is built and launched from: its
# device code and the host planner/launcher.  The tensor-core kernel's file (qg_mma.cuh) and the
# host packer are not among them, so a change there leaves the headline's DRAM capture valid.
ROWS_KERNEL_FILES = ("qg_api.cu", "qg_device.cuh", "qg_rows.cuh")
MMA_KERNEL_FILES = ROWS_KERNEL_FILES + ("qg_codes.cuh", "qg_mma.cuh")  # the B >= 2 tensor-core kernel
UMMA_KERNEL_FILES = ROWS_KERNEL_FILES + ("qg_codes.cuh", "qg_umma.cuh")  # the tcgen05 variant


def kernel_source_hash(files=None) -> str:
    """sha256 (16 hex digits) of the library's CUDA/C++ sources, or of the named ones only."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quant_dequant_gemv_q4_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".cpp", ".h")) and (files is None or f in files):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def bench_config(world: int) -> dict:
    """The workload both arms (this library and the CPU oracle) report on."""
    return {"workload": "ffn_gate Q4_K GEMV N=17408 K=5120 B=1, one call per step",
            "global_batch": 1, "seq_len": 1, "parallelism": f"replicas x{world}"}


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured", "raw": d}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback", "raw": None}


# ------------------------------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ------------------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_max(value: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_sum(value: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def aggregate(local_seconds: float, local_bytes: float, device) -> tuple[float, float]:
    """(max seconds over ranks, total bytes over ranks): a replica job's time and work."""
    return dist_max(local_seconds, device), dist_sum(local_bytes, device)


# ------------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="qg_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        maxp = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * maxp] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in loaded:
            for name, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": maxp,
                "samples": len(rows),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------------
# GPU measurement
# ------------------------------------------------------------------------------------------------
class CallSet:
    """Device inputs of a list of GEMV calls, replicated over R copies of the weights."""

    def __init__(self, calls, seed, device, l2_bytes, min_copies=2, max_copies=4096):
        import torch
        import quant_dequant_gemv_q4_b200 as qg
        self.qg = qg
        self.calls = list(calls)
        self.device = device
        wl = synth.Workload("bench", seed, tuple(self.calls))
        per_step = sum(c.weight_bytes for c in self.calls)
        self.copies = int(min(max_copies, max(min_copies, -(-4 * l2_bytes // per_step))))
        self.W, self.x, self.y, self.x_host = [], [], [], []
        for c in self.calls:
            W, x = wl.inputs(c)
            base = torch.from_numpy(W).to(device)
            self.W.append([base] + [base.clone() for _ in range(self.copies - 1)])
            self.x_host.append(x)
            self.x.append(torch.from_numpy(x.view(np.uint16)).to(device))
            self.y.append(torch.empty((c.N, c.B), dtype=torch.float32, device=device))
        self.bytes_per_step = sum(c.algorithmic_bytes for c in self.calls)
        self.weight_bytes_per_step = per_step

    def launch(self, r: int, stream, variant: int):
        for i, c in enumerate(self.calls):
            self.qg.qg_gemv_variant(self.W[i][r], c.fmt, c.N, c.K, self.x[i], c.B, self.y[i],
                                    stream, variant)

    def launches_per_step(self, variant: int) -> int:
        """Kernels one step launches (a split-K call of the DIRECT kernel adds its second pass;
        the streaming kernels add the K slices inside the same launch)."""
        import torch
        n = 0
        for i, c in enumerate(self.calls):
            self.qg.qg_gemv_variant(self.W[i][0], c.fmt, c.N, c.K, self.x[i], c.B, self.y[i],
                                    torch.cuda.current_stream(), variant)
            two = self.qg.qg_last_splits() > 1 and self.qg.qg_last_variant() == self.qg.QG_VARIANT_DIRECT
            n += 2 if two else 1
        torch.cuda.synchronize()
        return n


def time_callset(cs: CallSet, steps: int, warmup: int, variant: int, clocks: ClockSampler | None):
    """Time exactly `steps` steps (each: the call list on the next weight copy) from one CUDA
    graph; returns (seconds on this rank, ms per step).

    The graph holds `lead` untimed calls, the start event, the `steps` timed calls and the end
    event (event-record nodes, cudaEventRecordExternal), so the timed region opens while the GPU
    is already streaming: neither the graph's launch nor its upload (done by the warm-up replays,
    which run the whole graph) falls inside it, and every timed call is a steady-state call on a
    fresh weight copy.  The start event sits on a side branch forked after the last untimed call:
    it fires when that call completes, while the first timed call keeps its programmatic edge to
    it (its prologue may overlap the untimed call's tail, as every call's does in the chain).  The
    region is thus `steps` completion-to-completion intervals of the chain; the end event follows
    the last timed call's full completion."""
    import torch
    stream = torch.cuda.Stream(device=cs.device)
    R = cs.copies
    with torch.cuda.stream(stream):
        for r in range(min(R, 2)):
            cs.launch(r, stream, variant)  # allocates the workspace of this stream
    stream.synchronize()
    lead = max(R, 8)
    start = torch.cuda.Event(enable_timing=True, external=True)
    end = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=cs.device)
    with torch.cuda.graph(graph, stream=stream):
        for i in range(lead):
            cs.launch(i % R, stream, variant)
        side.wait_stream(stream)
        start.record(side)
        for i in range(steps):
            cs.launch((lead + i) % R, stream, variant)
        stream.wait_stream(side)
        end.record(stream)
    # warm-up: whole-graph replays until at least `warmup` steps have run (at least one replay,
    # which uploads the graph)
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-warmup // (lead + steps)))):
            graph.replay()
    stream.synchronize()
    ctx = clocks if clocks is not None else _null()
    with ctx:
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            graph.replay()
        stream.synchronize()
        torch.cuda.synchronize()
        barrier()
    secs = start.elapsed_time(end) / 1e3
    del graph
    return secs, secs * 1e3 / steps


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def time_gate_up(device, B: int, steps: int, warmup: int, l2_bytes: int) -> dict:
    """The fused FFN gate/up pair (two Q4_K 17408 x 5120 tensors on one x, h = silu(g) * u) per
    call, replayed from CUDA graphs over rotating copies of both tensors."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    N, K = HEADLINE.N, HEADLINE.K
    g_call = synth.Gemv("ffn_gate", synth.Q4_K, N, K, B, 0)
    u_call = synth.Gemv("ffn_up", synth.Q4_K, N, K, B, 1)
    wl = synth.Workload("gate_up", HEADLINE_SEED, (g_call, u_call))
    Wg, x = wl.inputs(g_call)
    Wu, _ = wl.inputs(u_call)
    pair_bytes = 2 * g_call.weight_bytes
    copies = int(max(2, -(-4 * l2_bytes // pair_bytes)))
    Wgs = [torch.from_numpy(Wg).to(device)]
    Wus = [torch.from_numpy(Wu).to(device)]
    for _ in range(copies - 1):
        Wgs.append(Wgs[0].clone())
        Wus.append(Wus[0].clone())
    xd = torch.from_numpy(x.view(np.uint16)).to(device)
    h = torch.empty((N, B), dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device=device)

    def launch(r):
        qg.qg_gemv_gate_up_silu(Wgs[r], Wus[r], synth.Q4_K, N, K, xd, B, h, stream)

    with torch.cuda.stream(stream):
        launch(0)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for r in range(copies):
            launch(r)
    reps = max(1, steps // copies)
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-warmup // copies))):
            graph.replay()
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(reps):
            graph.replay()
        b.record(stream)
    b.synchronize()
    secs = a.elapsed_time(b) / 1e3
    secs = dist_max(secs, device)
    calls = reps * copies
    nbytes = pair_bytes + 2 * K * B + 4 * N * B
    del graph
    return {"B": B, "us_per_call": round(secs * 1e6 / calls, 3),
            "gbs": round(nbytes * calls / secs / 1e9, 1),
            "bytes_per_call": nbytes, "calls": calls, "variant": qg.qg_last_variant(),
            "splits": qg.qg_last_splits()}


def time_e2e(cs: CallSet, steps: int, warmup: int, variant: int):
    """End to end through the public API with host activations: per step one qg_gemv_host call
    (pinned host x -> device, the GEMV, y -> pinned host, all on the stream); returns (seconds,
    h2d bytes/step, d2h bytes/step)."""
    import torch
    xh = [torch.from_numpy(x.view(np.uint16)).pin_memory() for x in cs.x_host]
    yh = [torch.empty(y.shape, dtype=torch.float32).pin_memory() for y in cs.y]
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    xp = [t.data_ptr() for t in xh]
    yp = [t.data_ptr() for t in yh]
    Wp = [[w.data_ptr() for w in ws] for ws in cs.W]
    L = cs.qg.lib()
    del variant  # qg_gemv_host takes the library's default kernel

    def step(r):
        for i, c in enumerate(cs.calls):
            rc = L.qg_gemv_host(Wp[i][r], c.fmt, c.N, c.K, xp[i], c.B, yp[i], sp)
            if rc != 0:
                raise RuntimeError(f"qg_gemv_host: {cs.qg.status_string(rc)}")

    for s in range(warmup):
        step(s % cs.copies)
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for s in range(steps):
        step(s % cs.copies)
    torch.cuda.synchronize()
    secs = time.perf_counter() - t0
    barrier()
    h2d = sum(x.nbytes for x in cs.x_host)
    d2h = sum(c.N * c.B * 4 for c in cs.calls)
    return secs, h2d, d2h


def time_latency(cs: CallSet, calls: int, variant: int) -> dict:
    """Per-call latency distribution: eager launches on one stream with a CUDA-event pair around
    each call (on rotating weight copies, so every call reads HBM); median, p10 and p90 in us.
    A call here is not overlapped with its neighbours, unlike the graph-replayed chain."""
    import torch
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(calls)]
    for r in range(min(cs.copies, 3)):
        cs.launch(r, stream, variant)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        cs.launch(i % cs.copies, stream, variant)
        b.record(stream)
    torch.cuda.synchronize()
    us = np.array([a.elapsed_time(b) * 1e3 for a, b in evs])
    return {"median": round(float(np.median(us)), 3), "p10": round(float(np.percentile(us, 10)), 3),
            "p90": round(float(np.percentile(us, 90)), 3), "calls": calls,
            "how": "eager launches, a CUDA-event pair around each call on the launching stream"}


def hbm_probe(device, nbytes=1 << 30, reps=10):
    """Copy (read+write) and read-only bandwidth of this library's probe kernels, best of reps."""
    import torch
    import quant_dequant_gemv_q4_b200 as qg
    src = torch.empty(nbytes, dtype=torch.uint8, device=device)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    out = torch.zeros(4096, dtype=torch.int32, device=device)
    s = torch.cuda.current_stream()
    res = {}
    for name, fn, moved in [("copy", lambda: qg.qg_hbm_copy(src, dst, nbytes, s), 2 * nbytes),
                            ("read", lambda: qg.qg_hbm_read(src, nbytes, out, s), nbytes)]:
        fn()
        torch.cuda.synchronize()
        best = 1e9
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            best = min(best, a.elapsed_time(b) / 1e3)
        res[name + "_gbs"] = round(moved / best / 1e9, 1)
    del src, dst
    torch.cuda.empty_cache()
    return res


def load_traffic(rows_hash: str) -> dict | None:
    """DRAM bytes per launch of the headline kernel from a committed ncu capture summary, if it
    was taken on the current sources of that kernel (same hash of ROWS_KERNEL_FILES); else
    None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("rows_kernel_hash") != rows_hash:
        return None
    return d


# ------------------------------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ------------------------------------------------------------------------------------------------
def oracle_sample_rate(call: synth.Gemv, seed: int, seconds: float):
    """Time the oracle on rows of `call` (wrapping around the matrix) for about `seconds`; returns
    (GB/s on the call's algorithmic bytes per row, rows timed, seconds, bytes)."""
    import oracle
    oracle.build()
    wl = synth.Workload("cpu", seed, (call,))
    W, x = wl.inputs(call)
    row_bytes = call.weight_bytes // call.N
    rows, done_rows, t_total = 8, 0, 0.0
    while t_total < seconds:
        r0 = done_rows % call.N
        sel = (np.arange(rows) + r0) % call.N
        t0 = time.perf_counter()
        oracle.gemv(W, call.fmt, call.N, call.K, x, call.B, rows=sel)
        t_total += time.perf_counter() - t0
        done_rows += rows
        rows = min(rows * 2, 4096)
    nbytes = done_rows * (row_bytes + 4 * call.B) + 2 * call.K * call.B
    return nbytes / t_total / 1e9, done_rows, t_total, nbytes


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# The workload calls the oracle is timed on per config (whole calls: median of 3 runs, 5 for the
# small attention call), on the same seeded inputs as the GPU table.
ORACLE_CONFIG_CALLS = (
    ("q4k_attn_kv_1024x5120", 5),
    ("q4k_ssm_qkv_10240x5120", 3),
    ("q4k_ffn_pair_b1", 3),
    ("mixed_q8_0_q4k_b1", 3),
    ("q4k_ffn_gate_verify", 3),
)


def oracle_config_table() -> dict:
    """The oracle per call of every workload config: median wall time of whole calls (single
    thread), us/call and GB/s on the call's algorithmic bytes."""
    import oracle
    oracle.build()
    out = {}
    for name, runs in ORACLE_CONFIG_CALLS:
        wl = synth.WORKLOADS[name]
        for c in wl.calls:
            W, x = wl.inputs(c)
            ts = []
            for _ in range(runs):
                t0 = time.perf_counter()
                oracle.gemv(W, c.fmt, c.N, c.K, x, c.B)
                ts.append(time.perf_counter() - t0)
            t = statistics.median(ts)
            out[f"{name}/{c.name}"] = {"us_per_call": round(t * 1e6, 1),
                                       "gbs": round(c.algorithmic_bytes / t / 1e9, 4), "runs": runs}
    return out


def run_reference(args):
    world, rank, _ = dist_env()
    if world > 1:
        # every rank joins the launcher's rendezvous once (gloo: no GPU work on this arm); rank 0
        # alone then times the oracle and prints
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("gloo", timeout=timedelta(seconds=300))
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    call = HEADLINE
    wl = synth.Workload("ref", HEADLINE_SEED, (call,))
    W, x = wl.inputs(call)
    row_bytes = call.weight_bytes // call.N
    # rows per step so that warmup + steps take about a minute
    t0 = time.perf_counter()
    oracle.gemv(W, call.fmt, call.N, call.K, x, call.B, rows=np.arange(64))
    per_row = (time.perf_counter() - t0) / 64
    total = max(1, args.steps + args.warmup)
    rows = int(max(1, min(call.N, args.ref_seconds / total / per_row)))

    def step(s):
        sel = (np.arange(rows) + s * rows) % call.N
        oracle.gemv(W, call.fmt, call.N, call.K, x, call.B, rows=sel)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(s)
    secs = time.perf_counter() - t0
    step_bytes = rows * (row_bytes + 4 * call.B) + 2 * call.K * call.B
    value = step_bytes * args.steps / secs / 1e9
    sample = (f"{rows} of {call.N} rows of the Q4_K N=17408 K=5120 B=1 GEMV per step "
              f"(dequant + fp64 dot, single-threaded C)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3 / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle dot; fp32 weights)",
        "data": "synthetic (seeded Q4_K bytes, x ~ N(0,1) fp16)",
        "config": bench_config(world),
        "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": round(value, 4),
                         "unit": UNIT},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ncu_case(args):
    """The headline tensor, one copy on the device: 3 launches at B=1, then 3 at B=8.  With
    --ncu-fmt 13, 14 or 23 the same tensor shape in Q5_K / Q6_K / IQ4_XS instead (3 launches at
    B=1, then 3 at B=8); --variant picks the kernel variant (0: the library's default, 5: the
    tcgen05 kernel)."""
    import torch
    from quant_dequant_gemv_q4_b200 import build as qbuild
    qbuild.build()
    import quant_dequant_gemv_q4_b200 as qg
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    calls = (HEADLINE, HEADLINE_B8)
    if args.ncu_fmt != synth.Q4_K:
        calls = tuple(synth.Gemv(f"ffn_gate_b{b}", args.ncu_fmt, HEADLINE.N, HEADLINE.K, b, 0)
                      for b in (1, 8))
    for call in calls:
        wl = synth.Workload("ncu", HEADLINE_SEED, (call,))
        W, x = wl.inputs(call)
        Wd = torch.from_numpy(W).to(device)
        xd = torch.from_numpy(x.view(np.uint16)).to(device)
        yd = torch.empty((call.N, call.B), dtype=torch.float32, device=device)
        s = torch.cuda.current_stream()
        for _ in range(3):
            qg.qg_gemv_variant(Wd, call.fmt, call.N, call.K, xd, call.B, yd, s, args.variant)
        torch.cuda.synchronize()
        del Wd, xd, yd
    print(json.dumps({"ncu_case": "done", "kernel_hash": kernel_source_hash(),
                      "rows_kernel_hash": kernel_source_hash(ROWS_KERNEL_FILES),
                      "mma_kernel_hash": kernel_source_hash(MMA_KERNEL_FILES),
                      "umma_kernel_hash": kernel_source_hash(UMMA_KERNEL_FILES)}), flush=True)
    return 0


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_replicas(n: int, argv: list[str]) -> int:
    """Run this script as n local ranks under torch.distributed.run (rendezvous on 127.0.0.1);
    returns the launcher's exit code.  Rank 0 prints the JSON line."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


# ------------------------------------------------------------------------------------------------
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="qg", choices=["qg", "reference"])
    ap.add_argument("--variant", type=int, default=0, help="QG_VARIANT_* (0 = library default)")
    ap.add_argument("--table-steps", type=int, default=4000)
    ap.add_argument("--no-table", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-cpu-configs", action="store_true",
                    help="skip the oracle's per-config table (whole calls of every config)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: CPU seconds the whole warm-up + timed run takes")
    ap.add_argument("--ncu-case", action="store_true",
                    help="launch the headline call 3x at B=1 then 3x at B=8 on one weight copy "
                         "and exit (the small case an ncu capture runs; nothing is timed)")
    ap.add_argument("--ncu-fmt", type=int, default=12,
                    help="--ncu-case format: 12 Q4_K (default), 13 Q5_K, 14 Q6_K, 23 IQ4_XS")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    # --gpus N > 1 started without a launcher: run N replica processes under torch.distributed.run
    # (one per GPU), each with these same arguments
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_replicas(args.gpus, sys.argv[1:] if argv is None else list(argv))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2

    if args.impl == "reference":
        return run_reference(args)
    if args.ncu_case:
        return run_ncu_case(args)

    import torch
    import torch.distributed as dist
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)
    from quant_dequant_gemv_q4_b200 import build as qbuild
    qbuild.build()
    import quant_dequant_gemv_q4_b200 as qg

    peaks = load_peaks()
    hbm = peaks["hbm_gbs"]
    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 126 << 20))

    # headline: B=1
    cs = CallSet([HEADLINE], HEADLINE_SEED, device, l2)
    launches = cs.launches_per_step(args.variant)
    variant_used = qg.qg_last_variant()
    sampler = ClockSampler(local)
    secs, ms_local = time_callset(cs, args.steps, args.warmup, args.variant, sampler)
    clocks = sampler.summary()
    secs_max, bytes_total = aggregate(secs, float(cs.bytes_per_step * args.steps), device)
    value = bytes_total / secs_max / 1e9
    per_launch_s = secs / (args.steps * launches)
    achieved = cs.bytes_per_step / launches / per_launch_s / 1e9
    khash = kernel_source_hash()
    rows_hash = kernel_source_hash(ROWS_KERNEL_FILES)
    traffic = load_traffic(rows_hash)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "traffic": (traffic or {}).get("bytes_per_launch"),
                "peak_source": f"{peaks['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peaks["source"] == "measured" else "fallback 6.65 TB/s"}

    # B = 8 on the same tensor
    cs8 = CallSet([HEADLINE_B8], HEADLINE_SEED, device, l2)
    steps8 = max(200, min(args.steps // 4, 20000))
    secs8, ms8 = time_callset(cs8, steps8, args.warmup, args.variant, None)
    secs8 = dist_max(secs8, device)
    b8 = {"us_per_call": round(secs8 * 1e6 / steps8, 3),
          "gbs": round(cs8.bytes_per_step * steps8 / secs8 / 1e9, 1),
          "frac_of_hbm": round(cs8.bytes_per_step * steps8 / secs8 / 1e9 / hbm, 4),
          "flops_tflops": round(2 * HEADLINE_B8.N * HEADLINE_B8.K * 8 * steps8 / secs8 / 1e12, 2),
          "steps": steps8}
    del cs8

    # B = 16 (verify width beyond 8: the tensor-core kernel's two 8-column tiles)
    cs16 = CallSet([HEADLINE_B16], HEADLINE_SEED, device, l2)
    secs16, _ = time_callset(cs16, steps8, args.warmup, args.variant, None)
    secs16 = dist_max(secs16, device)
    b16 = {"us_per_call": round(secs16 * 1e6 / steps8, 3),
           "gbs": round(cs16.bytes_per_step * steps8 / secs16 / 1e9, 1),
           "frac_of_hbm": round(cs16.bytes_per_step * steps8 / secs16 / 1e9 / hbm, 4),
           "splits": qg.qg_last_splits(), "steps": steps8}
    del cs16

    # the same tensor on the tcgen05 kernel (an explicit variant; the default kernels are the
    # CUDA-core one at B = 1 and the mma.sync one at B >= 2)
    tcgen05 = []
    for Bt, call in ((1, HEADLINE), (8, HEADLINE_B8), (16, HEADLINE_B16)):
        cst = CallSet([call], HEADLINE_SEED, device, l2)
        st_t = max(200, min(args.steps // 8, 4000))
        s_t, _ = time_callset(cst, st_t, args.warmup, qg.QG_VARIANT_TCGEN05, None)
        s_t = dist_max(s_t, device)
        tcgen05.append({"B": Bt, "us_per_call": round(s_t * 1e6 / st_t, 3),
                        "frac_of_hbm": round(cst.bytes_per_step * st_t / s_t / 1e9 / hbm, 4),
                        "splits": qg.qg_last_splits(), "steps": st_t})
        del cst
    torch.cuda.empty_cache()

    # the fused FFN gate/up pair (one launch, two weight streams, h = silu(g) * u)
    gate_up = []
    for Bg in (1, 8):
        r = time_gate_up(device, Bg, max(500, min(args.steps // 8, 20000)), args.warmup, l2)
        r["frac_of_hbm"] = round(r["gbs"] / hbm, 4)
        gate_up.append(r)
    torch.cuda.empty_cache()

    # every workload of the suite, per call
    table = {}
    if not args.no_table:
        for name, wl in synth.WORKLOADS.items():
            cst = CallSet(list(wl.calls), wl.seed, device, l2)
            st = max(args.table_steps, 3 * cst.copies)
            s_t, _ = time_callset(cst, st, args.warmup, args.variant, None)
            s_t = dist_max(s_t, device)
            per_call = {}
            for c in wl.calls:
                csc = CallSet([c], wl.seed, device, l2)
                s_c, _ = time_callset(csc, max(args.table_steps, 3 * csc.copies), args.warmup,
                                      args.variant, None)
                s_c = dist_max(s_c, device)
                n_c = max(args.table_steps, 3 * csc.copies)
                gbs = c.algorithmic_bytes * n_c / s_c / 1e9
                per_call[c.name] = {"N": c.N, "K": c.K, "B": c.B,
                                    "fmt": synth.FMT_NAMES[c.fmt],
                                    "us": round(s_c * 1e6 / n_c, 3), "gbs": round(gbs, 1),
                                    "frac": round(gbs / hbm, 4),
                                    "splits": qg.qg_last_splits()}
                del csc
            table[name] = {"us_per_step": round(s_t * 1e6 / st, 3),
                           "gbs": round(cst.bytes_per_step * st / s_t / 1e9, 1),
                           "calls": per_call, "copies": cst.copies}
            del cst
            torch.cuda.empty_cache()

    # per-call latency of isolated calls (not overlapped with their neighbours)
    latency = time_latency(cs, 200, args.variant)

    # end to end through the Python API with host buffers
    # (at least 500 steps after 20 warm-up steps, so a short --steps still reads the steady state)
    e2e_steps = max(min(args.steps, 3000), 500)
    s_e, h2d, d2h = time_e2e(cs, e2e_steps, max(min(args.warmup, 50), 20), args.variant)
    s_e = dist_max(s_e, device)
    e2e = {"value": round(cs.bytes_per_step * e2e_steps * world / s_e / 1e9, 2), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "us_per_step": round(s_e * 1e6 / e2e_steps, 2), "steps": e2e_steps,
           "via": "qg_gemv_host through the C ABI: pinned host x and y, the copies and the call on "
                  "one stream, one call per step, host clock around all steps"}
    probe = hbm_probe(device)
    del cs
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, rows, t, nb = oracle_sample_rate(HEADLINE, HEADLINE_SEED, args.cpu_seconds)
        cpu = {"value": round(rate, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{rows} rows ({rows / HEADLINE.N:.2f} passes, {nb / 1e6:.1f} MB) of the "
                         f"N=17408 K=5120 B=1 call in {t:.1f} s, single-threaded C oracle "
                         f"(dequant + fp64 dot)",
               "host_cores": os.cpu_count(), "host_cpu": host_cpu_model()}
        if not args.no_cpu_configs:
            cpu["per_config"] = oracle_config_table()

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs_max * 1e3 / args.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (Q4_K weights, f16 x, f32 accumulate)",
        "data": "synthetic (seeded Q4_K bytes with the workload's d/dmin/sc/m/q distributions, "
                "x ~ N(0,1) fp16)",
        "config": bench_config(world),
        "timing": {"l2": f"{cs_copies_note(HEADLINE, l2)}; L2 {l2 >> 20} MiB",
                   "how": "one CUDA graph per measurement: lead calls, a start-event node on a "
                          "side branch, exactly `steps` calls on rotating weight copies, an "
                          "end-event node; B=8 on the same tensor in 'b8'"},
        "latency_us": latency,
        "us_per_call": round(secs_max * 1e6 / args.steps, 3),
        "frac_of_hbm": round(value / world / hbm, 4),
        "variant": variant_used,
        "roofline": roofline,
        "b8": b8,
        "b16": b16,
        "tcgen05": tcgen05,
        "gate_up_silu": gate_up,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": args.steps * launches,
        "cpu_baseline": cpu,
        "hbm_probe": probe,
        "kernel_hash": khash,
        "rows_kernel_hash": rows_hash,
        "workloads": table,
    }
    print(json.dumps(line), flush=True)
    return 0


def cs_copies_note(call, l2):
    copies = max(2, -(-4 * l2 // call.weight_bytes))
    return (f"{copies} rotating weight copies ({copies * call.weight_bytes / 1e6:.0f} MB > 4x L2), "
            "so every step reads its weights from HBM")


if __name__ == "__main__":
    sys.exit(main())
