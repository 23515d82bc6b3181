"""Benchmark of the expert-routed quantized matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode|canvas|prefill|skewed] [--sweep] [--no-extras]

Default workload ("decode"): one MoE decode step for one token: the gate/up
projection (128 experts, top-8, k=2816, n=1408) followed by the down projection
(k=704, n=2816), both 4-bit affine with group 64, bf16 x, f32 out. Every step
uses fresh ids (8 distinct uniform experts), fresh x, and the next of 16 copies
of the expert weights (6.9 GB rotated, far above the 126 MB L2), so no step
finds its weights in L2. W untimed warm-up steps, then exactly K timed steps
replayed from a CUDA graph (up to 1000 steps per graph).

Metric: effective HBM GB/s = algorithmic bytes / time, algorithmic bytes = the
touched experts' packed codes + scales + biases read once, plus x and out.
The same JSON line also carries, measured outside the timed region:
  per_call     each decode projection alone (graphs of 100 calls, median of 5)
  roofline     the dominant kernel (gate/up) against MEASURED_PEAKS.json
  e2e          the decode step through the Python API with host buffers
  per_config   the canvas, prefill and skewed workloads (routing + tcgen05
               grouped GEMM): us/call, TFLOP/s, GB/s and roofline fractions
  sweep        decode with m = 1, 2, 4, 8 tokens per projection
  cpu_baseline the CPU oracle on a bounded sample of the decode step

--impl reference times the CPU oracle (the only reference there is) on a
bounded sample of the same workload. N > 1: independent replicas, one per GPU
(the operation has no exchange step), value = total bytes / max time; the
per_config and sweep entries are measured at N = 1 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/call; effective HBM GB/s (decode) and TFLOP/s (canvas/prefill) vs roofline"
N_LAYERS = 16
GRAPH_STEPS = 1000   # longest graph of timed steps (more steps replay it)
GRAPH_CALLS = 100    # calls per graph for the per-call figures
REPEATS = 5          # per-call figures: median of this many graph replays
# dram__bytes_read.sum + dram__bytes_write.sum of one gate/up launch of the decode
# kernel, from one ncu capture of it (cold L2): 17,876,992 B read, 0 B written
GATE_UP_DRAM_BYTES = 17876992
GATE_UP_TRAFFIC_NOTE = ("ncu capture of the third gate/up launch of `bench.py --probe decode --reps 4` "
                        "(gemv_aff4_rows<32, 3, 0>, cold L2): dram read 17,876,992 B, write 0 B")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------- setup

class Dist:
    def __init__(self, gpus):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if torch.cuda.is_available():
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, v: float) -> float:
        if not self.pg:
            return v
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def alg_bytes(P, ids_row_sets) -> float:
    """Algorithmic bytes of one call: touched experts' codes + scales (+ biases or
    scale2) read once, x read once, out written once."""
    from workloads.gen import FMT_AFFINE, FMT_CODEBOOK

    per_row = P.row_bytes + P.groups * (2 if P.fmt in (FMT_AFFINE, FMT_CODEBOOK) else 1)
    if P.fmt == FMT_AFFINE:
        per_row += P.groups * 2
    per_expert = P.n * per_row + (4 if P.fmt == 2 else 0)
    distinct = np.unique(ids_row_sets[ids_row_sets < P.num_experts]).size
    xb = P.m * P.k * (4 if P.x_dtype == 0 else 2)
    ob = P.R * P.n * (4 if P.out_dtype == 0 else 2)
    cb = (1 << P.bits) * 2 if P.fmt == FMT_CODEBOOK else 0
    return float(distinct * per_expert + xb + ob + cb)


def clocks_sampler(device_index: int):
    """Start nvidia-smi sampling SM clocks and throttle reasons every 200 ms."""
    try:
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        sel = ["--id=GPU-" + uuid] if uuid and not uuid.startswith("GPU-") else ["--id=" + uuid]
    except Exception:
        sel = []
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    try:
        return subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                text=True)
    except Exception:
        return None


def clocks_summary(proc):
    if proc is None:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
    proc.terminate()
    try:
        out, _ = proc.communicate(timeout=5)
    except Exception:
        proc.kill()
        out = ""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in out.strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for name, val in zip(names, f[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------------- our workload

class DecodeWorkload:
    """gate/up + down projections of one decode token, rotating weight copies.

    G sets of fresh ids (8 distinct uniform experts) and x rows; step s uses set
    s % G and weight copy s % N_LAYERS."""

    def __init__(self, G: int, seed: int = 2, pdl: bool = True):
        import moe_expert_routed_b200 as M
        from workloads.torch_io import to_device
        from workloads import config_problem
        from workloads.gen import bf16_bits, distinct_uniform_ids

        self.M = M
        self.projs = [config_problem("decode_gate_up"), config_problem("decode_down")]
        # launch modes of a step: gate/up as a programmatic dependent launch (it waits for
        # the previous kernel before reading anything); down also streams its weights
        # early, since its ids were ready before gate/up began
        self.launch = ("pdl", "early_weights") if pdl else (None, None)
        self.G = G
        rng = np.random.Generator(np.random.PCG64(seed + 100))
        self.layers = []
        for P in self.projs:
            base = to_device(P)
            copies = []
            for _ in range(N_LAYERS):
                copies.append({k: (v.clone() if k in ("packed", "scales", "aux") else v)
                               for k, v in base.items()})
            self.layers.append(copies)
        self.ids = [torch.from_numpy(distinct_uniform_ids(rng, G, 8, P.num_experts)
                                     .view(np.int32)).cuda() for P in self.projs]
        self.x = [torch.from_numpy(bf16_bits(rng.standard_normal((G, P.k), dtype=np.float32))
                                   .view(np.int16)).view(torch.bfloat16).cuda() for P in self.projs]
        self.out = [torch.empty((G, 8, P.n), dtype=torch.float32, device="cuda") for P in self.projs]
        # gated gate/up output: act(gate) * up, n/2 columns
        self.out_glu = torch.empty((G, 8, self.projs[0].n // 2), dtype=torch.float32, device="cuda")
        self.ws = [M.new_workspace(1, 8, P.num_experts) for P in self.projs]
        self.set_bytes = [
            [alg_bytes(P, self.ids[i][s].cpu().numpy().view(np.uint32)) for s in range(G)]
            for i, P in enumerate(self.projs)]

    def call(self, proj: int, s: int, act=None, launch=None):
        P = self.projs[proj]
        L = self.layers[proj][s % N_LAYERS]
        i = s % self.G
        self.M.qmm_id(self.x[proj][i:i + 1], self.ids[proj][i:i + 1], L["packed"], L["scales"],
                      L["aux"], n=P.n, group_size=P.group_size, bits=P.bits, fmt=P.fmt,
                      num_experts=P.num_experts, out=self.out_glu[i] if act else self.out[proj][i],
                      workspace=self.ws[proj], act=act, launch=launch)

    def step(self, s: int, projs=(0, 1), act=None, launch=None):
        """One step: the given projections of set s. launch None: the step's own
        launch modes for the full gate/up + down sequence, plain stream order for a
        single projection; otherwise that launch mode for every call."""
        full = tuple(projs) == (0, 1)
        for p in projs:
            self.call(p, s, act, launch if launch is not None else (self.launch[p] if full else None))

    def bytes(self, steps: int, projs=(0, 1), act=None) -> float:
        """Algorithmic bytes of steps 0..steps-1 (a gated output writes n/2 columns)."""
        b = 0.0
        for p in projs:
            b += sum(self.set_bytes[p][s % self.G] for s in range(steps))
            if act and p == 0:
                b -= steps * 8 * (self.projs[0].n // 2) * 4
        return b

    def capture(self, steps: int, projs=(0, 1), act=None, launch=None):
        return capture_graph(lambda s: self.step(s, projs, act, launch), steps)


def _cudart():
    """The CUDA runtime library torch itself uses (for cudaGraphUpload)."""
    import ctypes

    try:
        import nvidia.cuda_runtime as cr

        path = os.path.join(list(cr.__path__)[0], "lib", "libcudart.so.12")
        return ctypes.CDLL(path)
    except Exception:
        return ctypes.CDLL("libcudart.so.12")


def graph_upload(g) -> bool:
    """Upload an instantiated graph to the device (cudaGraphUpload) so that its
    first timed replay does not pay for it. False if the call is not available."""
    import ctypes

    try:
        rt = _cudart()
        rc = rt.cudaGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        return rc == 0
    except Exception:
        return False


def capture_graph(fn, calls: int, warm: int = 2):
    """CUDA graph of fn(0) .. fn(calls-1) on the current device; fn(0..warm-1) runs
    eagerly on a side stream first, outside the capture."""
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for i in range(min(warm, calls)):
            fn(i)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(calls):
            fn(i)
    torch.cuda.synchronize()
    return g


def time_graph(g, replays: int) -> float:
    """Seconds for `replays` replays of g, CUDA events on the current stream."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / 1e3


def per_call(g, calls: int, repeats: int = REPEATS) -> dict:
    """Median over `repeats` timed replays of a graph of `calls` calls (after one
    untimed replay): seconds per call, and every repeat's value."""
    g.replay()
    torch.cuda.synchronize()
    ts = [time_graph(g, 1) / calls for _ in range(repeats)]
    return {"s": statistics.median(ts), "repeats_us": [t * 1e6 for t in ts]}


def e2e_decode(W: DecodeWorkload, steps: int):
    """Through the public API with host buffers, pipelined the way a serving loop
    would run it: every step copies its own x rows and ids (both projections) in
    from pinned host memory on an input-copy stream, runs both projections
    (moe_expert_routed_b200.Plan, one per layer copy and projection, the step's
    launch modes) on the compute stream, and copies both outputs back to pinned
    host memory on an output-copy stream. Device buffers are double-buffered, so
    step s+1's input copy and step s-1's output copy overlap step s's kernels;
    events order each buffer's reuse. The steps are captured once in a CUDA graph
    and replayed."""
    M = W.M
    n = min(max(steps, 2), W.G)
    xb = [P.k * 2 for P in W.projs]
    ib = [W.ids[i][0].numel() * 4 for i in range(2)]
    offs, o = [], 0
    for b in xb + ib:
        offs.append(o)
        o += (b + 15) // 16 * 16
    blk = o
    hin = torch.zeros((n, blk), dtype=torch.uint8).pin_memory()
    for p in range(2):
        hin[:, offs[p]:offs[p] + xb[p]] = W.x[p][:n].cpu().contiguous().view(torch.uint8).reshape(n, -1)
        hin[:, offs[2 + p]:offs[2 + p] + ib[p]] = W.ids[p][:n].cpu().contiguous().view(torch.uint8).reshape(n, -1)
    nout = [8 * P.n for P in W.projs]
    hout = torch.empty((n, sum(nout)), dtype=torch.float32).pin_memory()
    din = [torch.empty(blk, dtype=torch.uint8, device="cuda") for _ in range(2)]
    dout_all = [torch.empty(sum(nout), dtype=torch.float32, device="cuda") for _ in range(2)]
    dx = [[d[offs[p]:offs[p] + xb[p]].view(torch.bfloat16).view(1, W.projs[p].k) for p in range(2)] for d in din]
    did = [[d[offs[2 + p]:offs[2 + p] + ib[p]].view(torch.int32).view(1, -1) for p in range(2)] for d in din]
    dout = [[d[:nout[0]].view(1, 8, W.projs[0].n), d[nout[0]:].view(1, 8, W.projs[1].n)] for d in dout_all]
    h2d = sum(xb) + sum(ib)
    d2h = sum(nout) * 4
    plans = [[M.Plan(L["packed"], L["scales"], L["aux"], m=1, k=P.k, n=P.n, group_size=P.group_size,
                     bits=P.bits, fmt=P.fmt, n_expert_used=8, num_experts=P.num_experts,
                     x_dtype=torch.bfloat16, out_dtype=torch.float32, workspace=W.ws[p],
                     launch=W.launch[p]) for L in W.layers[p]] for p, P in enumerate(W.projs)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_steps(count):
        comp = torch.cuda.current_stream()
        done = [None] * count
        copied = [None] * count
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for s in range(count):
            b = s % 2
            with torch.cuda.stream(s_in):
                if s >= 2:
                    s_in.wait_event(done[s - 2])      # step s-2's kernels no longer read din[b]
                din[b].copy_(hin[s % n], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            comp.wait_event(ready)
            if s >= 2:
                comp.wait_event(copied[s - 2])        # dout[b] of step s-2 has been copied out
            plans[0][s % N_LAYERS](dx[b][0], did[b][0], dout[b][0], comp)
            plans[1][s % N_LAYERS](dx[b][1], did[b][1], dout[b][1], comp)
            done[s] = torch.cuda.Event()
            done[s].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[s])
                hout[s % n].copy_(dout_all[b], non_blocking=True)
                copied[s] = torch.cuda.Event()
                copied[s].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run_steps(2)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_steps(n)
    torch.cuda.synchronize()
    reps = max(1, (steps + n - 1) // n)
    g.replay()
    torch.cuda.synchronize()
    secs = time_graph(g, reps)
    # the last replay's host outputs: the results of steps 0..n-1
    got = hout.clone()
    del g
    per_step_bytes = W.bytes(n) / n
    return secs, reps * n, f"CUDA graph of {n} pipelined steps replayed {reps}x", per_step_bytes, h2d, d2h, got


# ------------------------------------------------------------------- oracle

def oracle_decode_sample(budget_s: float = 12.0):
    """CPU oracle on a bounded sample of the decode step: every output of the
    gate/up and down projections of one token (both full calls), repeated until
    the time budget is used. Returns (GB/s in the metric's unit, seconds, threads,
    sample description)."""
    import oracle
    from workloads import config_problem

    projs = [config_problem("decode_gate_up"), config_problem("decode_down")]
    threads = oracle.default_threads()
    nbytes, secs, calls = 0.0, 0.0, 0
    while secs < budget_s or calls < 2:
        for P in projs:
            pairs = np.repeat(np.arange(P.R), P.n)
            cols = np.tile(np.arange(P.n), P.R)
            t0 = time.perf_counter()
            oracle.qmm_id_sample(P, pairs, cols, nthreads=threads)
            secs += time.perf_counter() - t0
            nbytes += alg_bytes(P, P.ids.reshape(-1))
            calls += 1
        if secs > 4 * budget_s:
            break
    return nbytes / secs / 1e9, secs, threads, (
        f"{calls // 2} full decode steps (gate/up + down, m=1, 8 pairs, all outputs), "
        f"{secs:.1f} s on {threads} threads")


def oracle_single_thread():
    """The oracle on one host thread: one tiny call and one full decode step."""
    import oracle
    from workloads import config_problem

    res = {}
    P = config_problem("tiny")
    t0 = time.perf_counter()
    oracle.qmm_id(P, nthreads=1)
    res["tiny_ms_per_call"] = (time.perf_counter() - t0) * 1e3
    secs, nbytes = 0.0, 0.0
    for name in ("decode_gate_up", "decode_down"):
        P = config_problem(name)
        t0 = time.perf_counter()
        oracle.qmm_id(P, nthreads=1)
        secs += time.perf_counter() - t0
        nbytes += alg_bytes(P, P.ids.reshape(-1))
    res["decode_step_ms"] = secs * 1e3
    res["decode_step_GB_per_s"] = nbytes / secs / 1e9
    return res


# --------------------------------------------------------------------- main

def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import oracle
    from workloads import config_problem

    projs = [config_problem("decode_gate_up"), config_problem("decode_down")]
    threads = oracle.default_threads()
    # one step = a bounded sample: all 8 pairs x every 8th output column of both projections
    samples = []
    for P in projs:
        cols = np.arange(0, P.n, 8)
        samples.append((P, np.repeat(np.arange(P.R), cols.size), np.tile(cols, P.R),
                        alg_bytes(P, P.ids.reshape(-1)) * cols.size / P.n))
    for _ in range(args.warmup):
        for P, pr, cl, _b in samples:
            oracle.qmm_id_sample(P, pr, cl, nthreads=threads)
    t0 = time.perf_counter()
    nbytes = 0.0
    for _ in range(args.steps):
        for P, pr, cl, b in samples:
            oracle.qmm_id_sample(P, pr, cl, nthreads=threads)
            nbytes += b
    secs = time.perf_counter() - t0
    value = nbytes / secs / 1e9
    sample = "every 8th output column of the gate/up and down calls of one decode token (8 pairs)"
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "decode step m=1: gate/up (E128 top8 k2816 n1408) + down (k704 n2816), "
                               "affine 4-bit g64, bf16 x, f32 out", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_per_call(W: DecodeWorkload) -> dict:
    """Per-call figures of the decode projections: each from a CUDA graph of
    GRAPH_CALLS calls (fresh ids and x per call, rotated weight copies), the median
    of REPEATS timed replays.
      gate_up, down      one projection, calls in plain stream order (each waits
                         for the previous call's completion, launch gap included)
      gate_up_pdl        gate/up calls as programmatic dependents of the previous
                         call (each still waits for it before reading anything)
      gate_up_silu       gate/up with the SiLU-gated epilogue (n/2 outputs)
      step               gate/up + down with the step's launch modes"""
    res = {}
    G = GRAPH_CALLS
    for name, projs, act, launch in (("gate_up", (0,), None, None), ("gate_up_pdl", (0,), None, "pdl"),
                                     ("down", (1,), None, None), ("down_pdl", (1,), None, "pdl"),
                                     ("gate_up_silu", (0,), "silu", None), ("step", (0, 1), None, None)):
        g = W.capture(G, projs, act, launch)
        r = per_call(g, G)
        del g
        b = W.bytes(G, projs, act) / G
        res[name] = {"us_per_call": r["s"] * 1e6, "GB_per_s": b / r["s"] / 1e9,
                     "algorithmic_bytes": b, "repeats_us": r["repeats_us"]}
    return res


def grouped_tile_rows(P) -> int:
    """Tile height of the grouped GEMM for this call (as the library picks it):
    256 pairs (128 with f32 x) when experts hold ~96+ pairs on average, else 64.
    Only sizes the routing prologue's tile list when the prologue is timed alone."""
    if P.R >= 96 * P.num_experts:
        return 128 if P.x_dtype == 0 else 256
    return 64


def w4a4_entry(pk: dict) -> dict:
    """The prefill workload with W4A4 (x quantised per token to NVFP4 first, then the
    block-scaled MMA; moe_qmm_id_w4a4): per-call time from a CUDA graph of GRAPH_CALLS
    calls (median of REPEATS replays), and the activation quantisation alone timed
    the same way."""
    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.torch_io import to_device

    P = config_problem("prefill")
    d = to_device(P)
    ws = torch.zeros(M.workspace_bytes_w4a4(P.m, P.k, P.n_expert_used, P.num_experts), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((P.m, P.n_expert_used, P.n), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((P.m, P.k // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((P.m, P.k // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(P.m, dtype=torch.float32, device="cuda")
    xhat = torch.empty((P.m, P.k), dtype=torch.float32, device="cuda")
    L = M.lib()

    def call(_i):
        M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                      bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out, workspace=ws)

    def quant(_i):
        st = L.moe_quantize_act_nvfp4(d["x"].data_ptr(), P.m, P.k, 1, codes.data_ptr(), scales.data_ptr(),
                                      g.data_ptr(), xhat.data_ptr(), torch.cuda.current_stream().cuda_stream)
        if st != 0:
            raise RuntimeError(f"moe_quantize_act_nvfp4: status {st}")

    call(0)
    torch.cuda.synchronize()
    if M.poll_error(ws) != 0:
        raise RuntimeError("prefill with W4A4: device error word set")
    gc = capture_graph(call, GRAPH_CALLS)
    rc = per_call(gc, GRAPH_CALLS)
    del gc
    gq = capture_graph(quant, GRAPH_CALLS)
    rq = per_call(gq, GRAPH_CALLS)
    del gq
    ids = P.ids.reshape(-1)
    flops = 2.0 * int((ids < P.num_experts).sum()) * P.n * P.k
    us = rc["s"] * 1e6
    tf = flops / us / 1e6
    # the block-scaled fp4 MMA's peak: the measured bf16 peak times the nominal dense
    # ratio of the two (9 / 2.25 PFLOP/s per GPU)
    fp4_peak = 4.0 * pk["bf16_tflops"]
    ent = {
        "workload": "prefill with W4A4: x quantised per token to NVFP4 (E2M1 codes, E4M3 scales per 16, f32 "
                    "per-token scale), then the block-scaled tensor-core MMA (kind::mxf4nvf4) on the codes of "
                    "both operands",
        "us_per_call": us, "quantize_us": rq["s"] * 1e6, "TFLOP_per_s": tf,
        "gpu_launches_per_call": 5,  # quantisation; routing histogram, scan, scatter; the block-scaled GEMM
        "roofline": {"bound": "tensor", "achieved": tf, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": tf / fp4_peak, "bf16_frac": tf / pk["bf16_tflops"],
                     "peak_source": pk["source"] + " bf16_tflops x 4 (nominal dense fp4 / bf16 ratio)"},
        "repeats_us": rc["repeats_us"],
        "timing": f"CUDA graph of {GRAPH_CALLS} calls, median of {REPEATS} replays",
    }
    del d, out, ws, codes, scales, g, xhat
    torch.cuda.empty_cache()
    return ent


def grouped_entry(name: str, pk: dict) -> dict:
    """One grouped-path workload (routing prologue + tcgen05 grouped GEMM), inputs
    resident in HBM: per-call time from a CUDA graph of GRAPH_CALLS calls (median
    of REPEATS replays), the routing prologue alone timed the same way, and the
    GEMM time as their difference."""
    import ctypes

    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.torch_io import to_device

    P = config_problem(name)
    d = to_device(P)
    # sized for the gathered x rows: the GEMM loads each tile of x rows with one tensor copy
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts, k=P.k, x_dtype=d["x"].dtype)
    out_dt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float16}[P.out_dtype]
    out = torch.empty((P.m, P.n_expert_used, P.n), dtype=out_dt, device="cuda")

    def call(_i):
        M.qmm_id(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                 bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out, workspace=ws)

    T = grouped_tile_rows(P)
    R = P.R
    rbuf = [torch.empty(sz, dtype=torch.int32, device="cuda")
            for sz in (P.num_experts + 1, P.num_experts + 2, R, 2 * (R // T + P.num_experts + 1), 1)]
    ws_r = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    L = M.lib()

    def route_call(_i):
        st = L.moe_qmm_id_route(d["ids"].data_ptr(), P.m, P.n_expert_used, P.num_experts, T,
                                *[b.data_ptr() for b in rbuf], ws_r.data_ptr(), ws_r.numel() * ws_r.element_size(),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(f"moe_qmm_id_route: status {st}")

    call(0)
    torch.cuda.synchronize()
    if M.poll_error(ws) != 0:
        raise RuntimeError(f"{name}: device error word set")
    gc = capture_graph(call, GRAPH_CALLS)
    rc = per_call(gc, GRAPH_CALLS)
    del gc
    gr = capture_graph(route_call, GRAPH_CALLS)
    rr = per_call(gr, GRAPH_CALLS)
    del gr
    ids = P.ids.reshape(-1)
    valid = int((ids < P.num_experts).sum())
    flops = 2.0 * valid * P.n * P.k
    nbytes = alg_bytes(P, ids)
    us, route_us = rc["s"] * 1e6, rr["s"] * 1e6
    gemm_us = us - route_us
    t_tc = flops / (pk["bf16_tflops"] * 1e12) * 1e6
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9) * 1e6
    bound = "tensor" if t_tc >= t_hbm else "hbm"
    tf, gb = flops / us / 1e6, nbytes / us / 1e3
    tf_g, gb_g = flops / gemm_us / 1e6, nbytes / gemm_us / 1e3
    ent = {
        "workload": f"E{P.num_experts} top{P.n_expert_used} m{P.m} (R={P.R}) k{P.k} n{P.n}, "
                    f"{ {0: 'affine', 1: 'codebook', 2: 'nvfp4', 3: 'mxfp4'}[P.fmt]} {P.bits}-bit "
                    f"g{P.group_size}, {({0: 'f32', 1: 'bf16', 2: 'f16'})[P.x_dtype]} x, "
                    f"{({0: 'f32', 1: 'bf16', 2: 'f16'})[P.out_dtype]} out",
        "us_per_call": us, "TFLOP_per_s": tf, "GB_per_s": gb,
        "route_us": route_us, "gemm_us": gemm_us,
        "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
        "ideal_us": {"tensor": t_tc, "hbm": t_hbm},
        "roofline": {"bound": bound,
                     "achieved": tf if bound == "tensor" else gb,
                     "peak": pk["bf16_tflops"] if bound == "tensor" else pk["hbm_gbs"],
                     "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                     "frac": (tf / pk["bf16_tflops"]) if bound == "tensor" else (gb / pk["hbm_gbs"]),
                     "tensor_frac": tf / pk["bf16_tflops"], "hbm_frac": gb / pk["hbm_gbs"],
                     "gemm_tensor_frac": tf_g / pk["bf16_tflops"], "gemm_hbm_frac": gb_g / pk["hbm_gbs"],
                     "peak_source": pk["source"] + " (bf16_tflops burst, hbm_gbs copy)"},
        "repeats_us": rc["repeats_us"], "route_repeats_us": rr["repeats_us"],
        "timing": f"CUDA graph of {GRAPH_CALLS} calls, median of {REPEATS} replays; routing prologue alone "
                  f"the same way; gemm_us = call - routing (the x pre-pass kernels and the GEMM)",
        "l2": f"weights {P.packed.nbytes / 1e6:.0f} MB + x {P.x.nbytes / 1e6:.0f} MB (> L2 126 MB)",
        "gpu_launches_per_call": grouped_launches(P),
    }
    del d, out, ws, ws_r, rbuf
    torch.cuda.empty_cache()
    return ent


def grouped_launches(P) -> int:
    """Kernels of one grouped call with the k-aware workspace: the routing histogram,
    scan and scatter; for f32 x the gather of its split rows; for 16-bit x with
    256-pair tiles the f16 image of B (and, for bf16 x, the per-token factor
    before it); the GEMM."""
    R = P.m * P.n_expert_used
    n = 3 + 1
    if P.x_dtype == 0:
        n += 1
    elif R > 64 and R > 2 * P.num_experts and P.k % 8 == 0 and R >= 96 * P.num_experts:
        n += 2 if P.x_dtype == 1 else 1
    return n


def decode_sweep(pk: dict) -> list:
    """Decode with m = 1, 2, 4, 8 tokens (top-8 of 128 experts), gate/up and down
    projections separately: a CUDA graph of GRAPH_CALLS calls with fresh ids and x
    each call and N_LAYERS rotated weight copies, median of REPEATS replays.
    Effective GB/s counts the distinct experts each call touches (E[D] = 8, 15.5,
    29.1, 51.6 for uniform ids)."""
    import types

    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.gen import bf16_bits, distinct_uniform_ids
    from workloads.torch_io import to_device

    calls = GRAPH_CALLS
    rng = np.random.Generator(np.random.PCG64(77))
    rows = []
    for name in ("decode_gate_up", "decode_down"):
        P = config_problem(name)
        base = to_device(P)
        layers = [{k: base[k].clone() for k in ("packed", "scales", "aux")} for _ in range(N_LAYERS)]
        for m in (1, 2, 4, 8):
            ids = distinct_uniform_ids(rng, m * calls, 8, P.num_experts).reshape(calls, m, 8)
            x = bf16_bits(rng.standard_normal((calls, m, P.k), dtype=np.float32))
            d_ids = torch.from_numpy(ids.view(np.int32)).cuda()
            d_x = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            out = torch.empty((calls, m, 8, P.n), dtype=torch.float32, device="cuda")
            ws = M.new_workspace(m, 8, P.num_experts)
            Pm = types.SimpleNamespace(row_bytes=P.row_bytes, groups=P.groups, fmt=P.fmt, n=P.n, k=P.k,
                                       bits=P.bits, num_experts=P.num_experts, m=m, R=8 * m,
                                       x_dtype=P.x_dtype, out_dtype=P.out_dtype)
            nbytes = sum(alg_bytes(Pm, ids[c]) for c in range(calls)) / calls
            distinct = float(np.mean([np.unique(ids[c]).size for c in range(calls)]))

            def one(c):
                L = layers[c % N_LAYERS]
                M.qmm_id(d_x[c], d_ids[c], L["packed"], L["scales"], L["aux"], n=P.n,
                         group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                         out=out[c], workspace=ws)

            g = capture_graph(one, calls)
            r = per_call(g, calls)
            del g
            rows.append({"projection": name.replace("decode_", ""), "m": m, "distinct_experts": distinct,
                         "us_per_call": r["s"] * 1e6, "GB_per_s": nbytes / r["s"] / 1e9,
                         "frac_of_hbm": nbytes / r["s"] / 1e9 / pk["hbm_gbs"],
                         "TFLOP_per_s": 2.0 * 8 * m * P.n * P.k / r["s"] / 1e12})
        del base, layers
        torch.cuda.empty_cache()
    return rows


def run_ours(args, dist: Dist):
    import moe_expert_routed_b200 as M

    M.lib()  # fails loudly if the CUDA library is missing
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    dev = dist.local if dist.world > 1 else 0
    torch.cuda.set_device(dev)
    K, Wm = args.steps, args.warmup
    Gt = min(GRAPH_STEPS, K)
    W = DecodeWorkload(max(Gt, GRAPH_CALLS), pdl=not args.no_pdl)
    # the timed graph holds steps 0..Gt-1; uploaded to the device before warm-up so
    # that its first replay is a plain replay. When the K steps fit one graph, the
    # timing events are event nodes inside it, right before the first step's kernel
    # and after the last step's, so the timed region is the K steps on the device
    # without the host's graph-launch latency.
    ev0 = torch.cuda.Event(enable_timing=True, external=True)
    ev1 = torch.cuda.Event(enable_timing=True, external=True)

    def timed_step(s):
        if s == 0:
            ev0.record()
        W.step(s)
        if s == Gt - 1:
            ev1.record()

    g = capture_graph(timed_step, Gt)
    uploaded = graph_upload(g)
    warm_done = Wm
    for s in range(Wm):  # W untimed warm-up steps (the step's own calls, issued one by one)
        W.step(s)
    if not uploaded:
        g.replay()
        warm_done += Gt
    torch.cuda.synchronize()
    replays = max(1, K // Gt)
    steps_timed = replays * Gt
    sampler = clocks_sampler(dev) if dist.rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    dist.barrier()
    torch.cuda.synchronize()
    secs = time_graph(g, replays)
    torch.cuda.synchronize()
    in_graph = replays == 1
    if in_graph:
        secs = ev0.elapsed_time(ev1) / 1e3
    dist.barrier()
    clocks = clocks_summary(sampler) if dist.rank == 0 else None
    del g
    secs_max = dist.max(secs)
    bytes_total = dist.sum(W.bytes(Gt) * replays)
    value = bytes_total / secs_max / 1e9
    ms_per_step = secs_max / steps_timed * 1e3

    pk = peaks()
    pc = decode_per_call(W)
    # dominant kernel: the gate/up launch, timed alone (graph of gate/up calls, median
    # of repeats); DRAM traffic per launch from an ncu capture of that kernel
    achieved = pc["gate_up"]["GB_per_s"]
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": GATE_UP_DRAM_BYTES,
                "traffic_note": GATE_UP_TRAFFIC_NOTE,
                "algorithmic_bytes": pc["gate_up"]["algorithmic_bytes"],
                "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)",
                "kernel": "gemv_aff4_rows, gate/up launch (plain stream order; "
                          f"{pc['gate_up_pdl']['us_per_call']:.2f} us as programmatic dependents)",
                "frac_pdl": pc["gate_up_pdl"]["GB_per_s"] / pk["hbm_gbs"],
                "step_frac": value / dist.world / pk["hbm_gbs"]}
    e_secs, e_steps, e_mode, per_step_bytes, h2d, d2h, got = e2e_decode(W, min(max(K, 100), 2000))
    # the pipelined loop's outputs equal the same steps run on the device directly
    n_chk = got.shape[0]
    for s in range(n_chk):
        W.step(s)
    torch.cuda.synchronize()
    ref = torch.cat([W.out[0][:n_chk].reshape(n_chk, -1), W.out[1][:n_chk].reshape(n_chk, -1)], 1).cpu()
    e2e_ok = bool(torch.equal(got, ref))
    e_secs = dist.max(e_secs)
    e2e = {"value": dist.sum(per_step_bytes * e_steps) / e_secs / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "us_per_step": e_secs / e_steps * 1e6, "steps": e_steps,
           "path": "moe_expert_routed_b200.Plan (Python binding -> moe_qmm_plan_run), pinned host buffers, "
                   "input and output copies on their own streams, double-buffered device buffers",
           "issue": e_mode, "outputs_match_device_steps": e2e_ok}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world, "steps": steps_timed,
        "warmup": warm_done, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "decode step m=1: gate/up (E128 top8 k2816 n1408) + down (k704 n2816), "
                               "affine 4-bit g64, bf16 x, f32 out",
                   "l2": f"inputs larger than L2: {N_LAYERS} rotated weight copies "
                         f"({N_LAYERS * 0.428:.1f} GB), fresh ids and x every step",
                   "timing": (f"CUDA graph of {Gt} steps, CUDA events recorded as nodes of the graph "
                              "before the first and after the last step" if in_graph else
                              f"CUDA graph of {Gt} steps replayed {replays}x, CUDA events around the replays")
                             + ("" if uploaded else " (graph replayed once more during warm-up)"),
                   "launch": ("gate/up: programmatic dependent launch; down: PDL with early weight "
                              "streaming (its ids were ready before gate/up began)")
                             if not args.no_pdl else "plain stream order",
                   "parallelism": f"replicas x{dist.world}"},
        "per_call": pc,
        "roofline": roofline,
        "gpu_launches": 2 * steps_timed,
        "clocks": clocks,
        "e2e": e2e,
    }
    del W
    torch.cuda.empty_cache()
    if dist.world == 1 and not args.no_extras:
        # the other workloads and the decode m-sweep, on this GPU, outside the timed region
        sampler = clocks_sampler(dev)
        line["per_config"] = {name: grouped_entry(name, pk) for name in ("canvas", "prefill", "skewed")}
        line["per_config"]["prefill_w4a4"] = w4a4_entry(pk)
        line["sweep"] = decode_sweep(pk)
        line["per_config_clocks"] = clocks_summary(sampler)
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        v, s, threads, sample = oracle_decode_sample(args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": sample, "single_thread": oracle_single_thread()}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def run_grouped(args, dist: Dist):
    """One grouped-path workload as the bench line (N independent replicas for N > 1)."""
    import moe_expert_routed_b200 as M

    M.lib()
    dev_i = dist.local if dist.world > 1 else 0
    torch.cuda.set_device(dev_i)
    pk = peaks()
    sampler = clocks_sampler(dev_i) if dist.rank == 0 else None
    dist.barrier()
    ent = grouped_entry(args.config, pk)
    dist.barrier()
    clocks = clocks_summary(sampler) if dist.rank == 0 else None
    us = dist.max(ent["us_per_call"])
    tf = dist.sum(ent["algorithmic_flops"]) / us / 1e6
    line = {
        "metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": dist.world,
        "steps": GRAPH_CALLS * REPEATS, "warmup": GRAPH_CALLS + 3, "ms_per_step": us / 1e3, "us_per_call": us,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ent["workload"].split(", ")[-2], "data": "synthetic",
        "config": {"workload": f"{args.config}: {ent['workload']}", "l2": ent["l2"], "timing": ent["timing"]},
        "per_config": {args.config: ent}, "roofline": ent["roofline"],
        "gpu_launches": ent["gpu_launches_per_call"] * GRAPH_CALLS * REPEATS, "clocks": clocks,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(args):
    pk = peaks()
    sampler = clocks_sampler(torch.cuda.current_device())
    rows = decode_sweep(pk)
    print(json.dumps({"sweep": "decode m=1..8 (E128 top8, affine 4-bit g64, bf16 x, f32 out), per projection",
                      "rows": rows, "peak_hbm_gbs": pk["hbm_gbs"], "peak_source": pk["source"],
                      "timing": f"CUDA graph of {GRAPH_CALLS} calls, median of {REPEATS} replays, fresh ids and "
                                f"x per call, {N_LAYERS} rotated weight copies",
                      "clocks": clocks_summary(sampler)}), flush=True)


def run_crossover(args):
    """The decode / grouped crossover: the decode gate/up and down shapes (E128 top8,
    affine 4-bit g64, bf16 x) at m = 1 .. 64 tokens (8 .. 512 routings), each call
    timed on the CUDA-core decode path (path="decode": routing fused for R <= 64,
    else the routing prologue and the routed GEMV) and on the tcgen05 grouped GEMM
    (path="grouped"): CUDA graphs of calls with fresh ids and x per call and
    N_LAYERS rotated weight copies, median of REPEATS replays."""
    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.gen import bf16_bits, distinct_uniform_ids
    from workloads.torch_io import to_device

    calls = 40
    rng = np.random.Generator(np.random.PCG64(91))
    sampler = clocks_sampler(torch.cuda.current_device())
    rows = []
    for name in ("decode_gate_up", "decode_down"):
        P = config_problem(name)
        base = to_device(P)
        layers = [{k: base[k].clone() for k in ("packed", "scales", "aux")} for _ in range(N_LAYERS)]
        for m in (1, 2, 4, 6, 8, 9, 12, 16, 24, 32, 48, 64):
            ids = distinct_uniform_ids(rng, m * calls, 8, P.num_experts).reshape(calls, m, 8)
            x = bf16_bits(rng.standard_normal((calls, m, P.k), dtype=np.float32))
            d_ids = torch.from_numpy(ids.view(np.int32)).cuda()
            d_x = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            out = torch.empty((calls, m, 8, P.n), dtype=torch.float32, device="cuda")
            ws = M.new_workspace(m, 8, P.num_experts, k=P.k, x_dtype=torch.bfloat16)
            row = {"projection": name.replace("decode_", ""), "m": m, "routings": 8 * m}
            for path in ("decode", "grouped"):
                def one(c, path=path):
                    L = layers[c % N_LAYERS]
                    M.qmm_id(d_x[c], d_ids[c], L["packed"], L["scales"], L["aux"], n=P.n,
                             group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                             out=out[c], workspace=ws, path=path)
                g = capture_graph(one, calls)
                r = per_call(g, calls)
                del g
                row[f"{path}_us"] = r["s"] * 1e6
            row["faster"] = "decode" if row["decode_us"] <= row["grouped_us"] else "grouped"
            rows.append(row)
        del base, layers
        torch.cuda.empty_cache()
    print(json.dumps({"crossover": "decode path vs grouped GEMM per call, E128 top8 affine 4-bit g64, bf16 x",
                      "rows": rows, "timing": f"CUDA graph of {calls} calls, median of {REPEATS} replays",
                      "threshold_in_library": "MOE_DECODE_MAX_ROUTINGS, MOE_DECODE_MAX_PAIRS_PER_EXPERT",
                      "clocks": clocks_summary(sampler)}), flush=True)


def run_probe(args):
    """A few untimed calls of one workload (for profiler captures): decode runs the
    gate/up projection `reps` times, then the down projection `reps` times; the
    grouped configs run one full call `reps` times; prefill_w4a4 runs the prefill
    workload through moe_qmm_id_w4a4 `reps` times."""
    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.torch_io import to_device

    M.lib()
    if args.probe == "prefill_w4a4":
        P = config_problem("prefill")
        d = to_device(P)
        ws = torch.zeros(M.workspace_bytes_w4a4(P.m, P.k, P.n_expert_used, P.num_experts), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty((P.m, P.n_expert_used, P.n), dtype=torch.bfloat16, device="cuda")
        for _ in range(args.reps):
            M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                          bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out, workspace=ws)
        torch.cuda.synchronize()
        if M.poll_error(ws) != 0:
            raise SystemExit("prefill_w4a4: device error word set")
        print(json.dumps({"probe": args.probe, "reps": args.reps, "status": "ok"}))
        return
    names = ["decode_gate_up", "decode_down"] if args.probe == "decode" else [args.probe]
    for name in names:
        P = config_problem(name)
        d = to_device(P)
        ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts, k=P.k, x_dtype=d["x"].dtype)
        out_dt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float16}[P.out_dtype]
        out = torch.empty((P.m, P.n_expert_used, P.n), dtype=out_dt, device="cuda")
        for _ in range(args.reps):
            M.qmm_id(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                     bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out, workspace=ws)
        torch.cuda.synchronize()
        if M.poll_error(ws) != 0:
            raise SystemExit(f"{name}: device error word set")
    print(json.dumps({"probe": args.probe, "reps": args.reps, "status": "ok"}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-pdl", action="store_true",
                    help="decode step without programmatic dependent launch between its calls")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--config", default="decode", choices=["decode", "canvas", "prefill", "skewed"])
    ap.add_argument("--probe", choices=["decode", "canvas", "prefill", "skewed", "prefill_w4a4"],
                    help="run a few untimed calls (for profiler captures) and exit")
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--no-extras", action="store_true",
                    help="decode bench line without the grouped workloads and the m-sweep")
    ap.add_argument("--sweep", action="store_true",
                    help="decode m = 1, 2, 4, 8 curve (one GPU), one JSON line, instead of the bench line")
    ap.add_argument("--crossover", action="store_true",
                    help="decode path vs grouped GEMM per call at m = 1 .. 64 tokens (one GPU), one JSON line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.crossover:
        run_crossover(args)
        return
    if args.probe:
        run_probe(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, dist)
        elif args.config != "decode":
            run_grouped(args, dist)
        else:
            run_ours(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
