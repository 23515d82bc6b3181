"""Benchmark of the expert-routed quantized matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode|canvas|prefill|skewed]

Default workload ("decode"): one MoE decode step for one token: the gate/up
projection (128 experts, top-8, k=2816, n=1408) followed by the down projection
(k=704, n=2816), both 4-bit affine with group 64, bf16 x, f32 out. Every step
uses fresh ids (8 distinct uniform experts), fresh x, and the next of 16 copies
of the expert weights (6.9 GB rotated, far above the 126 MB L2), so no step
finds its weights in L2. The K timed steps are replayed from CUDA graphs of up
to 1000 steps (launch overhead of the graph only, no host work).

Metric: effective HBM GB/s = algorithmic bytes / time, algorithmic bytes = the
touched experts' packed codes + scales + biases read once, plus x and out.
Also reported: us per call of each projection, the roofline fraction against
MEASURED_PEAKS.json's copy bandwidth, the end-to-end number through the Python
API with host buffers, and the CPU oracle on a bounded sample.

--impl reference times the CPU oracle (the only reference there is) on a
bounded sample of the same workload. N > 1: independent replicas, one per GPU
(the operation has no exchange step), value = total bytes / max time.
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
GRAPH_STEPS = 1000
# dram__bytes_read.sum + dram__bytes_write.sum of one gate/up launch of the decode
# kernel, from one ncu capture of it (cold L2)
GATE_UP_DRAM_BYTES = 17875200


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
    """gate/up + down projections of one decode token, rotating weight copies."""

    def __init__(self, steps_per_graph: int, seed: int = 2, pdl: bool = True):
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
        self.G = steps_per_graph
        rng = np.random.Generator(np.random.PCG64(seed + 100))
        self.layers = []
        for P in self.projs:
            base = to_device(P)
            copies = []
            for _ in range(N_LAYERS):
                copies.append({k: (v.clone() if k in ("packed", "scales", "aux") else v)
                               for k, v in base.items()})
            self.layers.append(copies)
        # fresh ids and x for every step of the graph
        self.ids = [torch.from_numpy(distinct_uniform_ids(rng, self.G, 8, P.num_experts)
                                     .view(np.int32)).cuda() for P in self.projs]
        self.x = [torch.from_numpy(bf16_bits(rng.standard_normal((self.G, P.k), dtype=np.float32))
                                   .view(np.int16)).view(torch.bfloat16).cuda() for P in self.projs]
        self.out = [torch.empty((self.G, 8, P.n), dtype=torch.float32, device="cuda")
                    for P in self.projs]
        # gated gate/up output: act(gate) * up, n/2 columns
        self.out_glu = torch.empty((self.G, 8, self.projs[0].n // 2), dtype=torch.float32, device="cuda")
        self.ws = [M.new_workspace(1, 8, P.num_experts) for P in self.projs]
        self.step_bytes = [
            [alg_bytes(P, self.ids[i][s].cpu().numpy().view(np.uint32)) for s in range(self.G)]
            for i, P in enumerate(self.projs)]

    def call(self, proj: int, s: int, act=None, launch=None):
        P = self.projs[proj]
        L = self.layers[proj][s % N_LAYERS]
        self.M.qmm_id(self.x[proj][s:s + 1], self.ids[proj][s:s + 1], L["packed"], L["scales"],
                      L["aux"], n=P.n, group_size=P.group_size, bits=P.bits, fmt=P.fmt,
                      num_experts=P.num_experts, out=self.out_glu[s] if act else self.out[proj][s],
                      workspace=self.ws[proj], act=act, launch=launch)

    def step(self, s: int, projs=(0, 1), act=None):
        # the step's launch modes apply to the full gate/up + down sequence only
        full = tuple(projs) == (0, 1)
        for p in projs:
            self.call(p, s, act, self.launch[p] if full else None)

    def bytes(self, projs=(0, 1)) -> float:
        return sum(sum(self.step_bytes[p]) for p in projs)

    def capture(self, projs=(0, 1), act=None):
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            for s in range(min(self.G, 4)):
                self.step(s, projs, act)  # warm the launch path outside capture
        torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for s in range(self.G):
                self.step(s, projs, act)
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


def e2e_decode(W: DecodeWorkload, steps: int):
    """Through the public API with host buffers: per step, one copy brings that
    step's x rows and ids of both projections in from pinned host memory, both
    projections run (moe_expert_routed_b200.Plan: one per layer copy and
    projection, bound before the timed region, the step's launch modes), one copy
    takes both outputs back."""
    M = W.M
    n = min(steps, W.G)
    # per-step input block: x of each projection (bf16), then ids of each projection
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
    din = torch.empty(blk, dtype=torch.uint8, device="cuda")
    dx = [din[offs[p]:offs[p] + xb[p]].view(torch.bfloat16).view(1, W.projs[p].k) for p in range(2)]
    did = [din[offs[2 + p]:offs[2 + p] + ib[p]].view(torch.int32).view(1, -1) for p in range(2)]
    nout = [8 * P.n for P in W.projs]
    dout_all = torch.empty(sum(nout), dtype=torch.float32, device="cuda")
    hout = torch.empty(sum(nout), dtype=torch.float32).pin_memory()
    dout = [dout_all[:nout[0]].view(1, 8, W.projs[0].n), dout_all[nout[0]:].view(1, 8, W.projs[1].n)]
    h2d = sum(xb) + sum(ib)
    d2h = sum(nout) * 4
    plans = [[M.Plan(L["packed"], L["scales"], L["aux"], m=1, k=P.k, n=P.n, group_size=P.group_size,
                     bits=P.bits, fmt=P.fmt, n_expert_used=8, num_experts=P.num_experts,
                     x_dtype=torch.bfloat16, out_dtype=torch.float32, workspace=W.ws[p],
                     launch=W.launch[p]) for L in W.layers[p]] for p, P in enumerate(W.projs)]
    hrows = [hin[i] for i in range(n)]

    def run_steps(st, count):
        for s in range(count):
            din.copy_(hrows[s % n], non_blocking=True)
            plans[0][s % N_LAYERS](dx[0], did[0], dout[0], st)
            plans[1][s % N_LAYERS](dx[1], did[1], dout[1], st)
            hout.copy_(dout_all, non_blocking=True)

    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    # the n steps (copy in, two calls, copy out) captured once in a CUDA graph and
    # replayed, so that the host's issue cost per call does not set the pace; the
    # copies still run every step
    try:
        g = torch.cuda.CUDAGraph()
        ws = torch.cuda.Stream()
        ws.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(ws):
            run_steps(ws, 2)
        torch.cuda.current_stream().wait_stream(ws)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            run_steps(torch.cuda.current_stream(), n)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, (steps + n - 1) // n)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        b.synchronize()
        done, mode = reps * n, f"CUDA graph of {n} steps (copies and calls) replayed {reps}x"
        del g
    except RuntimeError as exc:  # capture refused: time the same steps issued one by one
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        a.record()
        run_steps(st, steps)
        b.record()
        b.synchronize()
        done, mode = steps, f"eager ({type(exc).__name__} in graph capture)"
    secs = a.elapsed_time(b) / 1e3
    per_step_bytes = W.bytes() / W.G
    return secs, done, mode, per_step_bytes, h2d, d2h


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


def run_ours(args, dist: Dist):
    import moe_expert_routed_b200 as M

    M.lib()  # fails loudly if the CUDA library is missing
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    dev = dist.local if dist.world > 1 else 0
    torch.cuda.set_device(dev)
    K, Wm = args.steps, args.warmup
    G = min(GRAPH_STEPS, K)
    W = DecodeWorkload(G, pdl=not args.no_pdl)
    g = W.capture()
    replays = max(1, K // G)
    steps_timed = replays * G
    warm_replays = max(1, -(-Wm // G))
    for _ in range(warm_replays):
        g.replay()
    torch.cuda.synchronize()
    sampler = clocks_sampler(dev) if dist.rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    dist.barrier()
    torch.cuda.synchronize()
    secs = time_graph(g, replays)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = clocks_summary(sampler) if dist.rank == 0 else None
    secs_max = dist.max(secs)
    bytes_total = dist.sum(W.bytes() * replays)
    value = bytes_total / secs_max / 1e9
    ms_per_step = secs_max / steps_timed * 1e3

    # per-projection calls (separate graphs, outside the timed region)
    per_call = {}
    for p, name in ((0, "gate_up"), (1, "down")):
        gp = W.capture(projs=(p,))
        gp.replay()
        t = time_graph(gp, max(1, replays // 2))
        per_call[name] = {"us_per_call": t / (max(1, replays // 2) * G) * 1e6,
                          "GB_per_s": W.bytes((p,)) * max(1, replays // 2) / t / 1e9}
        del gp
    # the gate/up projection with its SiLU-gated epilogue (moe_qmm_id_glu): same
    # weights and x, half the output columns
    gp = W.capture(projs=(0,), act="silu")
    gp.replay()
    t = time_graph(gp, max(1, replays // 2))
    glu_bytes = W.bytes((0,)) - G * 8 * (W.projs[0].n // 2) * 4
    per_call["gate_up_silu"] = {"us_per_call": t / (max(1, replays // 2) * G) * 1e6,
                                "GB_per_s": glu_bytes * max(1, replays // 2) / t / 1e9}
    del gp

    pk = peaks()
    # dominant kernel: the gate/up launch (about 57% of the step); timed alone from a
    # graph of gate/up calls only. DRAM traffic per launch from one ncu capture of
    # this kernel.
    achieved = per_call["gate_up"]["GB_per_s"]
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": None,
                "traffic_note": f"{GATE_UP_DRAM_BYTES} B per launch (= the algorithmic bytes) in the last ncu "
                                "capture, taken before the launch-dependency and gated-output changes to "
                                "the kernel; null until re-captured",
                "algorithmic_bytes": W.bytes((0,)) / W.G,
                "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)",
                "kernel": "gemv_aff4_rows (rows of all pairs split evenly over the SMs), gate/up launch",
                "step_frac": W.bytes() * replays / secs / 1e9 / pk["hbm_gbs"]}
    e2e_steps = min(max(K // 10, 50), 2000)
    e_secs, e2e_steps, e2e_mode, per_step_bytes, h2d, d2h = e2e_decode(W, e2e_steps)
    e_secs = dist.max(e_secs)
    e2e = {"value": dist.sum(per_step_bytes * e2e_steps) / e_secs / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "us_per_step": e_secs / e2e_steps * 1e6, "steps": e2e_steps,
           "path": "moe_expert_routed_b200.Plan (Python binding -> moe_qmm_plan_run), pinned host buffers",
           "issue": e2e_mode}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": dist.world, "steps": steps_timed,
        "warmup": warm_replays * G, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "decode step m=1: gate/up (E128 top8 k2816 n1408) + down (k704 n2816), "
                               "affine 4-bit g64, bf16 x, f32 out",
                   "l2": f"inputs larger than L2: {N_LAYERS} rotated weight copies "
                         f"({N_LAYERS * 0.428:.1f} GB), fresh ids and x every step",
                   "timing": f"CUDA graph of {G} steps replayed {replays}x, CUDA events",
                   "launch": ("gate/up: programmatic dependent launch; down: PDL with early weight "
                              "streaming (its ids were ready before gate/up began)")
                             if not args.no_pdl else "plain stream order",
                   "parallelism": f"replicas x{dist.world}"},
        "per_call": per_call,
        "roofline": roofline,
        "gpu_launches": 2 * steps_timed,
        "clocks": clocks,
        "e2e": e2e,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        v, s, threads, sample = oracle_decode_sample(args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": sample, "single_thread": oracle_single_thread()}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    del g


def run_grouped(args, dist: Dist):
    """One call of the named grouped-path workload per step (routing prologue +
    tcgen05 grouped GEMM), inputs resident in HBM, CUDA graph of G calls."""
    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.torch_io import to_device

    M.lib()
    dev_i = dist.local if dist.world > 1 else 0
    torch.cuda.set_device(dev_i)
    P = config_problem(args.config)
    d = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out_dt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float16}[P.out_dtype]
    out = torch.empty((P.m, P.n_expert_used, P.n), dtype=out_dt, device="cuda")

    def call():
        M.qmm_id(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                 bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out, workspace=ws)

    def route_only():
        M.route(d["ids"], P.num_experts, 256 if P.R >= 96 * P.num_experts else 64, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    assert M.poll_error(ws) == 0
    G = max(1, min(args.steps, 20))
    graphs = []
    for fn in (call,):
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            fn()
        torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for _ in range(G):
                fn()
        graphs.append(g)
    replays = max(1, args.steps // G)
    graphs[0].replay()
    sampler = clocks_sampler(dev_i) if dist.rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    dist.barrier()
    torch.cuda.synchronize()
    secs = time_graph(graphs[0], replays)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = clocks_summary(sampler) if dist.rank == 0 else None
    calls = replays * G
    # routing prologue alone (outside the timed region): share of a call
    for _ in range(3):
        route_only()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(50):
        route_only()
    b.record()
    b.synchronize()
    route_us = a.elapsed_time(b) / 50 * 1e3
    secs_max = dist.max(secs)
    ids = P.ids.reshape(-1)
    valid = int((ids < P.num_experts).sum())
    flops = 2.0 * valid * P.n * P.k
    nbytes = alg_bytes(P, ids)
    us = secs_max / calls * 1e6
    tflops = dist.sum(flops * calls) / secs_max / 1e12
    gbs = dist.sum(nbytes * calls) / secs_max / 1e9
    pk = peaks()
    gemm_us = max(us - route_us, 1e-9)
    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": dist.world, "steps": calls,
        "warmup": max(args.warmup, 3), "ms_per_step": us / 1e3, "us_per_call": us,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {0: "f32", 1: "bf16", 2: "f16"}[P.x_dtype] + " x / fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": f"{args.config}: E{P.num_experts} top{P.n_expert_used} m{P.m} k{P.k} n{P.n} "
                               f"fmt{P.fmt} bits{P.bits} g{P.group_size}",
                   "l2": f"weights {P.packed.nbytes / 1e6:.0f} MB (> L2 126 MB), one call per step",
                   "timing": f"CUDA graph of {G} calls replayed {replays}x, CUDA events"},
        "effective_GB_per_s": gbs,
        "route_us": route_us,
        "gemm_us_estimate": gemm_us,
        "roofline": {"tensor": {"achieved": flops / gemm_us / 1e6, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": flops / gemm_us / 1e6 / pk["bf16_tflops"]},
                     "hbm": {"achieved": nbytes / gemm_us / 1e3, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": nbytes / gemm_us / 1e3 / pk["hbm_gbs"]},
                     "kernel": "grouped_gemm_kernel (tcgen05), time = call - routing prologue"},
        "gpu_launches": 4 * calls,
        "clocks": clocks,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(args):
    """Decode with m = 1, 2, 4, 8 tokens (top-8 of 128 experts), gate/up and down
    projections timed separately: a CUDA graph of calls with fresh ids and x each
    call and 16 rotated weight copies. Effective GB/s counts the distinct experts
    each call actually touches (E[D] = 8, 15.5, 29.1, 51.6 for uniform ids)."""
    import types

    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.gen import bf16_bits, distinct_uniform_ids
    from workloads.torch_io import to_device

    calls = 200
    rng = np.random.Generator(np.random.PCG64(77))
    sampler = clocks_sampler(torch.cuda.current_device())
    pk = peaks()
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
            nbytes = sum(alg_bytes(Pm, ids[c]) for c in range(calls))
            distinct = float(np.mean([np.unique(ids[c]).size for c in range(calls)]))

            def one(c):
                L = layers[c % N_LAYERS]
                M.qmm_id(d_x[c], d_ids[c], L["packed"], L["scales"], L["aux"], n=P.n,
                         group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                         out=out[c], workspace=ws)

            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                for c in range(4):
                    one(c)
            torch.cuda.current_stream().wait_stream(st)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for c in range(calls):
                    one(c)
            time_graph(g, max(3, args.warmup // calls))
            reps = max(1, args.steps // calls)
            secs = time_graph(g, reps)
            del g
            us = secs / (reps * calls) * 1e6
            gbs = nbytes * reps / secs / 1e9
            rows.append({"projection": name.replace("decode_", ""), "m": m, "distinct_experts": distinct,
                         "us_per_call": us, "GB_per_s": gbs, "frac_of_hbm": gbs / pk["hbm_gbs"]})
    line = {"sweep": "decode m=1..8 (E128 top8, affine 4-bit g64, bf16 x, f32 out), per projection",
            "rows": rows, "peak_hbm_gbs": pk["hbm_gbs"], "peak_source": pk["source"],
            "timing": f"CUDA graph of {calls} calls, fresh ids and x per call, {N_LAYERS} rotated weight copies",
            "clocks": clocks_summary(sampler)}
    print(json.dumps(line), flush=True)


def run_probe(args):
    """A few untimed calls of one workload (for profiler captures): decode runs the
    gate/up projection `reps` times, then the down projection `reps` times; the
    grouped configs run one full call `reps` times."""
    import moe_expert_routed_b200 as M
    from workloads import config_problem
    from workloads.torch_io import to_device

    M.lib()
    names = ["decode_gate_up", "decode_down"] if args.probe == "decode" else [args.probe]
    for name in names:
        P = config_problem(name)
        d = to_device(P)
        ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
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
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-pdl", action="store_true",
                    help="decode step without programmatic dependent launch between its calls")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--config", default="decode", choices=["decode", "canvas", "prefill", "skewed"])
    ap.add_argument("--probe", choices=["decode", "canvas", "prefill", "skewed"],
                    help="run a few untimed calls (for profiler captures) and exit")
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--sweep", action="store_true",
                    help="decode m = 1, 2, 4, 8 curve (one GPU), one JSON line, instead of the bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
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
