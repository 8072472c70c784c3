"""Benchmark of the SSD layer on B200.

A step is one chunked forward (all four steps of the block-decomposed
algorithm: chunk states, inter-chunk recurrence, intra-chunk masked C B^T
term and entering-state term + D skip) over the 2.7B-layer workload
(batch 4, L 8192, H 80, P 64, N 128, G 1, chunk 256, bf16 x/B/C, fp32 dt/A/D,
random initial states, final states returned), with inputs resident in HBM.
The decode step (batch 256, H 80, P 64, N 128) is timed in the same run and
reported under "decode".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
With N > 1 (launched by torchrun) every rank runs the same per-GPU workload
(weak scaling; the layer shards over batch and heads with no exchange) and
rank 0 prints one JSON line with the max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SSD fwd tokens/s and TFLOP/s (% bf16 TC peak) at 2.7B-layer shape; decode GB/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- workload model
def fwd_model(w):
    """Algorithmic FLOPs and minimum HBM bytes of one chunked forward."""
    b, L, H, P, N, G, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk
    sx = 2 if w.dtype == "bf16" else 4
    # causal half of the diagonal blocks, C B^T once per group, states in and out
    f_alg = 2 * b * L * (G * N * (Q + 1) / 2 + H * P * (Q + 1) / 2 + 2 * H * N * P)
    f_dense = 2 * b * L * (G * N * Q + H * P * Q + 2 * H * N * P)
    n_state = b * H * P * N
    bytes_min = (b * L * (2 * H * P * sx + 2 * G * N * sx + 4 * H)
                 + 4 * n_state * (int(w.with_init) + int(w.want_final)))
    return f_alg, f_dense, bytes_min


def kernel_bytes(w):
    """Per kernel of either data flow: (alg, io).

    alg: the kernel's share of the forward's minimum bytes (bytes_min: x, y,
    B, C, dt, initial and final states, each once) -- the inputs and outputs
    of the layer that the kernel itself must read or write.  Intermediates
    (chunk states, entering states) count zero: a better data flow removes
    them.  io: everything the kernel reads and writes, intermediates
    included, each once."""
    b, L, H, P, N, G, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk
    sx = 2 if w.dtype == "bf16" else 4
    T = (L + Q - 1) // Q
    ns = b * T * H * P * N
    x = b * L * H * P * sx
    bc = b * L * G * N * sx
    dt = b * L * H * 4
    init = 4 * b * H * P * N * int(w.with_init)
    fin = 4 * b * H * P * N * int(w.want_final)
    ld = 4 * b * T * H
    return {
        "chunk_state": (x + bc + dt, x + bc + dt + 4 * ns + ld),
        "state_pass": (init + fin, 4 * ns + ld + sx * ns + init + fin),
        "state_walk": (x + bc + dt + init + fin, x + bc + dt + sx * ns + init + fin),
        "chunk_out": (2 * x + 2 * bc + dt, 2 * x + 2 * bc + dt + sx * ns),
        # walkers and output tiles in one launch: the whole forward's bytes_min;
        # its own I/O reads x and B twice (walkers and tiles) and writes and
        # reads the entering states
        "walk_out": (2 * x + 2 * bc + dt + init + fin,
                     3 * x + 3 * bc + 2 * dt + init + fin + 2 * sx * ns),
    }


KERNEL_SOURCES = {
    "state_walk": ["state_walk_tc.cu", "state_walk_body.cuh", "sm100.cuh"],
    "chunk_state": ["chunk_state_tc.cu", "sm100.cuh"],
    "state_pass": ["state_pass.cu"],
    "chunk_out": ["chunk_out_tc.cu", "chunk_out_body.cuh", "sm100.cuh"],
    "walk_out": ["walk_out_tc.cu", "state_walk_body.cuh", "chunk_out_body.cuh", "sm100.cuh"],
    "decode": ["decode.cu"],
}


def code_text(src: str) -> str:
    """A CUDA source with its comments removed and its whitespace collapsed:
    what a kernel's DRAM traffic can depend on."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        p = os.path.join(ROOT, "ssd_chunked_scan_02_b200", "csrc", f)
        if os.path.exists(p):
            with open(p) as fh:
                h.update(code_text(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("workload") != workload or e.get("source_sha") != source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"ssd_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(n, backend: str = "nccl"):
    """One process per GPU (launched by torchrun): join the process group and
    return (rank, world, local_rank).  backend "gloo" is for CPU tests of
    this logic."""
    if n <= 1:
        return 0, 1, 0
    import datetime

    import torch
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    """The maximum of a per-rank number over all ranks (device time of the
    slowest rank)."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_scaling_value(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own tokens_per_rank per
    step; the step takes the slowest rank's time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------- CPU oracle baseline
def cpu_oracle_sample(w, inp_cpu, seconds_budget: float = 12.0):
    """Time the fp64 oracle on a bounded sample of the workload: batch
    element 0 (all heads, the whole sequence), repeated for about
    ``seconds_budget`` seconds.  Returns
    (tokens/s scaled to the full layer, description, cores)."""
    import oracle
    cores = os.cpu_count() or 1
    heads = w.nheads
    sl = {
        "x": inp_cpu["x"][0:1, :, :heads], "dt": inp_cpu["dt"][0:1, :, :heads],
        "A": inp_cpu["A"][:heads], "B": inp_cpu["B"][0:1], "C": inp_cpu["C"][0:1],
        "D": inp_cpu["D"][:heads],
        "init": inp_cpu["init"][0:1, :heads] if inp_cpu.get("init") is not None else None,
    }
    args = [oracle._f64(sl[k]) for k in ("x", "dt", "A", "B", "C", "D")]
    init = oracle._f64(sl["init"]) if sl["init"] is not None else None
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.recurrence(*args, init, threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el > seconds_budget or reps >= 1000:
            break
    per = el / reps
    # the sample covers heads/H of one batch element's tokens
    frac = heads / w.nheads
    tok_s = w.seqlen * frac / per
    desc = (f"fp64 oracle recurrence over batch 0, heads 0..{heads - 1} of {w.nheads}, "
            f"L={w.seqlen} ({reps} reps, {per:.3f} s each); tokens/s scaled by heads")
    return tok_s, desc, cores


def cpu_model() -> str:
    """The host CPU's model name (lscpu), or the platform's processor string."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baselines(w, inp_cpu, budget_s: float = 12.0):
    """The oracle timed on the host as it stands (a reported baseline, not a
    target), on bounded samples of each workload:
      - the 2.7B layer on all cores (batch 0, all heads, the whole sequence)
        and on one thread (batch 0, heads 0..7);
      - the 130M layer on all cores (batch 0, all heads);
      - decode (b256 H80 P64 N128): 16 sequences x 1024 steps of the same
        recurrence on all cores, reported per step of the full batch.
    Returns the cpu_baseline object of the bench line."""
    import oracle
    from ssd_chunked_scan_02_b200 import inputs
    cores = os.cpu_count() or 1
    tok_s, desc, cores = cpu_oracle_sample(w, inp_cpu, seconds_budget=budget_s)

    def timed(fn, budget):
        t0 = time.perf_counter()
        reps = 0
        while True:
            fn()
            reps += 1
            el = time.perf_counter() - t0
            if el > budget or reps >= 1000:
                return el / reps, reps

    # one thread, 8 heads of batch 0 of the same layer
    hs = 8
    one = [oracle._f64(inp_cpu[k][0:1, :, :hs]) for k in ("x", "dt")]
    args1 = [one[0], one[1], oracle._f64(inp_cpu["A"][:hs]), oracle._f64(inp_cpu["B"][0:1]),
             oracle._f64(inp_cpu["C"][0:1]), oracle._f64(inp_cpu["D"][:hs])]
    init1 = oracle._f64(inp_cpu["init"][0:1, :hs]) if inp_cpu.get("init") is not None else None
    per1, reps1 = timed(lambda: oracle.recurrence(*args1, init1, threads=1), 4.0)
    tok1 = w.seqlen * hs / w.nheads / per1
    # the 130M layer, batch 0, all heads, all cores
    w1 = inputs.LAYER_130M
    i1 = inputs.make_inputs(w1.with_(batch=1))
    a130 = [oracle._f64(i1[k]) for k in ("x", "dt", "A", "B", "C", "D")]
    per130, reps130 = timed(lambda: oracle.recurrence(*a130, None, threads=cores), 3.0)
    # decode: 16 sequences x 1024 steps
    dw = inputs.DECODE_2P7B
    nb, steps = 16, dw.steps
    dd = inputs.make_inputs(inputs.Workload("decode_cpu_sample", nb, steps, dw.nheads, dw.headdim,
                                            dw.dstate, dw.ngroups, 256, dw.dtype, with_init=True,
                                            want_final=True, seed=dw.seed))
    adec = [oracle._f64(dd[k]) for k in ("x", "dt", "A", "B", "C", "D")]
    idec = oracle._f64(dd["init"])
    perd, _ = timed(lambda: oracle.recurrence(*adec, idec, threads=cores), 1.0)
    step_s_full = perd / steps * (dw.batch / nb)          # one step of the full b=256 batch
    dec_bytes = 2 * 4 * dw.batch * dw.nheads * dw.headdim * dw.dstate
    return {
        "value": tok_s, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
        "cpu_model": cpu_model(),
        "single_thread": {"value": tok1, "unit": UNIT, "cores": 1,
                          "sample": f"batch 0, heads 0..{hs - 1} of {w.nheads}, L={w.seqlen} "
                                    f"({reps1} reps, {per1:.3f} s each); tokens/s scaled by heads"},
        "other_configs": [
            {"workload": w1.name, "value": w1.seqlen / per130, "unit": UNIT, "cores": cores,
             "sample": f"batch 0 of {w1.batch}, all {w1.nheads} heads, L={w1.seqlen} "
                       f"({reps130} reps, {per130:.3f} s each)"},
            {"workload": dw.name, "ms_per_step": 1e3 * step_s_full, "cores": cores,
             "state_gbs": dec_bytes / step_s_full / 1e9,
             "sample": f"{nb} of {dw.batch} sequences x {steps} steps as one recurrence "
                       f"({perd:.2f} s); per step of the full batch by scaling"},
        ],
    }


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    """The reference arm here is the fp64 CPU oracle, timed as it stands."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from ssd_chunked_scan_02_b200 import inputs
    w = inputs.LAYER_2P7B
    inp = inputs.make_inputs(w)
    times = []
    cores = os.cpu_count() or 1
    desc = None
    for i in range(args.warmup + args.steps):
        tok_s, desc, cores = cpu_oracle_sample(w, inp, seconds_budget=3.0)
        if i >= args.warmup:
            times.append(tok_s)
    value = statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.tokens / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups,
                   "chunk": w.chunk, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- secondary configs
def measure_config(w, dev, stream, flush, reps, world, rank):
    """Forward time of one more workload (the 130M layer, the length sweep):
    L2 flushed before every timed forward, device time, max over ranks."""
    import torch
    from ssd_chunked_scan_02_b200 import inputs, ssd
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 1000 * rank)
    inp = inputs.make_inputs(w, device=dev, gen=gen)
    y = torch.empty_like(inp["x"])
    fin = (torch.empty((w.batch, w.nheads, w.headdim, w.dstate), device=dev, dtype=torch.float32)
           if w.want_final else None)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
    ws = torch.empty(ssd.ssd_chunk_scan_fwd_workspace_size(dims, w.chunk, inp["x"].dtype),
                     device=dev, dtype=torch.uint8)

    def fwd():
        ssd.ssd_chunk_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                               w.chunk, init_states=inp["init"], y=y, final_states=fin,
                               workspace=ws, stream=stream)
    for _ in range(3):
        flush.zero_()
        fwd()
    torch.cuda.synchronize(dev)
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for st, en in evs:
        flush.zero_()
        st.record(stream)
        fwd()
        en.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(sum(st.elapsed_time(en) for st, en in evs), world) / reps
    f_alg, f_dense, bytes_min = fwd_model(w)
    t = ms * 1e-3
    flow = ssd.ssd_chunk_scan_fwd_data_flow(dims, w.chunk, inp["x"].dtype)
    out = {"workload": w.name, "data_flow": FLOW_NAMES.get(flow, "simt"), "ms_per_step": ms, "tokens_per_s": world * w.tokens / t,
           "tflops_alg": f_alg / t / 1e12, "tflops_dense": f_dense / t / 1e12,
           "bytes_min": bytes_min, "hbm_gbs_at_bytes_min": bytes_min / t / 1e9}
    del inp, y, fin, ws
    torch.cuda.empty_cache()
    return out


def bwd_bytes(w) -> int:
    """Algorithmic bytes of the backward: its inputs read once (x, dy, B, C in
    the input dtype; dt fp32; the initial state when given) and its outputs
    written once (dx, ddt, dB, dC, d(initial state) in fp32)."""
    s = 2 if w.dtype == "bf16" else 4
    bl = w.batch * w.seqlen
    reads = bl * (2 * w.nheads * w.headdim * s + 2 * w.ngroups * w.dstate * s + 4 * w.nheads)
    writes = bl * (w.nheads * w.headdim * 4 + 4 * w.nheads + 2 * w.ngroups * w.dstate * 4)
    states = 4 * w.batch * w.nheads * w.headdim * w.dstate * ((1 if w.with_init else 0) + 1)
    return reads + writes + states


def measure_backward(w, dev, stream, flush, reps, world, rank, peak_gbs):
    """Device time of ssd_chunk_scan_bwd on one workload (L2 flushed before
    every timed call, max over ranks), with its HBM roofline fraction."""
    import torch
    from ssd_chunked_scan_02_b200 import inputs, ssd
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 2000 + 1000 * rank)
    inp = inputs.make_inputs(w, device=dev, gen=gen)
    dy = torch.randn(inp["x"].shape, device=dev, generator=gen).to(inp["x"].dtype)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
    ws = torch.empty(max(16, ssd.ssd_chunk_scan_bwd_workspace_size(dims, inp["x"].dtype)),
                     device=dev, dtype=torch.uint8)

    def bwd():
        ssd.ssd_chunk_scan_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], dy,
                               init_states=inp["init"], workspace=ws, stream=stream)
    for _ in range(3):
        flush.zero_()
        bwd()
    torch.cuda.synchronize(dev)
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for st, en in evs:
        flush.zero_()
        st.record(stream)
        bwd()
        en.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(sum(st.elapsed_time(en) for st, en in evs), world) / reps
    nbytes = bwd_bytes(w)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tc = ssd.ssd_chunk_scan_bwd_uses_tensor_cores(dims, inp["x"].dtype) == 1
    kind = ("tcgen05 block decomposition in 128-token chunks (entering states, reverse pass "
            "over the chunks for dL/dh, then dx/ddt and dB/dC kernels)" if tc else
            "exact fp32 SIMT, one CTA per block of state rows of a (batch, head)")
    out = {"workload": w.name, "kernel": kind, "tensor_cores": tc,
           "ms_per_step": ms, "tokens_per_s": world * w.tokens / (ms * 1e-3),
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak_gbs, "unit": "GB/s",
                        "frac": gbs / peak_gbs, "alg_bytes_per_launch": nbytes}}
    del inp, dy, ws
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- sequence-parallel split
def correction_bytes(w, Ls):
    """Algorithmic bytes of one shard's correction (every token corrected):
    C and dt read, y read and written, h_in read, final state read and
    written."""
    sx = 2 if w.dtype == "bf16" else 4
    ns = w.batch * w.nheads * w.headdim * w.dstate
    return (w.batch * Ls * (w.ngroups * w.dstate * sx + 4 * w.nheads + 2 * w.nheads * w.headdim * sx)
            + 4 * ns + 2 * 4 * ns)


def measure_seqpar(w, dev, stream, flush, reps, shards=2):
    """Per-rank device time of the sequence-parallel forward with the
    sequence split into ``shards`` equal pieces, each rank's steps run on
    this GPU one rank after another: the shard's zero-start forward, its
    log-decay, the combine of the gathered values and the correction.  The
    all-gather between them needs several GPUs and is not timed here."""
    import torch
    from ssd_chunked_scan_02_b200 import inputs, seqpar, ssd
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 4000)
    inp = inputs.make_inputs(w, device=dev, gen=gen)
    Ls = w.seqlen // shards
    parts = [{k: inp[k][:, r * Ls:(r + 1) * Ls].contiguous() for k in ("x", "dt", "B", "C")}
             for r in range(shards)]
    A, D, init = inp["A"], inp["D"], inp["init"]
    y = torch.empty_like(parts[0]["x"])
    fin = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), device=dev)
    dims = ssd.make_dims(w.batch, Ls, w.nheads, w.headdim, w.dstate, w.ngroups)
    ws = torch.empty(ssd.ssd_chunk_scan_fwd_workspace_size(dims, w.chunk, y.dtype), device=dev,
                     dtype=torch.uint8)
    cws = torch.empty(max(16, ssd.ssd_state_correction_workspace_size(dims, y.dtype)),
                      device=dev, dtype=torch.uint8)
    # the gathered values every rank would receive
    outs = []
    for p in parts:
        yy, ff = ssd.ssd_chunk_scan_fwd(p["x"], p["dt"], A, p["B"], p["C"], D, w.chunk,
                                        return_final_states=True)
        outs.append(seqpar.pack(ff, ssd.ssd_seq_logdecay(p["dt"], A)))
    finals, lds = seqpar.unpack(torch.stack(outs), tuple(fin.shape), (w.batch, w.nheads))
    h_in = torch.empty_like(fin)
    names = ("forward", "logdecay", "combine", "correction")
    per = {r: {k: [] for k in names} for r in range(shards)}
    for it in range(reps + 2):
        for r, p in enumerate(parts):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            flush.zero_()
            ev[0].record(stream)
            ssd.ssd_chunk_scan_fwd(p["x"], p["dt"], A, p["B"], p["C"], D, w.chunk, y=y,
                                   final_states=fin, workspace=ws, stream=stream)
            ev[1].record(stream)
            ssd.ssd_seq_logdecay(p["dt"], A, stream=stream)
            ev[2].record(stream)
            ssd.ssd_state_exchange_combine(finals, lds, r, init_states=init, out=h_in,
                                           stream=stream)
            ev[3].record(stream)
            ssd.ssd_state_correction_fwd(h_in, p["dt"], A, p["C"], y, final_states=fin,
                                         workspace=cws, stream=stream)
            ev[4].record(stream)
            torch.cuda.synchronize(dev)
            if it >= 2:
                for i, k in enumerate(names):
                    per[r][k].append(ev[i].elapsed_time(ev[i + 1]))
    means = {r: {k: statistics.mean(v) for k, v in per[r].items()} for r in range(shards)}
    rank_ms = {r: sum(m.values()) for r, m in means.items()}
    slow = max(rank_ms, key=rank_ms.get)
    cb = correction_bytes(w, Ls)
    corr_ms = max(m["correction"] for m in means.values())
    del inp, parts, y, fin, ws, cws, finals, lds, h_in
    torch.cuda.empty_cache()
    return {"workload": w.name, "shards": shards, "tokens_per_shard": Ls,
            "ms_per_rank": rank_ms, "steps_ms_slowest_rank": means[slow],
            "tokens_per_s_if_parallel": w.tokens / (rank_ms[slow] * 1e-3),
            "correction": {"ms": corr_ms, "alg_bytes_if_all_tokens": cb,
                           "gbs_if_all_tokens": cb / (corr_ms * 1e-3) / 1e9,
                           "note": "tokens whose decay from the shard start underflowed to "
                                   "zero are skipped, so fewer bytes move than counted here"},
            "all_gather": "not timed: it needs one GPU per rank (b*H*(P*N+1) fp32 per rank)"}


# ---------------------------------------------------------------- per-kernel timing
FLOW_KERNELS = {1: ("chunk_state", "state_pass", "chunk_out"), 2: ("state_walk", "chunk_out"),
                3: ("walk_out",)}
FLOW_NAMES = {1: "three-kernel", 2: "walk+output", 3: "walk+output, one launch"}


def kernel_times(w, flow, inp, y, fin, dims, dev, stream, flush, reps):
    """Mean device time (ms) of each kernel of a tensor-core data flow, each
    launched through its own entry point, with CUDA events on the launching
    stream between the launches."""
    import ctypes

    import torch
    from ssd_chunked_scan_02_b200 import ssd
    x, dt, A, Bm, Cm, D, init = (inp[k] for k in ("x", "dt", "A", "B", "C", "D", "init"))
    T = (w.seqlen + w.chunk - 1) // w.chunk
    shape = (w.batch, T, w.nheads, w.headdim, w.dstate)
    prev_buf = torch.empty(shape, device=dev, dtype=x.dtype)
    S_buf = (torch.empty(shape, device=dev, dtype=torch.float32)
             if flow == ssd.SSD_FLOW_TC_THREE_KERNEL else None)
    ld_buf = torch.empty((w.batch, T, w.nheads), device=dev, dtype=torch.float32)
    lib = ssd.load()
    sp = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    names = FLOW_KERNELS[flow]
    kt = {k: [] for k in names}
    ws = None
    if flow == ssd.SSD_FLOW_WALK_OUTPUT_FUSED:
        # one launch (after the memset of its scheduling counters): the forward
        # itself, in that data flow
        ws = torch.empty(max(ssd.ssd_chunk_scan_fwd_workspace_size(dims, w.chunk, x.dtype,
                                                                   flow=flow), 16),
                         device=dev, dtype=torch.uint8)

    def launch(k):
        if k == "walk_out":
            st = lib.ssd_chunk_scan_fwd_with_flow(P(x), P(dt), P(A), P(Bm), P(Cm), P(D), w.chunk,
                                                  P(init), P(y), P(fin), ctypes.byref(dims),
                                                  ssd.SSD_BF16, P(ws), ws.numel(), sp, flow)
        elif k == "chunk_state":
            st = lib.ssd_chunk_state_fwd(P(x), P(dt), P(A), P(Bm), w.chunk, P(S_buf), P(ld_buf),
                                         ctypes.byref(dims), ssd.SSD_BF16, sp)
        elif k == "state_pass":
            st = lib.ssd_state_passing_fwd(P(S_buf), P(ld_buf), P(init), P(prev_buf), P(fin),
                                           w.chunk, ctypes.byref(dims), ssd.SSD_BF16, sp)
        elif k == "state_walk":
            st = lib.ssd_state_walk_fwd(P(x), P(dt), P(A), P(Bm), P(init), P(prev_buf), P(fin),
                                        w.chunk, ctypes.byref(dims), ssd.SSD_BF16, sp)
        else:
            st = lib.ssd_chunk_output_fwd(P(x), P(dt), P(A), P(Bm), P(Cm), P(D), P(prev_buf),
                                          w.chunk, P(y), ctypes.byref(dims), ssd.SSD_BF16, sp)
        if st != ssd.SSD_OK:
            raise RuntimeError(f"{k}: {ssd.status_name(st)}: {lib.ssd_last_error_detail()}")

    for r in range(reps + 2):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        flush.zero_()
        ev[0].record(stream)
        for i, k in enumerate(names):
            launch(k)
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        if r >= 2:
            for i, k in enumerate(names):
                kt[k].append(ev[i].elapsed_time(ev[i + 1]))
    del prev_buf, S_buf, ld_buf, ws
    return {k: statistics.mean(v) for k, v in kt.items()}


# ---------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the 130M-layer and length-sweep lines and the backward")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    import torch
    from ssd_chunked_scan_02_b200 import inputs, ssd

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()

    w = inputs.LAYER_2P7B
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 1000 * rank)
    inp = inputs.make_inputs(w, device=dev, gen=gen)
    x, dt, A, Bm, Cm, D, init = (inp[k] for k in ("x", "dt", "A", "B", "C", "D", "init"))
    y = torch.empty_like(x)
    fin = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), device=dev, dtype=torch.float32)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
    need = ssd.ssd_chunk_scan_fwd_workspace_size(dims, w.chunk, x.dtype)
    ws = torch.empty(need, device=dev, dtype=torch.uint8)
    flush = torch.empty(L2_FLUSH_BYTES, device=dev, dtype=torch.uint8)
    uses_tc = ssd.ssd_chunk_scan_fwd_uses_tensor_cores(dims, w.chunk, x.dtype) == 1

    def fwd():
        ssd.ssd_chunk_scan_fwd(x, dt, A, Bm, Cm, D, w.chunk, init_states=init, y=y,
                               final_states=fin, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        fwd()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for s, e in evs:
        flush.zero_()                      # L2 flush between timed steps (not timed)
        s.record(stream)
        fwd()
        e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in evs]
    total_ms = max_over_ranks(sum(step_ms), world)
    clocks = sampler.stop() if sampler else None
    ms_per_step = total_ms / args.steps

    # ---- per-kernel times: the kernels of the forward's data flow, launched
    # one by one through their entry points on the same stream, CUDA events
    # between them (L2 flushed before each sequence)
    flow = ssd.ssd_chunk_scan_fwd_data_flow(dims, w.chunk, x.dtype)
    kmean = kernel_times(w, flow, inp, y, fin, dims, dev, stream, flush, max(5, args.steps // 2))
    # the other tensor-core flow, for comparison (not part of the forward)
    alt_flow = {ssd.SSD_FLOW_WALK_OUTPUT_FUSED: ssd.SSD_FLOW_WALK_OUTPUT,
                ssd.SSD_FLOW_WALK_OUTPUT: ssd.SSD_FLOW_TC_THREE_KERNEL}.get(
                    flow, ssd.SSD_FLOW_WALK_OUTPUT)
    kalt = kernel_times(w, alt_flow, inp, y, fin, dims, dev, stream, flush,
                        max(5, args.steps // 4))
    dom = max(kmean, key=kmean.get)
    kb = kernel_bytes(w)
    dom_gbs = kb[dom][0] / (kmean[dom] * 1e-3) / 1e9
    dom_io_gbs = kb[dom][1] / (kmean[dom] * 1e-3) / 1e9

    # ---- decode step (b=256, H=80, P=64, N=128), state resident
    dw = inputs.DECODE_2P7B
    dgen = torch.Generator(device=dev)
    dgen.manual_seed(dw.seed + 1000 * rank)
    _, dpar = inputs.make_decode_params(dw, device=dev, gen=dgen)
    toks = [inputs.make_decode_token(dw, dgen, device=dev) for _ in range(4)]
    dstate = dpar["state"]
    ydec = torch.empty((dw.batch, dw.nheads, dw.headdim), device=dev, dtype=torch.bfloat16)

    def dstep(i):
        t = toks[i % len(toks)]
        ssd.ssd_step(dstate, t["x"], t["dt"], dpar["A"], t["B"], t["C"], dpar["D"], y=ydec,
                     stream=stream)
    for i in range(5):
        dstep(i)
    torch.cuda.synchronize(dev)
    dms = []
    for i in range(args.decode_steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        s.record(stream)
        dstep(i)
        e.record(stream)
        dms.append((s, e))
    torch.cuda.synchronize(dev)
    dec_ms = statistics.mean([s.elapsed_time(e) for s, e in dms])
    dec_bytes = (2 * 4 * dw.batch * dw.nheads * dw.headdim * dw.dstate
                 + dw.batch * dw.nheads * (2 * dw.headdim * 2 + 4)
                 + 2 * 2 * dw.batch * dw.ngroups * dw.dstate)
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
    y_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    f_host = torch.empty(fin.shape, dtype=fin.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for k, v in host.items()
              if v is not None and k not in ("A", "D")) + A.numel() * 4 + D.numel() * 4
    d2h = y.numel() * y.element_size() + fin.numel() * 4

    # Two device buffer sets and three streams: step k uploads into set k % 2
    # while step k - 1 computes and downloads, so host->device and
    # device->host copies (full duplex) and compute overlap across steps.
    # Every step still copies all of its inputs in and its y and final
    # states out; the timed region covers all of it.
    sets = [inp, {k: (torch.empty_like(v) if v is not None else None) for k, v in inp.items()}]
    outs = [(y, fin), (torch.empty_like(y), torch.empty_like(fin))]
    y_hosts = [y_host, torch.empty(y.shape, dtype=y.dtype, pin_memory=True)]
    f_hosts = [f_host, torch.empty(fin.shape, dtype=fin.dtype, pin_memory=True)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set j uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]    # forward on set j done
    ev_out = [torch.cuda.Event() for _ in range(2)]     # results of set j downloaded
    started = [False, False]

    def e2e_step(k):
        j = k & 1
        d_in, (yy, ff) = sets[j], outs[j]
        with torch.cuda.stream(s_in):
            if started[j]:
                s_in.wait_event(ev_used[j])
            for key in ("x", "dt", "B", "C", "init", "A", "D"):
                if host[key] is not None:
                    d_in[key].copy_(host[key], non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if started[j]:
            stream.wait_event(ev_out[j])
        ssd.ssd_chunk_scan_fwd(d_in["x"], d_in["dt"], d_in["A"], d_in["B"], d_in["C"], d_in["D"],
                               w.chunk, init_states=d_in["init"], y=yy, final_states=ff,
                               workspace=ws, stream=stream)
        ev_used[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_used[j])
            y_hosts[j].copy_(yy, non_blocking=True)
            f_hosts[j].copy_(ff, non_blocking=True)
            ev_out[j].record(s_out)
        started[j] = True

    for k in range(4):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_steps = max(8, args.steps // 2)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(s_in)
    for k in range(e2e_steps):
        e2e_step(k)
    s_in.wait_event(ev_out[(e2e_steps - 1) & 1])
    s_in.wait_event(ev_out[e2e_steps & 1])
    e.record(s_in)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s.elapsed_time(e), world) / e2e_steps
    # the link alone: one host->device copy of a step's input bytes and one
    # device->host copy of its output bytes (pinned buffers), each timed by
    # itself, to show what bounds the end-to-end number
    link = {}
    for name, nbytes, src_host in (("h2d", h2d, True), ("d2h", d2h, False)):
        hb = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
        db = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        ts = []
        for r in range(4):
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if src_host:
                db.copy_(hb, non_blocking=True)
            else:
                hb.copy_(db, non_blocking=True)
            z.record(stream)
            torch.cuda.synchronize(dev)
            if r:
                ts.append(a.elapsed_time(z))
        link[name] = {"ms": statistics.mean(ts), "gbs": nbytes / (statistics.mean(ts) * 1e-3) / 1e9}
        del hb, db

    # ---- the other configurations of the metric: 130M layer and the N = 64 sweep
    extra = None
    if not args.no_extra_configs:
        reps = max(3, args.steps // 4)
        extra = [measure_config(cw, dev, stream, flush, reps, world, rank)
                 for cw in (inputs.LAYER_130M,) + tuple(inputs.SWEEP)]
        for e in extra:
            e["hbm_frac_at_bytes_min"] = e["hbm_gbs_at_bytes_min"] / pk["hbm_gbs"]
            e["pct_bf16_peak_dense"] = 100 * e["tflops_dense"] / pk["bf16_tflops"]
    # ---- the backward (gradients), at the 130M-layer shape
    bwd = None
    if not args.no_extra_configs:
        bwd = measure_backward(inputs.LAYER_130M, dev, stream, flush, max(3, args.steps // 4),
                               world, rank, pk["hbm_gbs"])

    # ---- the sequence-parallel split (per-rank work, on this GPU)
    spl = None
    if not args.no_extra_configs and world == 1:
        spl = measure_seqpar(inputs.LAYER_2P7B, dev, stream, flush, max(3, args.steps // 4))
    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
        cpu = cpu_baselines(w, inp_cpu)

    if rank == 0:
        f_alg, f_dense, bytes_min = fwd_model(w)
        t = ms_per_step * 1e-3
        tok_s = weak_scaling_value(w.tokens, world, ms_per_step)
        t_roof = max(bytes_min / (pk["hbm_gbs"] * 1e9), f_dense / (pk["bf16_tflops"] * 1e12))
        bound = "hbm"
        peak_gbs = pk["hbm_gbs"]
        line = {
            "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                       "nheads": w.nheads, "headdim": w.headdim, "dstate": w.dstate,
                       "ngroups": w.ngroups, "chunk": w.chunk, "init_states": True,
                       "final_states": True, "tensor_cores": uses_tc,
                       "l2": "flushed (512 MiB write) before every timed step; inputs > L2"},
            "tflops": {"alg": f_alg / t / 1e12, "dense": f_dense / t / 1e12,
                       "pct_bf16_peak_dense": 100 * f_dense / t / 1e12 / pk["bf16_tflops"],
                       "pct_bf16_peak_alg": 100 * f_alg / t / 1e12 / pk["bf16_tflops"],
                       "peak_tflops": pk["bf16_tflops"], "peak_source": pk["source"]},
            "roofline_step": {"bound": "hbm", "bytes_min": bytes_min,
                              "achieved_gbs": bytes_min / t / 1e9,
                              "t_min_ms": 1e3 * t_roof, "frac": t_roof / t,
                              "note": "the whole forward against its minimum bytes: the "
                                      "headline roofline figure"},
            "roofline": {"bound": bound, "kernel": dom, "achieved": dom_gbs, "peak": peak_gbs,
                         "unit": "GB/s", "frac": dom_gbs / peak_gbs,
                         "traffic": traffic_for(dom, w.name),
                         "alg_bytes_per_launch": kb[dom][0],
                         "alg_bytes": "the kernel's share of bytes_min (layer inputs and "
                                      "outputs it touches, each once; intermediates count 0)",
                         "io_bytes_per_launch": kb[dom][1],
                         "io_gbs": dom_io_gbs, "io_frac": dom_io_gbs / peak_gbs,
                         "ms_per_launch": kmean[dom], "peak_source": pk["source"]},
            "data_flow": FLOW_NAMES.get(flow, "simt"),
            "kernels_ms": kmean,
            "kernels_ms_other_flow": kalt,
            "decode": {"workload": dw.name, "ms_per_step": dec_ms, "gbs": dec_gbs,
                       "frac_hbm": dec_gbs / peak_gbs, "bytes_per_step": dec_bytes},
            "e2e": {"value": world * w.tokens / (e2e_ms * 1e-3), "unit": UNIT,
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "device_ms_per_step": ms_per_step, "link": link,
                    "bound": "host<->device copies: the layer's input and output are as "
                             "large as its own HBM traffic, so the copies (h2d and d2h "
                             "overlapping, full duplex) take far longer than the forward"},
            "other_configs": extra,
            "backward": bwd,
            "seqpar": spl,
            "cpu_baseline": cpu,
            "gpu_launches": len(FLOW_KERNELS.get(flow, (0, 0, 0))) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
