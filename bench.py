#!/usr/bin/env python
"""Benchmark of the quantized recurrent-state decode step (one JSON line on rank 0).

A step is one decode step of one layer of the long-horizon, large-batch Gated
DeltaNet workload B=1024, H=16, d_k=d_v=128, packed INT4 state with
per-value-column scales, Philox stochastic rounding, bf16 q/k/v (the largest
workload that fits one GPU; --workload selects the others).  Consecutive steps cycle through enough independent layer states
(and input sets) that their footprint is >= 3x the L2 cache, as the layers of a
model do, so every step reads its state from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --drift [--workload W] [--drift-steps T] [--drift-every E]
  python bench.py --sweep [--steps K] [--jsonl results.jsonl]

N > 1 is launched by torchrun (one process per GPU); every rank runs its own
requests (weak scaling, no collective on the data path); the time is the max
over ranks.  --impl reference times the CPU oracle on the host cores instead.
--drift runs the long-horizon study instead (default: Gated DeltaNet B=1024,
H=16, d=128, 4096 steps): the relative state drift of INT4/INT8 trajectories
with stochastic and nearest rounding against the FP32 trajectory, every 256
steps, as one JSON line.  --sweep measures every row of the throughput table
(each workload and rounding, key-axis and window variant) in one process, one
line each; --jsonl appends every line to a file as well.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "gdn_b1024_h16_d128_int4_sr_long"
DRIFT_WORKLOAD = "gdn_b1024_h16_d128_int4_sr_long"


def algorithmic_bytes_per_head(w: W.Workload, bits: int, key_axis: bool = False) -> int:
    """Bytes the method must move per head update: codes and scales read and
    written, the input vectors and gates, and the float output."""
    esz = 2 if w.in_dtype == "bf16" else 4
    codes = w.dk * w.dv * bits // 8
    # a full-precision state has no scales; key-axis groups keep one per row
    scales = 0 if bits == 32 else 4 * (w.dk if key_axis else w.dv)
    out = 4 * w.dv
    if w.family == "gdn":
        vecs = esz * (2 * w.dk + w.dv) + 8          # q, k, v, alpha, beta
    elif w.family in ("gla", "kda"):
        vecs = esz * (2 * w.dk + w.dv) + 4 * w.dk + (4 if w.family == "kda" else 0)  # + decay vector
    else:
        vecs = esz * w.dv + 4                       # x, dt (B, C, A, D added per request / head)
    return 2 * codes + 2 * scales + vecs + out


def window_bytes_per_head(w: W.Workload, window: int) -> int:
    """Pure-write window traffic per head update: the FP8 a and b vectors and
    their scales, read and written."""
    return 2 * (window * (w.dk + w.dv) + 2 * 4 * window) if window else 0


def step_bytes(w: W.Workload, head_bits, window: int = 0, key_axis: bool = False) -> int:
    per = sum(algorithmic_bytes_per_head(w, int(b), key_axis) + window_bytes_per_head(w, window)
              for b in head_bits) * w.B
    if w.family == "mamba2":
        esz = 2 if w.in_dtype == "bf16" else 4
        per += w.B * w.ngroups * 2 * w.dk * esz + 8 * w.H   # B, C per request; A, D per head
    return per


def source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ssm_decode_02_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons, sampled every 100 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() in ("active", "1", "yes"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def emit(line: dict, args) -> None:
    """Print the result line; with --jsonl also append it to that file."""
    text = json.dumps(line)
    print(text, flush=True)
    if getattr(args, "jsonl", None):
        with open(args.jsonl, "a") as f:
            f.write(text + "\n")


# The rows of the throughput table: (workload, rounding or None, window, key-axis)
SWEEP = (
    ("gdn_b64_h16_d128_int8_sr", None, 0, False), ("gdn_b64_h16_d128_int8_sr", "rtn", 0, False),
    ("gdn_b64_h16_d128_int8_sr", "bdr", 0, False), ("gdn_b64_h16_d128_int8_sr", "sr_bdr", 0, False),
    ("gdn_b256_h32_d128_mixed_sr", None, 0, False), ("mamba2_b128_h80_p64_n128_int8_sr", None, 0, False),
    ("gdn_b1024_h16_d128_int4_sr_long", None, 0, False), ("gla_b64_h16_d128_int8_sr", None, 0, False),
    ("kda_b64_h16_d128_int8_sr", None, 0, False), ("gdn_b1024_h16_d128_int4_sr_long", "sr_bdr", 0, False),
    ("gdn_b64_h16_d128_int8_sr", None, 0, True), ("gdn_b64_h16_d128_int8_sr", "rtn", 0, True),
    ("gdn_b1024_h16_d128_int4_sr_long", None, 0, True), ("gdn_b64_h16_d128_int8_sr", None, 4, False),
    ("gdn_b64_h16_d128_int8_sr", None, 8, False), ("gdn_b64_h16_d128_int8_sr", None, 16, False),
    ("gdn_b1024_h16_d128_int4_sr_long", None, 8, False),
    ("gdn_b64_h8_d256_int8_sr", None, 0, False), ("gdn_b64_h8_d256_int8_sr", "rtn", 0, False),
    ("gdn_b64_h8_d256_int8_sr", "sr_bdr", 0, False), ("mamba2_b128_h80_p64_n256_int8_sr", None, 0, False),
    ("gdn_b64_h16_d128_int8_sr", "sr16", 0, False), ("gdn_b1024_h16_d128_int4_sr_long", "sr16", 0, False),
    ("gdn_b1024_h16_d128_int4_sr_long", "rtn", 0, False), ("gdn_b256_h32_d128_mixed_sr", "rtn", 0, False),
    ("mamba2_b128_h80_p64_n128_int8_sr", "rtn", 0, False), ("gdn_b64_h8_d256_int8_sr", "bdr", 0, False),
)


def run_sweep(args) -> int:
    """Every row of SWEEP on one GPU, one JSON line each (and --jsonl records)."""
    import copy
    import dataclasses
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print("--sweep runs on one GPU", file=sys.stderr)
        return 2
    for name, rounding, window, key_axis in SWEEP:
        a = copy.copy(args)
        a.window, a.key_axis, a.no_cpu_baseline = window, key_axis, True
        w = W.BY_NAME[name]
        if rounding:
            w = dataclasses.replace(w, rounding=rounding)
        rc = run_ours(a, w)
        if rc:
            return rc
    return 0


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (the timed interval of a
    multi-GPU run is the slowest rank's); identity without a process group."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_input_step(t: int, rank: int) -> int:
    """Input-generator step index of local step t on a rank: every rank serves its
    own requests (independent shards, no exchange), so the draws must differ."""
    return t + 100000 * rank


def measured_peak_gbs():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def profiled_traffic(workload: str, kernel_tag: str):
    """DRAM bytes per launch of `kernel_tag` on `workload` from a committed ncu
    summary, if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel") == kernel_tag and e.get("source_hash") == source_hash():
            return float(e["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        pass
    return None


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_rate(w: W.Workload, head_bits, budget_s: float, heads_per_call: int = 8):
    """Head updates per second of the single-threaded CPU oracle on a bounded sample
    of the workload (the first requests of a few steps, from the zero state)."""
    import oracle
    R = 8 if w.dk <= 128 else 16
    rounding = ROUNDING[w.rounding]
    n_done, t_used, t = 0, 0.0, 0
    nb = max(1, min(w.B, heads_per_call // w.H + 1))
    st = oracle.zero_state(nb, w.H, w.dk, w.dv, fp32=w.state == "fp32")
    while t_used < budget_s:
        inp = W.inputs(w, t, B=nb)
        heads = [(b, h) for b in range(nb) for h in range(w.H)][:heads_per_call]
        t0 = time.perf_counter()
        st, _ = _oracle_step(oracle, w, st, inp, head_bits, rounding, t, R, heads)
        t_used += time.perf_counter() - t0
        n_done += len(heads)
        t += 1
    return n_done / t_used, n_done, t


def _oracle_rate_job(job):
    w, bits, budget_s = job
    rate, n, _ = oracle_rate(w, bits, budget_s)
    return n, n / rate


def oracle_rate_all_cores(w: W.Workload, head_bits, budget_s: float):
    """The same oracle sample run by one spawned process per host core at once
    (each core its own heads): head updates of all processes / the longest
    process time.  Returns (rate, processes)."""
    import multiprocessing as mp
    n = max(1, os.cpu_count() or 1)
    with mp.get_context("spawn").Pool(n) as pool:
        res = pool.map(_oracle_rate_job, [(w, head_bits, budget_s)] * n)
    return sum(r[0] for r in res) / max(r[1] for r in res), n


def _oracle_step(oracle, w: W.Workload, st, inp, bits, rounding, t, R, heads):
    kw = dict(rounding=rounding, seed=w.sr_seed, step=t, R=R, heads=heads)
    if w.family == "gdn":
        return oracle.gdn_step(st, inp, bits, **kw)
    if w.family == "gla":
        return oracle.gla_step(st, inp, bits, **kw)
    if w.family == "kda":
        return oracle.kda_step(st, inp, bits, **kw)
    return oracle.mamba2_step(st, inp, bits, ngroups=w.ngroups, **kw)


FAMILY = {"gdn": 0, "mamba2": 1, "gla": 2, "kda": 3}   # rsq_family values


def head_bits_of(w: W.Workload, rsq=None):
    if w.state == "mixed":
        score = W.mean_alpha_per_head(w)
        n_hi = int(w.H * w.high_frac)
        if rsq is not None:
            return rsq.rsq_allocate_bits(score, n_hi)
        import oracle
        return oracle.allocate_bits(score, n_hi)
    return W.head_bits_for(w)


def run_reference(args, w: W.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    bits = head_bits_of(w)
    # time one oracle head to size the per-step sample so the whole run stays within minutes
    rate, _, _ = oracle_rate(w, bits, 0.5, heads_per_call=1)
    per_head = 1.0 / rate
    total_budget = 180.0
    n_heads = int(max(1, min(w.B * w.H, total_budget / max(1, args.steps + args.warmup) / per_head)))
    import oracle
    R = 8 if w.dk <= 128 else 16
    rounding = ROUNDING[w.rounding]
    nb = max(1, min(w.B, (n_heads + w.H - 1) // w.H))
    heads = [(b, h) for b in range(nb) for h in range(w.H)][:n_heads]
    st = oracle.zero_state(nb, w.H, w.dk, w.dv, fp32=w.state == "fp32")
    inp_cache = [W.inputs(w, t, B=nb) for t in range(4)]
    elapsed = 0.0
    for t in range(args.warmup + args.steps):
        inp = inp_cache[t % 4]
        t0 = time.perf_counter()
        st, _ = _oracle_step(oracle, w, st, inp, bits, rounding, t, R, heads)
        dt = time.perf_counter() - t0
        if t >= args.warmup:
            elapsed += dt
    value = n_heads * args.steps / elapsed
    line = {
        "impl": "reference", "metric": "head-updates/s", "value": value, "unit": "head-updates/s",
        "n_gpus": args.gpus, "runs_on": "host CPU, rank 0 only (the oracle uses no GPU)",
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * elapsed / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B, "heads": w.H, "dk": w.dk, "dv": w.dv,
                   "state": w.state, "rounding": w.rounding, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "head-updates/s", "cores": 1, "kind": "oracle",
                         "sample": "%d heads of one layer per step, single-threaded C oracle" % n_heads},
        "e2e": {"value": value, "unit": "head-updates/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    emit(line, args)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, w: W.Workload):
    import torch
    import torch.distributed as dist
    from torch.cuda import nvtx  # ranges rsq.warmup / rsq.timed / rsq.l2_hot / rsq.e2e for ncu --nvtx

    import ssm_decode_02_b200 as rsq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))

    bits = np.asarray(head_bits_of(w, rsq), np.int8)
    fam = FAMILY[w.family]
    ctx = rsq.Context(fam, w.B, w.H, w.dk, w.dv, head_bits=bits,
                      rounding=ROUNDING[w.rounding],
                      in_dtype=rsq.RSQ_BF16 if w.in_dtype == "bf16" else rsq.RSQ_F32,
                      seed=w.sr_seed + 7919 * rank, ngroups=w.ngroups, window=args.window,
                      key_axis=int(args.key_axis))
    state_bytes = ctx.code_bytes + ctx.scale_bytes
    layers = max(2, -(-3 * l2 // state_bytes))
    if args.layers:
        layers = args.layers
    # independent layer states, initialised from random full-precision states
    states = []
    S0 = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + rank)
    for _ in range(layers):
        st = ctx.alloc_state(dev)
        S0.normal_(0.0, 0.05, generator=g)
        ctx.quantize(S0, st, step=0)
        states.append(st)
    del S0
    # pure-write windows: a ping-pong pair per layer (the step reads one, writes the other)
    wins = [(ctx.alloc_window(dev), ctx.alloc_window(dev)) for _ in range(layers)] if args.window else None
    # input sets (seeded host generation, uploaded once)
    inp_bytes = None
    n_sets = max(8, min(256, -(-3 * l2 // max(1, step_input_bytes(w)))))
    sets = []
    for t in range(n_sets):
        host = W.inputs(w, rank_input_step(t, rank))
        d = {k: _to_dev(v, dev) for k, v in host.items()}
        sets.append(d)
    inp_bytes = step_input_bytes(w)
    outs = [torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device=dev) for _ in range(layers)]
    structs = [_inputs_struct(rsq, w, s) for s in sets]
    stream = torch.cuda.Stream(device=dev)

    def step_on(li, ins, t, visit):
        """One decode step of layer li (its window ping-pong by visit parity)."""
        if wins is None:
            ctx.decode_step(states[li], states[li], ins, outs[li], t, stream.cuda_stream)
        else:
            ctx.decode_step_window(states[li], states[li], wins[li][visit % 2], wins[li][(visit + 1) % 2],
                                   ins, outs[li], t, stream.cuda_stream)

    def launch(t):
        step_on(t % layers, structs[t % n_sets], t, t // layers)

    # CUDA graphs of up to CH consecutive steps (launch-bound inner loop); CH is a
    # multiple of the layer count so the rotation continues across graph replays
    # (an even number of visits per layer, so the window ping-pong ends where it began)
    CH = 2 * max(1, (args.chunk or 1024) // layers) * layers

    def capture(t0, n):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(gr, stream=stream):
                for t in range(t0, t0 + n):
                    launch(t)
        return gr

    with torch.cuda.stream(stream):
        for t in range(min(8, args.warmup)):
            launch(t)
    stream.synchronize()
    if ctx.check_flags(stream.cuda_stream):
        raise RuntimeError("non-finite state during warm-up")

    def plan(total):
        chunks, t = [], 0
        while t < total:
            n = min(CH, total - t)
            chunks.append((t, n))
            t += n
        return chunks

    warm_graphs = [capture(t0, n) for t0, n in plan(args.warmup)]
    timed_plan = plan(args.steps)
    # distinct graphs for distinct chunk sizes; step numbers only matter for the SR counter
    graph_cache = {}
    for t0, n in timed_plan:
        if n not in graph_cache:
            graph_cache[n] = capture(args.warmup, n)
    uuid = str(getattr(props, "uuid", ""))
    clocks = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local)))
    clocks.start()
    time.sleep(0.3)
    # graphs replay on the current stream: make it the timed stream
    with torch.cuda.stream(stream), nvtx.range("rsq.warmup"):
        for gr in warm_graphs:
            gr.replay()
        # every graph the timed region replays runs once first, so its upload and
        # first-launch cost stay outside the timed region
        for gr in graph_cache.values():
            gr.replay()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream), nvtx.range("rsq.timed"):
        ev0.record(stream)
        for t0, n in timed_plan:
            graph_cache[n].replay()
        ev1.record(stream)
    ev1.synchronize()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    time.sleep(0.15)
    clk = clocks.stop()
    elapsed = max_over_ranks(ev0.elapsed_time(ev1) / 1e3, dist if world > 1 else None, dev)
    flag = ctx.check_flags(stream.cuda_stream)

    # L2-hot reference point (labelled, not the headline): one layer state and one
    # input set, so the whole step's working set stays in L2
    n_hot = 2 * max(1, min(args.steps, 2000) // 2)
    hot = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(hot, stream=stream):
            for t in range(n_hot):
                step_on(0, structs[0], args.warmup + t, t)
        hot.replay()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx.range("rsq.l2_hot"):
            h0.record(stream)
            hot.replay()
            h1.record(stream)
    h1.synchronize()
    hot_ms = h0.elapsed_time(h1) / n_hot
    del hot

    # end-to-end through the public API with host buffers (pinned), per step:
    # the library's host-buffer pipeline (rsq_pipe) copies the step's packed
    # inputs in, runs the decode step and copies its output back, with three
    # steps in flight on its own copy-in / compute / copy-out streams, as a
    # server would, over the same rotating layer states as the timed region.
    # Timed with events on the pipe's streams.
    n_e2e = max(2, min(args.steps, 500))
    pipe = rsq.Pipe(ctx)
    host_in = [rsq.pack_host_inputs(ctx, W.inputs(w, rank_input_step(200000 + t, rank))) for t in range(4)]
    h2d = host_in[0].numel()
    host_out = [torch.empty((w.B, w.H, w.dv), dtype=torch.float32, pin_memory=True) for _ in range(4)]
    d2h = host_out[0].numel() * 4
    s_in = torch.cuda.ExternalStream(pipe.copy_in, device=dev)
    s_out = torch.cuda.ExternalStream(pipe.copy_out, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    nvtx.range_push("rsq.e2e")
    e0.record(s_in)
    for t in range(n_e2e):
        # the layer states rotate as in the timed region, so every step reads
        # its state from HBM
        step_t, li, visit = args.warmup + args.steps + t, t % layers, t // layers
        if wins is None:
            pipe.step(states[li], states[li], host_in[t % 4], host_out[t % 4], step_t)
        else:
            pipe.step(states[li], states[li], host_in[t % 4], host_out[t % 4], step_t,
                      wins[li][visit % 2], wins[li][(visit + 1) % 2])
    # the last output copy follows every earlier copy and kernel of the pipe
    e1.record(s_out)
    nvtx.range_pop()
    e1.synchronize()
    pipe.sync()
    pipe.close()
    e2e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, dev)

    hu_step = w.B * w.H
    value = world * hu_step * args.steps / elapsed
    e2e_value = world * hu_step * n_e2e / e2e_elapsed
    per_launch = elapsed / args.steps
    alg = step_bytes(w, bits, args.window, bool(args.key_axis))
    peak, peak_kind = measured_peak_gbs()
    achieved = alg / per_launch / 1e9
    kernel_tag = "rsq_decode_kernel<%s,dk=%d,blocks=%d,%s>" % (w.family, w.dk, min(4, w.dv // 16),
                                                                 "fp32" if w.state == "fp32" else w.rounding)
    line = {
        "metric": "head-updates/s", "value": value, "unit": "head-updates/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * per_launch,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B * world, "heads": w.H, "dk": w.dk,
                   "dv": w.dv, "state": w.state, "rounding": w.rounding, "inputs": w.in_dtype,
                   "window": args.window, "scale_groups": "key-axis" if args.key_axis else "value-axis",
                   "parallelism": "dp%d" % world, "layers_rotated": layers,
                   "l2": "inputs larger than L2: %d layer states + %d input sets = %.0f MB per "
                         "rotation (L2 %.0f MB)" % (layers, n_sets,
                                                    (layers * state_bytes + n_sets * inp_bytes) / 1e6,
                                                    l2 / 1e6),
                   "graphs": "CUDA graphs of <= %d steps" % CH},
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": (profiled_traffic(w.name, kernel_tag)
                                 if not (args.window or args.key_axis or getattr(args, "state", None))
                                 else None),
                     "algorithmic_bytes_per_launch": alg, "kernel": kernel_tag},
        "frac_of_8tbs_datasheet": achieved / 8000.0,
        "e2e": {"value": e2e_value, "unit": "head-updates/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e,
                "path": "rsq_pipe (pinned host buffers, 3 steps in flight), rotating layer states"},
        "l2_hot": {"ms_per_step": hot_ms, "steps": n_hot,
                   "setup": "one layer state and one input set, resident in L2 (not the headline)"},
        "gpu_launches": args.steps,
        "wall_s_timed_region": wall,
        "clocks": clk,
        "nonfinite_flag": flag,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, steps = oracle_rate(w, bits, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "head-updates/s", "cores": 1, "kind": "oracle",
                                "sample": "%d head updates (%d decode steps of the first requests) "
                                          "in ~%.0f s, single-threaded C oracle" % (n, steps, args.cpu_seconds)}
        rate_all, procs = oracle_rate_all_cores(w, bits, args.cpu_seconds)
        line["cpu_baseline_all_cores"] = {
            "value": rate_all, "unit": "head-updates/s", "cores": procs, "kind": "oracle",
            "sample": "the same sample in %d concurrent processes (one per host core), ~%.0f s each"
                      % (procs, args.cpu_seconds)}
    if rank == 0:
        emit(line, args)
    for gr in list(graph_cache.values()) + warm_graphs:
        del gr
    graph_cache.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    ctx.close()
    return 0


# ---------------------------------------------------------------------------
# Long-horizon state drift (quantized trajectories against the FP32 trajectory)
# ---------------------------------------------------------------------------
# (label, bits, rounding, variant): "noisy" = the quantized state's own column
# maxima as scales, "copy" = the column maxima of the FP32 trajectory, "wN" = a
# pure-write window of N FP8 slots beside the low-bit history (GDN),
# "keyaxis" = one scale per key row instead of per value column (GDN)
DRIFT_VARIANTS = (("int4_sr", 4, "sr", "noisy"), ("int4_rtn", 4, "rtn", "noisy"),
                  ("int4_bdr", 4, "bdr", "noisy"), ("int4_sr_bdr", 4, "sr_bdr", "noisy"),
                  ("int4_sr_copy", 4, "sr", "copy"), ("int4_rtn_copy", 4, "rtn", "copy"),
                  ("int4_sr_w8", 4, "sr", "w8"), ("int4_rtn_w8", 4, "rtn", "w8"),
                  ("int8_sr", 8, "sr", "noisy"), ("int8_rtn", 8, "rtn", "noisy"),
                  ("int8_bdr", 8, "bdr", "noisy"), ("int8_sr_copy", 8, "sr", "copy"),
                  ("int8_sr_w8", 8, "sr", "w8"),
                  ("int4_sr_keyaxis", 4, "sr", "keyaxis"), ("int4_rtn_keyaxis", 4, "rtn", "keyaxis"),
                  ("int8_sr_keyaxis", 8, "sr", "keyaxis"))
# rsq_rounding values; "sr" is stochastic rounding with 8-bit uniforms, "sr16"
# the same with 16-bit uniforms
ROUNDING = {"rtn": 0, "sr": 5, "bdr": 2, "sr_bdr": 7, "sr16": 1, "sr16_bdr": 3}


def _drift_inputs(job):
    w, B, t = job
    return t, W.inputs(w, t, B=B)


def drift_series(w: W.Workload, steps: int, every: int, B: int | None = None, variants=DRIFT_VARIANTS,
                 pool=None, device="cuda") -> dict:
    """Relative state drift ||deq(S_q) - S_fp32||_F / ||S_fp32||_F of quantized
    trajectories against the full-precision trajectory run by the same kernel
    with 32-bit heads, all from S_0 = 0 on identical inputs, sampled every
    `every` steps.  Also the relative error of the readout at those steps.
    Variants with the "copy" scale source take each step's scales from the
    FP32 trajectory's column maxima instead of their own state.

    Returns {label: [[t, global drift, max per-head drift, readout error], ...]}."""
    import torch

    import ssm_decode_02_b200 as rsq

    B = w.B if B is None else B
    fam = FAMILY[w.family]
    in_dtype = rsq.RSQ_BF16 if w.in_dtype == "bf16" else rsq.RSQ_F32

    def make(bits, rounding, window=0, key_axis=0):
        ctx = rsq.Context(fam, B, w.H, w.dk, w.dv, head_bits=np.full(w.H, bits, np.int8),
                          rounding=ROUNDING[rounding],
                          in_dtype=in_dtype, seed=w.sr_seed, ngroups=w.ngroups, window=window,
                          key_axis=key_axis)
        st = ctx.alloc_state(device)
        ctx.quantize(torch.zeros((B, w.H, w.dk, w.dv), dtype=torch.float32, device=device), st)
        out = torch.empty((B, w.H, w.dv), dtype=torch.float32, device=device)
        return ctx, st, out

    def window_of(src):
        return int(src[1:]) if src.startswith("w") else 0

    ref = make(32, "rtn")
    runs = {label: make(bits, rnd, window_of(src), int(src == "keyaxis")) for label, bits, rnd, src in variants}
    source = {label: src for label, _, _, src in variants}
    wins = {label: [runs[label][0].alloc_window(device), runs[label][0].alloc_window(device)]
            for label, _, _, src in variants if window_of(src)}
    copy_max = torch.empty((B, w.H, w.dv), dtype=torch.float32, device=device)
    sums = torch.empty((B, w.H, 2), dtype=torch.float64, device=device)
    series = {label: [] for label, _, _, _ in variants}
    jobs = [(w, B, t) for t in range(steps)]
    it = pool.imap(_drift_inputs, jobs, chunksize=2) if pool is not None else map(_drift_inputs, jobs)
    for t, host in it:
        d = {k: _to_dev(v, device) for k, v in host.items()}
        ins = _inputs_struct(rsq, w, d)
        ref[0].decode_step(ref[1], ref[1], ins, ref[2], t)
        ref[0].column_absmax(ref[1], copy_max)
        for label, (ctx, st, out) in runs.items():
            if source[label] == "copy":
                ctx.decode_step_copy_scale(st, st, ins, copy_max, out, t)
            elif label in wins:
                ctx.decode_step_window(st, st, wins[label][t % 2], wins[label][(t + 1) % 2], ins, out, t)
            else:
                ctx.decode_step(st, st, ins, out, t)
        if (t + 1) % every == 0:
            o_ref = ref[2].double()
            for label, (ctx, st, out) in runs.items():
                if label in wins or source[label] == "keyaxis":
                    num, den = _full_drift_sums(ctx, st, wins[label][(t + 1) % 2] if label in wins else None,
                                                ref, B, w, device)
                else:
                    rsq.rsq_state_drift(ctx.ctx, st, ref[0].ctx, ref[1], sums)
                    s = sums.cpu().numpy()
                    num, den = s[..., 0], s[..., 1]
                per_head = np.sqrt(num[den > 0] / den[den > 0])
                o_err = float(torch.linalg.vector_norm(out.double() - o_ref) /
                              torch.linalg.vector_norm(o_ref))
                series[label].append([t + 1, float(np.sqrt(num.sum() / den.sum())),
                                      float(per_head.max()) if per_head.size else 0.0, o_err])
    for ctx, _, _ in [ref] + list(runs.values()):
        if ctx.check_flags():
            raise RuntimeError("non-finite state in the drift study")
        ctx.close()
    return series


def _full_drift_sums(ctx, st, win, ref, B, w, device):
    """Per-head sums of (state - FP32 state)^2 and FP32 state^2 through the
    library's dequantization (any scale grouping); with a pure-write window the
    state is the dequantized history + sum_w a_w b_w^T."""
    import torch
    Hq = torch.empty((B, w.H, w.dk, w.dv), dtype=torch.float32, device=device)
    F = torch.empty_like(Hq)
    ctx.dequantize(st, Hq)
    ref[0].dequantize(ref[1], F)
    full = Hq.double()
    if win is not None:
        Wn = ctx.window
        dec = lambda codes: codes.view(torch.float8_e4m3fn).to(torch.float32)
        a = dec(win.a) * win.a_scale[..., None]                                   # [B][H][W][dk]
        b = dec(win.b).permute(0, 1, 3, 2, 4).reshape(B, w.H, Wn, w.dv) * win.b_scale[..., None]
        full = full + torch.einsum("bhwi,bhwj->bhij", a.double(), b.double())
    F = F.double()
    num = ((full - F) ** 2).sum(dim=(2, 3)).cpu().numpy()
    den = (F ** 2).sum(dim=(2, 3)).cpu().numpy()
    return num, den


def run_drift(args, w: W.Workload, pool) -> int:
    import torch
    torch.cuda.set_device(0)
    steps = args.drift_steps or w.steps
    t0 = time.perf_counter()
    series = drift_series(w, steps, args.drift_every, pool=pool)
    line = {
        "metric": "relative state drift ||deq(S_q) - S_fp32||_F / ||S_fp32||_F",
        "workload": w.name, "batch": w.B, "heads": w.H, "dk": w.dk, "dv": w.dv, "steps": steps,
        "every": args.drift_every, "start": "S_0 = 0",
        "reference": "FP32 trajectory: the same kernel with 32-bit heads, identical inputs",
        "columns": ["step", "global drift", "max per-head drift", "readout relative error"],
        "series": series, "input_workers": getattr(pool, "_processes", 0),
        "wall_s": time.perf_counter() - t0,
    }
    emit(line, args)
    return 0


def step_input_bytes(w: W.Workload) -> int:
    esz = 2 if w.in_dtype == "bf16" else 4
    if w.family == "gdn":
        return w.B * w.H * (esz * (2 * w.dk + w.dv) + 8)
    if w.family in ("gla", "kda"):
        return w.B * w.H * (esz * (2 * w.dk + w.dv) + 4 * w.dk + (4 if w.family == "kda" else 0))
    return w.B * w.H * (esz * w.dv + 4) + w.B * w.ngroups * 2 * w.dk * esz + 8 * w.H


def _to_dev(a: np.ndarray, dev):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a.copy()).to(dev)


def _to_pinned(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a.copy()).pin_memory()


def _inputs_struct(rsq, w: W.Workload, d: dict):
    if w.family == "gdn":
        return rsq.gdn_inputs(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    if w.family in ("gla", "kda"):
        return rsq.diag_inputs(d["q"], d["k"], d["v"], d["alpha"], d.get("beta"))
    return rsq.mamba2_inputs(d["x"], d["Bm"], d["Cm"], d["dt"], d["A"], d["D"], None)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, choices=sorted(W.BY_NAME),
                    help="default: %s (the drift study: %s)" % (DEFAULT_WORKLOAD, DRIFT_WORKLOAD))
    ap.add_argument("--layers", type=int, default=0, help="override the number of rotated layer states")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--rounding", choices=sorted(ROUNDING), default=None,
                    help="override the workload's requantization rule")
    ap.add_argument("--state", choices=["int8", "int4", "fp32"], default=None,
                    help="override the workload's state format with one width for every head")
    ap.add_argument("--window", type=int, default=0,
                    help="pure-write window slots (Gated DeltaNet): 0, 4, 8 or 16")
    ap.add_argument("--key-axis", action="store_true",
                    help="one scale per key row instead of per value column (Gated DeltaNet)")
    ap.add_argument("--drift", action="store_true",
                    help="run the long-horizon state drift study instead of the throughput bench")
    ap.add_argument("--drift-steps", type=int, default=0, help="horizon (default: the workload's)")
    ap.add_argument("--drift-every", type=int, default=256)
    ap.add_argument("--jsonl", default=None, help="also append each result line to this file")
    ap.add_argument("--seed", type=int, default=None, help="override the workload's stochastic-rounding seed")
    ap.add_argument("--chunk", type=int, default=0,
                    help="steps per captured CUDA graph (rounded to an even number of visits per layer)")
    ap.add_argument("--sweep", action="store_true",
                    help="measure every row of the throughput table (one GPU), one line each")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.workload is None:
        args.workload = DRIFT_WORKLOAD if args.drift else DEFAULT_WORKLOAD
    if args.sweep:
        return run_sweep(args)
    if args.drift:
        w = W.BY_NAME[args.workload]
        # the input generator pool starts before the first CUDA call
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(max(1, min(32, (os.cpu_count() or 2) - 1))) as pool:
            return run_drift(args, w, pool)
    w = W.BY_NAME[args.workload]
    if args.rounding or args.seed is not None or args.state:
        import dataclasses
        if args.rounding:
            w = dataclasses.replace(w, rounding=args.rounding)
        if args.seed is not None:
            w = dataclasses.replace(w, sr_seed=args.seed)
        if args.state:
            w = dataclasses.replace(w, state=args.state)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
