#!/usr/bin/env python
"""Benchmark of the Mamba-3 SSM forward on B200: prefill scan tokens/s (the
headline line) plus the decode step, each with its roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one m3_scan_fwd over the whole batch of the SISO bf16 prefill
workload (batch 8, T=4096, 32 heads, P=64, N=128, R=1), inputs resident in
HBM (943 MB per step, larger than the 126 MB L2, so no flush is needed).
With N > 1 (torchrun) every rank runs its own batch (weak scaling, replicas:
the (batch, head) slices are independent, there is no collective on the data
path); time is the max over ranks of CUDA-event time.  Rank 0 prints one JSON
line.  `--impl reference` times the fp64 CPU oracle on bounded samples of the
same workload instead (rank 0 only).

Besides the headline the line carries `configs`: every workload the method is
measured on, each timed on its own with CUDA events and its own roofline --
the small fp32 scan (batch 1, T=256, 4 heads, P=N=64; smaller than L2, so
L2 is flushed between calls), the SISO prefill (the headline itself), the
MIMO rank-4 prefill (batch 8, T=4096, 32 heads, N=64), the batch-256 decode
steps (rank 1 and rank 4, 1000 graph-captured steps from a 1024-token
prefill) and the long-context MIMO prefill (batch 1, T=65536, 64 heads,
N=128, R=4) followed by 256 decode steps of its own sequences.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Mamba-3 SSM tokens/s (prefill scan, decode step) and % of roofline, 1 B200"
PREFILL_WORKLOAD = "siso_bf16_b8_t4096_h32_p64_n128"
DECODE_WORKLOADS = ["decode_bf16_b256_h32_p64_n128_r1", "decode_bf16_b256_h32_p64_n128_r4"]
# the five workloads the method is measured on, in order (the decode entry
# stands for both ranks of DECODE_WORKLOADS)
CONFIG_WORKLOADS = ["siso_f32_b1_t256_h4_p64_n64", PREFILL_WORKLOAD, "mimo_bf16_b8_t4096_h32_p64_n64_r4",
                    DECODE_WORKLOADS[0], "long_mimo_bf16_b1_t65536_h64_p64_n128_r4"]
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser(description="Mamba-3 SSM forward benchmark: one JSON line on stdout (rank 0).")
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one process each, launched by torchrun for N > 1)")
    ap.add_argument("--steps", type=int, default=20, help="timed steps")
    ap.add_argument("--warmup", type=int, default=5, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="ours: the CUDA library; reference: the fp64 oracle on the host cores")
    ap.add_argument("--workload", default=PREFILL_WORKLOAD, help="prefill workload (a name in m3_inputs.WORKLOADS)")
    ap.add_argument("--algo", choices=["auto", "simt", "tc"], default="auto", help="prefill kernel choice")
    ap.add_argument("--decode-steps", type=int, default=1000, help="graph-captured steps of the decode lines")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode lines")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the variant lines (per-token A, per-head theta, BC-norm) of the prefill workload")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' lines (small fp32 scan, MIMO, decode, long context)")
    ap.add_argument("--case", choices=["prefill", "prefill_proj", "prefill_a_per_token", "prefill_theta_per_head",
                                       "prefill_bcnorm", "decode"], default=None,
                    help="profiling case: only run --case-launches launches of one kernel at --case-batch "
                         "(for ncu captures; prints no bench line); prefill_<variant> runs the workload "
                         "with that variant's layout or prologue")
    ap.add_argument("--case-batch", type=int, default=None, help="batch of the profiling case")
    ap.add_argument("--case-seqlen", type=int, default=None, help="sequence length of the profiling case")
    ap.add_argument("--case-launches", type=int, default=3, help="launches of the profiling case")
    ap.add_argument("--compare-fp32", action="store_true",
                    help="kernel study: the fp32 tensor-core prefill against the SIMT kernel on fp32 shapes "
                         "(one JSON line per shape; prints no bench line)")
    return ap.parse_args()


def run_case(args):
    """Small fixed case for ncu captures: the workload's shape at a reduced
    batch, a few launches of the one kernel, no timing."""
    import torch

    import state_space_sequence_ssm_b200 as m3
    from m3_inputs import WORKLOADS, make_prefill, make_state, make_steps

    keys = ("x", "B", "C", "dt", "lam", "theta", "A", "D")
    if args.case.startswith("prefill"):
        s = WORKLOADS[args.workload]
        s = s.with_(batch=args.case_batch or s.batch, seqlen=args.case_seqlen or s.seqlen)
        kind = args.case[len("prefill_"):]
        proj = bcn = None
        if kind == "proj":  # the same shape with the fused MIMO projections
            from m3_inputs import make_prefill_proj, make_proj
            inp = make_prefill_proj(s, device="cuda")
            w = make_proj(s, device="cuda")
            proj = m3.MimoProj(w["wx"], w["wB"], w["wC"], w["wy"])
        elif kind in ("a_per_token", "theta_per_head"):
            inp = make_prefill(s, device="cuda", **{kind: True})
        else:
            inp = make_prefill(s, device="cuda")
        if kind == "bcnorm":
            from m3_inputs import make_bcnorm
            p = make_bcnorm(s, device="cuda")
            bcn = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
        for _ in range(args.case_launches):
            m3.scan_fwd(*(inp[k] for k in keys), None, proj=proj, bcnorm=bcn)
    else:
        # a decode workload, or the long-context workload's own sequences
        name = args.workload if args.workload.startswith(("decode", "long")) else DECODE_WORKLOADS[0]
        s = WORKLOADS[name]
        s = s.with_(batch=args.case_batch or s.batch)
        st = m3.State(*(t.cuda() for t in make_state(s)))
        steps = make_steps(s, args.case_launches, device="cuda")
        pre = make_prefill(s.with_(seqlen=1), device="cuda")
        for i in range(args.case_launches):
            m3.step(*(steps[k][i] for k in keys[:6]), pre["A"], pre["D"], st)
    m3.stream_status()
    torch.cuda.synchronize()
    print(f"case {args.case} {s} x{args.case_launches} done")


def run_compare_fp32(args):
    """Both prefill kernels that take fp32 I/O on the same inputs: the small
    fp32 workload and the SISO workload's batch, length and heads at
    dstate 64 (ranks 1, 2, 4).  Median of --steps calls, each timed alone
    with CUDA events after a 256 MiB write that flushes L2."""
    import dataclasses

    import torch

    import state_space_sequence_ssm_b200 as m3
    from m3_inputs import WORKLOADS, make_prefill

    keys = ("x", "B", "C", "dt", "lam", "theta", "A", "D")
    hbm, src = peaks()
    big = WORKLOADS[PREFILL_WORKLOAD]
    shapes = [WORKLOADS["siso_f32_b1_t256_h4_p64_n64"]] + [
        big.with_(dstate=64, rank=r, io="f32") for r in (1, 2, 4)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for s in shapes:
        inp = make_prefill(s, device="cuda")
        y = torch.empty_like(inp["x"])
        fin = m3.empty_state(s.batch, s.nheads, s.dstate, s.headdim, s.rank, device="cuda")
        dims = m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)
        line = {"study": "fp32 prefill kernels", "shape": dataclasses.asdict(s),
                "algorithmic_bytes": prefill_bytes(s), "peak_gbs": hbm, "peak_source": src}
        for name, algo in (("tc", m3.ALGO_TC), ("simt", m3.ALGO_SIMT)):
            line[name + "_kernel"] = m3.scan_plan_info(dims, algo).kernel_name
            for _ in range(max(args.warmup, 3)):
                m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, algo=algo)
            ts = []
            for i in range(args.steps):
                flush.fill_(i & 0xff)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, algo=algo)
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            m3.stream_status()
            ms = statistics.median(ts)
            line[name + "_ms"] = ms
            line[name + "_frac"] = prefill_bytes(s) / (ms * 1e-3) / 1e9 / hbm
        line["speedup"] = line["simt_ms"] / line["tc_ms"]
        print(json.dumps(line, default=str), flush=True)
        del inp, y, fin


# ---------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (earlier measurement on this pool)"


def file_hash(paths):
    h = hashlib.sha256()
    for p in sorted(paths):
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def kernel_sources(kernel):
    csrc = os.path.join(ROOT, "state_space_sequence_ssm_b200", "csrc")
    files = {"prefill_simt_kernel": ["prefill_simt.cu"], "step_kernel": ["decode.cu"],
             "step_stream_kernel": ["decode.cu"],
             "prefill_tc_kernel": ["prefill_tc.cu", "tc_primitives.cuh"],
             "prefill_tc32_kernel": ["prefill_tc32.cu", "tc_primitives.cuh", "bcnorm.cuh"]}[kernel]
    return [os.path.join(csrc, f) for f in files if os.path.exists(os.path.join(csrc, f))]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, valid only while the
    kernel's source is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}:{workload}")
    if not d or d.get("source_hash") != file_hash(kernel_sources(kernel)):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="m3_clocks_", suffix=".csv")
        self.fh = os.fdopen(fd, "w")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
            self.fh.close()
            os.unlink(self.path)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            text = f.read()
        os.unlink(self.path)
        return self.summarise(text)

    @staticmethod
    def summarise(text):
        """Median SM clock under load, max clock, throttle reasons seen and
        peak power from the sampled CSV rows (None if there are none)."""
        rows = [l.split(",") for l in text.strip().splitlines() if l.strip()]
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 10]
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        pw = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        load = [s for s, p in zip(sm, pw) if p >= 0.5 * max(pw)] if pw else sm
        return {"sm_mhz": statistics.median(load or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None}


def prefill_bytes(s, with_final=True, with_init=False, a_per_token=False, theta_per_head=False, proj=False):
    """Algorithmic HBM bytes of one prefill call: each input read once, y
    written once, the final state written once (init read once if given);
    a data-dependent A adds one fp32 per token-head, angle rates fixed per head
    are read once per head instead of once per token-head; with the MIMO
    projections x, B, C and y hold one row per token-head and the fp32
    weights are read once."""
    io = 2 if s.io == "bf16" else 4
    th = s.batch * s.seqlen * s.nheads
    theta_tok = 0 if theta_per_head else s.dstate // 2
    rio = 1 if proj else s.rank
    per_tok = io * (2 * rio * s.headdim + 2 * rio * s.dstate + 2 + theta_tok) + 4 * int(a_per_token)
    th_w = 4 * s.nheads * s.rank * 2 * (s.headdim + s.dstate) if proj else 0
    state = 4 * s.batch * s.nheads * (s.dstate * s.headdim + s.rank * (s.dstate + s.headdim))
    a_bytes = 0 if a_per_token else 4 * s.nheads
    theta_bytes = io * s.nheads * (s.dstate // 2) if theta_per_head else 0
    return th * per_tok + state * (int(with_final) + int(with_init)) + 4 * s.nheads + a_bytes + theta_bytes + th_w


def step_bytes(s):
    """Algorithmic HBM bytes of one decode step (state read + written once,
    pending inputs read + written once, the token's io inputs, y)."""
    io = 2 if s.io == "bf16" else 4
    bh = s.batch * s.nheads
    state = 4 * (s.dstate * s.headdim + s.rank * (s.dstate + s.headdim))
    inp = io * (s.rank * s.headdim + 2 * s.rank * s.dstate + 2 + s.dstate // 2)
    return bh * (2 * state + inp + io * s.rank * s.headdim) + 8 * s.nheads


# ---------------------------------------------------------------- ranks (replicas, no data-path collective)
def dist_helpers(world, device=None):
    """barrier() and max_over_ranks(v) over the default process group of
    `world` ranks (both plain no-ops for one rank).  Timing is taken as the
    maximum over ranks of each rank's device-timed interval."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def replica_shape(name, rank):
    """Weak scaling: every rank runs the whole workload on its own seeded batch."""
    from m3_inputs import WORKLOADS
    return WORKLOADS[name].with_(seed=WORKLOADS[name].seed + rank)


def workload_config(name, s, world):
    """The `config` of the JSON line: the workload by name and sizes, the same
    dict in both arms."""
    ab = prefill_bytes(s)
    return {"workload": name, "batch": s.batch, "seq_len": s.seqlen, "nheads": s.nheads, "headdim": s.headdim,
            "dstate": s.dstate, "rank": s.rank, "io": s.io, "global_batch": world * s.batch,
            "parallelism": f"replicas x{world} (no collective)",
            "l2": (f"inputs larger than L2 ({ab / 1e6:.0f} MB per step), no flush" if ab > (200 << 20) else
                   f"inputs ({ab / 1e6:.1f} MB) smaller than L2")}


def job_tokens_per_s(world, steps, shape, elapsed_s):
    """Whole-job throughput: tokens of all ranks over the max-over-ranks time."""
    return world * steps * shape.batch * shape.seqlen / elapsed_s


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    import torch

    import oracle
    from m3_inputs import WORKLOADS, make_prefill

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = WORKLOADS[args.workload]
    cores = oracle.num_cores()
    nslices = max(1, cores)
    sub = s.with_(batch=1, nheads=nslices)  # bounded sample: `cores` full-length slices
    inp = {k: v.double().numpy() for k, v in make_prefill(sub).items()}
    keys = ("x", "B", "C", "dt", "lam", "theta", "A", "D")
    for _ in range(args.warmup):
        oracle.scan(*(inp[k] for k in keys))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.scan(*(inp[k] for k in keys))
    el = time.perf_counter() - t0
    # tokens of the workload's model (all heads) per second
    value = args.steps * nslices * s.seqlen / s.nheads / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload, s, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{nslices} (batch, head) slices x {s.seqlen} tokens per step, "
                                       f"scaled to tokens of all {s.nheads} heads"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def time_prefill(m3, name, args, dev, rank, world, barrier, max_over_ranks, hbm_peak, peak_src, keys, stream,
                 algo, steps, flush_l2=False):
    """Time `steps` prefill calls of workload `name` (inputs resident in HBM)
    with CUDA events on the launching stream: the whole timed region (max
    over ranks) and each call alone (mean, for the roofline).  With flush_l2
    (inputs smaller than L2, a call far shorter than the host's own time per
    call) the calls are timed on the device alone: `steps` pairs of (256 MiB
    write to flush L2, call) replayed from one CUDA graph, minus a graph of
    the writes alone.  Returns the entry, the state after the last call and
    the workload's (A, D)."""
    import torch
    from m3_inputs import make_prefill

    s = replica_shape(name, rank)
    inp = make_prefill(s, device=dev)
    dims = m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)
    info = m3.scan_plan_info(dims, algo)
    kernel = info.kernel_name
    y = torch.empty_like(inp["x"])
    fin = m3.empty_state(s.batch, s.nheads, s.dstate, s.headdim, s.rank, device=dev)
    ws = torch.empty(max(info.workspace_bytes, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None

    def call(st=stream):
        m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, workspace=ws, algo=algo, stream=st)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    if flush_l2:
        graphs = {}
        for kind in ("pairs", "flushes"):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(steps):
                    flush.fill_(i & 0xff)
                    if kind == "pairs":
                        call(torch.cuda.current_stream())
            graphs[kind] = g
        t = {}
        for kind, g in graphs.items():
            g.replay()
            torch.cuda.synchronize()
            barrier()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(3):
                g.replay()
            g1.record(stream)
            torch.cuda.synchronize()
            barrier()
            t[kind] = max_over_ranks(g0.elapsed_time(g1) / 1e3 / 3)
        device_call = (t["pairs"] - t["flushes"]) / steps
        del graphs
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xff)
        ev[2 * i].record(stream)
        call()
        ev[2 * i + 1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    m3.stream_status(stream)
    elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    launch = statistics.mean(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)) / 1e3
    host_call = launch
    if flush_l2:
        launch = device_call
    abytes = prefill_bytes(s)
    achieved = abytes / launch / 1e9
    per_call = launch if flush_l2 else elapsed / steps
    entry = {"workload": name, "kind": "prefill", "value": world * s.batch * s.seqlen / per_call,
             "unit": "tokens/s", "steps": steps, "ms_per_step": 1e3 * per_call,
             "gpu_launches": steps * info.launches, "dtype": "bf16" if s.io == "bf16" else "f32",
             "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                          "frac": achieved / hbm_peak, "traffic": recorded_traffic(kernel, name),
                          "kernel": kernel, "algorithmic_bytes_per_launch": abytes, "launch_ms": launch * 1e3,
                          "peak_source": peak_src},
             "schedule": {"ctas": info.ctas, "segments_per_sequence": info.segments,
                          "kernel_launches_per_call": info.launches}}
    if info.launches > 1:
        entry["roofline"]["note"] = ("sequences split into segments: summary pass, then the main pass launched as "
                                     "its programmatic dependent, with a look-back over the published summaries; "
                                     "launch_ms and achieved cover the whole call")
    if flush_l2:
        entry["l2"] = f"inputs ({abytes / 1e6:.1f} MB) smaller than L2: 256 MiB written before every call"
        entry["timing"] = ("device time per call: a CUDA graph of (flush, call) pairs minus a graph of the "
                           "flushes alone; eagerly, with the host's work per call in the interval, "
                           f"{host_call * 1e3:.3f} ms per call")
    else:
        entry["l2"] = f"inputs larger than L2 ({abytes / 1e6:.0f} MB per step), no flush"
    AD = (inp["A"], inp["D"])
    del inp, y, ws, flush
    return entry, fin, AD


def run_ours(args):
    import torch
    import torch.distributed as dist

    import state_space_sequence_ssm_b200 as m3
    from m3_inputs import WORKLOADS, make_prefill

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    barrier, max_over_ranks = dist_helpers(world, dev)

    hbm_peak, peak_src = peaks()
    keys = ("x", "B", "C", "dt", "lam", "theta", "A", "D")
    algo = {"auto": m3.ALGO_AUTO, "simt": m3.ALGO_SIMT, "tc": m3.ALGO_TC}[args.algo]
    s = replica_shape(args.workload, rank)
    inp = make_prefill(s, device=dev)
    dims = m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)
    info = m3.scan_plan_info(dims, algo)
    kernel = info.kernel_name
    use_tc = info.kernel == m3.KERNEL_TC
    y = torch.empty_like(inp["x"])
    fin = m3.empty_state(s.batch, s.nheads, s.dstate, s.headdim, s.rank, device=dev)
    ws = torch.empty(max(info.workspace_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def prefill():
        m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, workspace=ws, algo=algo, stream=stream)

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    clocks = ClockSampler(uuid)
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        ev[2 * i].record(stream)
        prefill()
        ev[2 * i + 1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    m3.stream_status(stream)
    elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    launch = statistics.mean(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)) / 1e3
    value = job_tokens_per_s(world, K, s, elapsed)
    abytes = prefill_bytes(s)
    achieved = abytes / launch / 1e9
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if use_tc else "f32",
            "data": "synthetic",
            "config": workload_config(args.workload, s, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": recorded_traffic(kernel, args.workload),
                         "kernel": kernel, "algorithmic_bytes_per_launch": abytes,
                         "launch_ms": launch * 1e3, "peak_source": peak_src,
                         "segments_per_sequence": info.segments, "kernel_launches_per_call": info.launches,
                         "ctas": info.ctas},
            "gpu_launches": K * info.launches, "clocks": clk}
    if info.launches > 1:
        line["roofline"]["note"] = ("sequences split into segments: summary pass, then the main pass launched as "
                                    "its programmatic dependent, with a look-back over the published summaries; "
                                    "launch_ms and achieved cover the whole call")

    # ---- end to end through the public API: m3_scan_fwd_host on pinned host buffers (copies in,
    #      scan, copies of y and the final state out, pipelined over time slices by the library)
    if not args.no_e2e:
        host = {k: v.to("cpu").pin_memory() for k, v in inp.items()}
        yh = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
        fh = m3.State(*(torch.empty(t.shape, dtype=torch.float32, pin_memory=True) for t in fin))
        hplan = m3.scan_host_plan(m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io))
        hws = torch.empty(hplan.workspace_bytes, dtype=torch.uint8, device=dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = yh.numel() * yh.element_size() + sum(t.numel() * 4 for t in fh)

        def e2e_step():
            m3.scan_fwd_host(*(host[k] for k in keys), None, y=yh, final=fh, workspace=hws, stream=stream)

        for _ in range(min(2, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        el2 = max_over_ranks(e0.elapsed_time(e1) / 1e3)
        # the copies alone: one plain pinned copy per direction (at most 1 GiB), same stream
        ref = {}
        for name, nbytes in (("h2d", h2d), ("d2h", d2h)):
            n = min(nbytes, 1 << 30)
            hbuf = torch.empty(n, dtype=torch.uint8, pin_memory=True)
            dbuf = torch.empty(n, dtype=torch.uint8, device=dev)
            src, dst = (hbuf, dbuf) if name == "h2d" else (dbuf, hbuf)
            for _ in range(2):
                dst.copy_(src, non_blocking=True)
            torch.cuda.synchronize()
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(3):
                dst.copy_(src, non_blocking=True)
            c1.record(stream)
            torch.cuda.synchronize()
            ref[name] = 3 * n / (c0.elapsed_time(c1) / 1e3) / 1e9
            del hbuf, dbuf
        bound = max(h2d / ref["h2d"], d2h / ref["d2h"]) / 1e9  # seconds per step if the copies alone set the pace
        # both directions at once (two streams), the step's bytes scaled to at most 1 GiB in total
        f = min(1.0, (1 << 30) / (h2d + d2h))
        nin, nout = max(16, int(h2d * f)), max(16, int(d2h * f))
        hin = torch.empty(nin, dtype=torch.uint8, pin_memory=True)
        din = torch.empty(nin, dtype=torch.uint8, device=dev)
        hout = torch.empty(nout, dtype=torch.uint8, pin_memory=True)
        dout = torch.empty(nout, dtype=torch.uint8, device=dev)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for rep in range(2):
            torch.cuda.synchronize()
            c0.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            with torch.cuda.stream(s_in):
                din.copy_(hin, non_blocking=True)
            with torch.cuda.stream(s_out):
                hout.copy_(dout, non_blocking=True)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            c1.record(stream)
            torch.cuda.synchronize()
        duplex = c0.elapsed_time(c1) / 1e3 / f
        del hin, din, hout, dout
        line["e2e"] = {"value": job_tokens_per_s(world, K, s, el2), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "api": "m3_scan_fwd_host", "ms_per_step": el2 / K * 1e3,
                       "copy_reference": {"h2d_gbs": ref["h2d"], "d2h_gbs": ref["d2h"], "bound_ms": bound * 1e3,
                                          "frac": bound / (el2 / K), "duplex_ms": duplex * 1e3,
                                          "frac_of_duplex": duplex / (el2 / K)},
                       "pipeline": {"units": hplan.units, "slice_tokens": hplan.slice_tokens,
                                    "group_batch": hplan.group_batch}}
        del host, yh, fh, hws

    if not args.no_variants and use_tc:
        line["variants"] = [run_variant(m3, kind, args, dev, rank, world, barrier, max_over_ranks, hbm_peak,
                                        peak_src, keys, stream) for kind in VARIANTS]
    del inp, y, fin, ws
    torch.cuda.empty_cache()

    # ---- every workload the method is measured on, each timed on its own:
    #      the small fp32 scan, the SISO prefill (the line above), the MIMO
    #      prefill, the batch-256 decode steps and the long-context prefill
    #      followed by 256 decode steps of its own sequences
    if not args.no_configs and args.workload == PREFILL_WORKLOAD:
        configs = []
        for idx, name in enumerate(CONFIG_WORKLOADS):
            if name == PREFILL_WORKLOAD:
                configs.append({"config": idx, "workload": name, "kind": "prefill", "value": value,
                                "unit": "tokens/s", "ms_per_step": line["ms_per_step"], "steps": K,
                                "gpu_launches": line["gpu_launches"], "roofline": line["roofline"],
                                "note": "the headline line itself"})
            elif name.startswith("decode"):
                if not args.no_decode:
                    for dname in DECODE_WORKLOADS:
                        e = run_decode(m3, dname, args, dev, rank, world, barrier, max_over_ranks, hbm_peak,
                                       peak_src, keys)
                        configs.append({"config": idx, **e})
            else:
                small = WORKLOADS[name].seqlen * WORKLOADS[name].batch * WORKLOADS[name].nheads < (1 << 20)
                e, st, AD = time_prefill(m3, name, args, dev, rank, world, barrier, max_over_ranks, hbm_peak,
                                         peak_src, keys, stream, m3.ALGO_AUTO, K, flush_l2=small)
                configs.append({"config": idx, **e})
                if name.startswith("long") and not args.no_decode:
                    e = run_decode(m3, name, args, dev, rank, world, barrier, max_over_ranks, hbm_peak, peak_src,
                                   keys, state=st, AD=AD)
                    configs.append({"config": idx, **e})
                del st, AD
                torch.cuda.empty_cache()
        line["configs"] = configs
    elif not args.no_decode:
        # another --workload: the long-context one continues its own sequences
        # (its prefill's state, then 256 steps); every other reports the batch-256 decode workloads
        names = [args.workload] if args.workload.startswith("long") else DECODE_WORKLOADS
        line["decode"] = [run_decode(m3, name, args, dev, rank, world, barrier, max_over_ranks, hbm_peak,
                                     peak_src, keys) for name in names]

    # ---- CPU baseline: the oracle as it stands on this machine's host cores (rank 0, N = 1)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(s, keys)

    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


VARIANTS = {"a_per_token": "data-dependent A_t (M3_FLAG_A_PER_TOKEN)",
            "theta_per_head": "angle rates fixed per head (M3_FLAG_THETA_PER_HEAD)",
            "bcnorm": "fused BC-norm prologue (m3_scan_fwd_bcnorm)",
            "mimo_proj": "fused MIMO projections (m3_scan_fwd_proj) on the MIMO workload's shape"}
MIMO_WORKLOAD = "mimo_bf16_b8_t4096_h32_p64_n64_r4"


def run_variant(m3, kind, args, dev, rank, world, barrier, max_over_ranks, hbm_peak, peak_src, keys, stream):
    """The prefill workload with a data-dependent A_t ([Bt, T, H] fp32) or
    with theta fixed per head ([H, N/2]), timed like the headline (CUDA events
    on the launching stream, K launches)."""
    import torch
    from m3_inputs import make_bcnorm, make_prefill, make_prefill_proj, make_proj

    workload = MIMO_WORKLOAD if kind == "mimo_proj" else args.workload
    s = replica_shape(workload, rank)
    bcn = proj = None
    if kind == "mimo_proj":
        inp = make_prefill_proj(s, device=dev)
        w = make_proj(s, device=dev)
        proj = m3.MimoProj(w["wx"], w["wB"], w["wC"], w["wy"])
    else:
        inp = make_prefill(s, device=dev, **({} if kind == "bcnorm" else {kind: True}))
    if kind == "bcnorm":
        p = make_bcnorm(s, device=dev)
        bcn = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
    y = torch.empty_like(inp["x"])
    fin = m3.empty_state(s.batch, s.nheads, s.dstate, s.headdim, s.rank, device=dev)
    for _ in range(args.warmup):
        m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, stream=stream, bcnorm=bcn, proj=proj)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        m3.scan_fwd(*(inp[k] for k in keys), None, y=y, final=fin, stream=stream, bcnorm=bcn, proj=proj)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    m3.stream_status(stream)
    el = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    ab = prefill_bytes(s, **({} if kind == "bcnorm" else {"proj" if kind == "mimo_proj" else kind: True}))
    if kind == "bcnorm":  # the norm weights and the biases, read once
        ab += 4 * (2 * s.dstate + 2 * s.nheads * s.rank * s.dstate)
    ach = ab / (el / K) / 1e9
    del inp, y, fin
    torch.cuda.empty_cache()
    return {"variant": VARIANTS[kind], "workload": workload,
            "value": world * K * s.batch * s.seqlen / el, "unit": "tokens/s", "steps": K,
            "ms_per_step": 1e3 * el / K, "gpu_launches": K,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                         "traffic": recorded_traffic("prefill_tc_kernel", f"{workload}+{kind}"),
                         "kernel": "prefill_tc_kernel", "algorithmic_bytes_per_launch": ab,
                         "peak_source": peak_src}}


def run_decode(m3, name, args, dev, rank, world, barrier, max_over_ranks, hbm_peak, peak_src, keys, state=None,
               AD=None):
    """Decode steps of workload `name`, all captured in one CUDA graph: from
    the state of its own prefill (`state` with the prefill's (A, D) `AD`, or a
    prefill run here), 256 steps for the long-context workload,
    --decode-steps for the others."""
    import torch
    from m3_inputs import LONG_DECODE_STEPS, make_prefill, make_steps

    s = replica_shape(name, rank)
    if state is None:
        pre = make_prefill(s, device=dev)
        _, st = m3.scan_fwd(*(pre[k] for k in keys), None)
        A, D = pre["A"], pre["D"]
        del pre
    else:
        st = state
        A, D = AD
    torch.cuda.empty_cache()
    S = LONG_DECODE_STEPS if name.startswith("long") else args.decode_steps
    steps = make_steps(s, S, device=dev)
    y = torch.empty(s.batch, s.nheads, s.rank, s.headdim, dtype=s.torch_io, device=dev)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    sk = ("x", "B", "C", "dt", "lam", "theta")
    # warm-up launches (they advance the state, as real decode would)
    with torch.cuda.stream(stream):
        for i in range(3):
            m3.step(*(steps[k][i] for k in sk), A, D, st, y=y, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(S):
            m3.step(*(steps[k][i] for k in sk), A, D, st, y=y, stream=stream)
    g.replay()  # warm replay
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    m3.stream_status(stream)
    el = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    per = el / S
    ab = step_bytes(s)
    kernel = decode_kernel_name(s)
    ach = ab / per / 1e9
    del g, steps
    torch.cuda.empty_cache()
    return {"workload": name, "kind": "decode", "value": world * s.batch / per, "unit": "tokens/s", "steps": S,
            "us_per_step": per * 1e6, "gpu_launches": S,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                         "frac": ach / hbm_peak, "traffic": recorded_traffic(kernel, name),
                         "kernel": kernel, "algorithmic_bytes_per_launch": ab,
                         "note": "per-step time includes graph launch gaps", "peak_source": peak_src}}


def decode_kernel_name(s):
    """The decode kernel the library runs for this shape: rank 1 (and P = 128
    or N = 256) one CTA per slice, rank >= 2 with P = 64, N in {64, 128} the
    persistent streaming kernel."""
    return "step_stream_kernel" if (s.rank >= 2 and s.headdim == 64 and s.dstate in (64, 128)) else "step_kernel"


def cpu_baseline(s, keys):
    import oracle
    from m3_inputs import make_prefill

    cores = oracle.num_cores()
    nslices = max(1, cores)
    sub = s.with_(batch=1, nheads=nslices, seed=s.seed)
    inp = {k: v.double().numpy() for k, v in make_prefill(sub).items()}
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.scan(*(inp[k] for k in keys))
        reps += 1
        if time.perf_counter() - t0 > 10.0:
            break
    el = time.perf_counter() - t0
    value = reps * nslices * s.seqlen / s.nheads / el
    return {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} x {nslices} (batch, head) slices x {s.seqlen} tokens of the same workload, "
                      f"{el:.1f} s, scaled to tokens of all {s.nheads} heads"}


def main():
    args = parse()
    if args.case:
        run_case(args)
    elif args.compare_fp32:
        run_compare_fp32(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
