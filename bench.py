#!/usr/bin/env python
"""Benchmark of the VanillaMarkov head's hot path on B200.

One step = one pass over the whole path on its seeded synthetic workloads:
  * teacher-forced apply_block_logits, 320 rows (B=4, 16 blocks of 5),
    V=129280, rank 128, bf16 (the workload the metric is quoted on);
  * greedy sample_block_tokens, B=32 blocks of M=5, V=129280, rank 128;
  * temperature sample_block_tokens, B=32, M=8, V=151936, rank 64, T=0.7.
The metric is corrected-logit rows per second over the step (apply rows plus
sampled positions), with per-part rows/s, blocks/s, GB/s and roofline
fractions beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one rank per GPU; every rank runs its
own copy of the workload (weak scaling, no data-path collective) and the
step time is the max over ranks. ``--impl reference`` times the CPU fp64
oracle on the host cores instead (rank 0 only).
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
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rank_markov_draft_vanillamarkov_b200 import workloads as W  # noqa: E402

METRIC = "corrected-logit rows/s + achieved HBM GB/s (% roofline); sampled blocks/s at M=5"
UNIT = "rows/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
PARTS = (("apply", W.APPLY_320), ("greedy", W.greedy(32)), ("temperature", W.TEMPERATURE))
EXTRA = (("apply_2560", W.APPLY_2560), ("apply_fp32", W.APPLY_320_FP32), ("transition", W.TRANSITION_320),
         ("backward", W.BACKWARD_320), ("fused_lm_head", W.FUSED_320), ("greedy_b1", W.greedy(1)),
         ("greedy_b8", W.greedy(8)), ("greedy_b64", W.greedy(64)))
L2_BYTES = 126 * 1024 * 1024


def part_rows(wl: W.Workload) -> int:
    return wl.rows if wl.mode in ("apply", "transition", "backward", "fused") else wl.batch * wl.proposal_len


# --------------------------------------------------------------- helpers --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Sustained dense bf16 TFLOP/s (a kernel timed inside a long loop)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def profile_field(kernel_tag: str, field: str):
    """A per-launch figure from the committed ncu summary of this kernel
    (profiles/<tag>.md), valid only while every source file it lists still
    has the recorded hash."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(field + r":\s*([0-9.eE+]+)", text)
    pairs = re.findall(r"source_file:\s*(\S+)\s+source_sha256:\s*([0-9a-f]{64})", text)
    if not (m_b and pairs):
        return None
    for rel, digest in pairs:  # the kernel file and the headers it includes
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != digest:
            return None
    return float(m_b.group(1))


def profile_traffic(kernel_tag: str):
    """DRAM read + write bytes per launch (roofline.traffic)."""
    return profile_field(kernel_tag, "traffic_bytes_per_launch")


ISSUE_SLOTS_PER_SM = 4  # one warp instruction per clock per SM sub-partition


def issue_roofline(kernel_tag: str, seconds: float, sm_mhz: float, sms: int):
    """The issue bound of a kernel limited by its instruction stream: warp
    instructions per launch (ncu smsp__inst_executed.sum) over the launch
    time, against SMs x 4 issue slots x the SM clock sampled during the run."""
    inst = profile_field(kernel_tag, "inst_executed_per_launch")
    if inst is None or not sm_mhz:
        return None
    peak = sms * ISSUE_SLOTS_PER_SM * sm_mhz * 1e6
    return {"achieved": inst / seconds, "peak": peak, "unit": "warp-inst/s", "frac": inst / seconds / peak,
            "inst_per_launch": inst, "sm_mhz": sm_mhz}


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.6)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- our arm ----

class Part:
    """Device-resident inputs (several rotating sets, together larger than
    L2) and outputs of one workload of the step."""

    def __init__(self, name, wl, device, seed_offset, min_bytes=3 * L2_BYTES):
        from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov
        self.name, self.wl, self.device = name, wl, device
        per = wl.bytes_moved()
        self.nsets = max(2, -(-min_bytes // per))
        self.sets = []
        for i in range(self.nsets):
            d = W.make_inputs(wl.with_(data_seed=wl.data_seed + seed_offset + i))
            dev = {k: v.to(device) for k, v in d.items() if isinstance(v, torch.Tensor)}
            dev["head"] = VanillaMarkov(dev["w1"], dev["w2"])
            if wl.mode == "apply":
                dev["out"] = torch.empty_like(dev["base"])
            elif wl.mode == "backward":
                dev["gw1"] = torch.empty(wl.vocab, wl.rank, dtype=torch.float32, device=device)
                dev["gw2"] = torch.empty(wl.vocab, wl.rank, dtype=torch.float32, device=device)
            elif wl.mode == "fused":
                dev["out"] = torch.empty(*dev["prev_ids"].shape, wl.vocab, dtype=torch.float32, device=device)
            elif wl.mode == "transition":
                ids = dev["prev_ids"]
                dev["out"] = torch.empty(*ids.shape, wl.vocab, dtype=torch.bfloat16, device=device)
                dev["emb"] = torch.empty(*ids.shape, wl.rank, dtype=torch.bfloat16, device=device)
            else:
                dev["tokens"] = torch.empty(wl.batch, wl.proposal_len, dtype=torch.long, device=device)
                dev["out"] = torch.empty_like(dev["base"])
            self.sets.append(dev)
        self.host = W.make_inputs(wl.with_(data_seed=wl.data_seed + seed_offset))

    def run(self, i):
        s = self.sets[i % self.nsets]
        if self.wl.mode == "apply":
            s["head"].apply_block_logits(s["base"], token_ids=s["prev_ids"], out=s["out"])
        elif self.wl.mode == "transition":
            s["head"].transition_logits(s["prev_ids"], out=s["out"], out_embeddings=s["emb"])
        elif self.wl.mode == "fused":
            s["head"].fused_lm_head_logits(s["hidden"], s["lm_head"], token_ids=s["prev_ids"], out=s["out"])
        elif self.wl.mode == "backward":
            s["head"].apply_block_logits_backward(s["base"], token_ids=s["prev_ids"], grad_w1=s["gw1"],
                                                  grad_w2=s["gw2"])
        else:
            s["head"].sample_block_tokens(s["base"], first_prev_token_ids=s["first_prev"],
                                          temperature=self.wl.temperature, seed=self.wl.philox_seed,
                                          out_tokens=s["tokens"], out_logits=s["out"])

    @property
    def rows(self):
        return part_rows(self.wl)


TIMED_LAUNCHES = {"last": 0}  # this library's kernel launches inside the last timed loop


def time_region(parts, steps, warmup, world):
    """Warm up, then time exactly `steps` steps between a barrier and a device
    synchronise on both sides. Returns (region seconds max over ranks, per-part
    mean kernel seconds); the launches of the timed loop alone go to
    TIMED_LAUNCHES."""
    import torch.distributed as dist
    from rank_markov_draft_vanillamarkov_b200 import launch_count
    for i in range(warmup):
        for p in parts:
            p.run(i)
    torch.cuda.synchronize()
    ev = {p.name: [] for p in parts}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    n0 = launch_count()
    start.record()
    for i in range(steps):
        for p in parts:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            p.run(warmup + i)
            b.record()
            ev[p.name].append((a, b))
    end.record()
    TIMED_LAUNCHES["last"] = launch_count() - n0
    torch.cuda.synchronize()
    region = start.elapsed_time(end) / 1e3
    per = {k: sum(a.elapsed_time(b) for a, b in v) / len(v) / 1e3 for k, v in ev.items()}
    if world > 1:
        t = torch.tensor([region], device=parts[0].device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        region = float(t.item())
        dist.barrier()
    return region, per


def time_e2e(parts, steps, world):
    """The same step through the public API with host buffers: each step
    copies its inputs host->device from pinned memory, runs the three calls
    and copies every output (corrected logits and tokens) back to pinned host
    memory; all inside the timed region. Copies in the two directions and the
    calls run on three streams with two sets of device buffers, so the link's
    two directions and the kernels overlap across consecutive parts and steps
    (the link is full duplex); every step still moves all its bytes."""
    import torch.distributed as dist
    from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov
    dev = parts[0].device
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    jobs, h2d, d2h = [], 0, 0
    for p in parts:
        h = {k: v.pin_memory() for k, v in p.host.items() if isinstance(v, torch.Tensor) and k not in ("w1", "w2")}
        keys = ["base", "prev_ids"] if p.wl.mode == "apply" else ["base", "first_prev"]
        head = VanillaMarkov(p.sets[0]["w1"], p.sets[0]["w2"])
        bufs = []
        for _ in range(2):  # device inputs and outputs, one set per step parity
            d = {k: torch.empty_like(h[k], device=dev) for k in keys}
            d["out"] = torch.empty_like(d["base"])
            if p.wl.mode == "sample":
                d["tok"] = torch.empty(p.wl.batch, p.wl.proposal_len, dtype=torch.long, device=dev)
            d["copied"], d["done"], d["read"] = (torch.cuda.Event() for _ in range(3))
            d["read"].record(s_out)
            bufs.append(d)
        out_host = torch.empty_like(h["base"]).pin_memory()
        tok_host = torch.empty(p.wl.batch, p.wl.proposal_len, dtype=torch.long).pin_memory() \
            if p.wl.mode == "sample" else None
        h2d += sum(h[k].numel() * h[k].element_size() for k in keys)
        d2h += out_host.numel() * out_host.element_size() + (tok_host.numel() * 8 if tok_host is not None else 0)
        jobs.append((p, head, h, keys, bufs, out_host, tok_host))

    def one(i):
        for p, head, h, keys, bufs, out_host, tok_host in jobs:
            d = bufs[i & 1]
            with torch.cuda.stream(s_in):
                s_in.wait_event(d["read"])  # this set's previous outputs have been read back
                for k in keys:
                    d[k].copy_(h[k], non_blocking=True)
                d["copied"].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(d["copied"])
                if p.wl.mode == "apply":
                    head.apply_block_logits(d["base"], token_ids=d["prev_ids"], out=d["out"])
                else:
                    head.sample_block_tokens(d["base"], first_prev_token_ids=d["first_prev"],
                                             temperature=p.wl.temperature, seed=p.wl.philox_seed,
                                             out_tokens=d["tok"], out_logits=d["out"])
                d["done"].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(d["done"])
                out_host.copy_(d["out"], non_blocking=True)
                if tok_host is not None:
                    tok_host.copy_(d["tok"], non_blocking=True)
                d["read"].record(s_out)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    a.record(cur)
    for st in (s_in, s_run, s_out):
        st.wait_stream(cur)  # nothing of the timed region starts before `a`
    for i in range(steps):
        one(i)
    for st in (s_in, s_run, s_out):
        cur.wait_stream(st)
    b.record(cur)
    torch.cuda.synchronize()
    sec = a.elapsed_time(b) / 1e3
    if world > 1:
        t = torch.tensor([sec], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        sec = float(t.item())
    return sec, h2d, d2h


# ------------------------------------------------------- oracle (CPU) arm --

def _np(t):
    return t.to(torch.float64).numpy()


def oracle_threads():
    """Threads of the BLAS library the oracle's matrix products run on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def host_cores():
    """Cores this process may run on (its CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_parallelism():
    return (f"the oracle's matrix products use {oracle_threads()} BLAS threads; its rounding, selection and "
            f"the sampler's step loop run on one thread")


def oracle_full_step(inputs):
    """The oracle over one whole step (every part at full size)."""
    import oracle
    rows = 0
    for (name, wl), d in zip(PARTS, inputs):
        if wl.mode == "apply":
            oracle.apply_block_logits(_np(d["base"]), _np(d["w1"]), _np(d["w2"]), d["prev_ids"].numpy(), "bf16")
        else:
            oracle.sample_block_tokens(_np(d["base"]), _np(d["w1"]), _np(d["w2"]), d["first_prev"].numpy(), "bf16",
                                       wl.temperature, wl.philox_seed)
        rows += part_rows(wl)
    return rows


class OracleUnits:
    """The step's work as a sequence of small units in the step's proportions:
    one apply row, one greedy block or one temperature block per unit."""

    def __init__(self):
        self.inputs = [W.make_inputs(wl) for _, wl in PARTS]
        self.np = [{k: (_np(v) if v.is_floating_point() else v.numpy()) for k, v in d.items()} for d in self.inputs]
        self.units = []
        for pi, (name, wl) in enumerate(PARTS):
            n = wl.rows if wl.mode == "apply" else wl.batch
            self.units += [(pi, j) for j in range(n)]

    def run(self, i):
        import oracle
        pi, j = self.units[i % len(self.units)]
        wl = PARTS[pi][1]
        d = self.np[pi]
        if wl.mode == "apply":
            base = d["base"].reshape(-1, wl.vocab)[j:j + 1]
            ids = d["prev_ids"].reshape(-1)[j:j + 1]
            oracle.apply_block_logits(base[None], d["w1"], d["w2"], ids[None], "bf16")
            return 1
        oracle.sample_block_tokens(d["base"][j:j + 1], d["w1"], d["w2"], d["first_prev"][j:j + 1], "bf16",
                                   wl.temperature, wl.philox_seed)
        return wl.proposal_len


def reference_arm(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    units = OracleUnits()
    for i in range(args.warmup):
        units.run(i)
    rows = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        rows += units.run(args.warmup + i)
    sec = time.perf_counter() - t0
    value = rows / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                         "threads": oracle_parallelism(),
                         "sample": "each step is one unit of the step's work in its proportions (one apply row, "
                                   "one greedy block of 5 or one temperature block of 8), in order"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(n_gpus):
    return {
        "workload": "apply_r320_v129280_k128 + greedy_b32_m5_v129280_k128 + temp0.7_b32_m8_v151936_k64",
        "parts": {name: wl.name for name, wl in PARTS},
        "logits_dtype": "bf16", "weights_dtype": "bf16", "accumulate": "fp32",
        "l2": "inputs rotate over >= 3 x L2 of distinct buffers per part, so no step finds its data in L2",
        "parallelism": f"replicas{n_gpus}" if n_gpus > 1 else "single",
    }


PROFILE_TAGS = {"apply": "apply_tc_r320_v129280_k128", "greedy": "sample_tc_greedy_b32_m5_v129280_k128",
                "temperature": "sample_rows_temp_b32_m8_v151936_k64"}


def roofline_block(dom, tag, achieved, hbm_peak, peak_kind, partinfo):
    """The dominant kernel's roofline, against the bound that binds it: HBM
    (algorithmic bytes over the launch time) or, where the kernel's own
    instruction stream takes longer than its bytes would at peak bandwidth,
    the issue rate ("alu")."""
    hbm = {"bound": "hbm", "kernel": dom.name, "achieved": achieved, "peak": hbm_peak, "peak_kind": peak_kind,
           "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": profile_traffic(tag),
           "algorithmic_bytes": dom.wl.bytes_moved()}
    iss = partinfo[dom.name].get("issue")
    if not iss or iss["frac"] <= hbm["frac"]:
        return hbm
    return {"bound": "alu", "kernel": dom.name, "achieved": iss["achieved"], "peak": iss["peak"],
            "peak_kind": "derived: SMs x 4 issue slots x sampled SM clock", "unit": iss["unit"],
            "frac": iss["frac"], "traffic": profile_traffic(tag), "algorithmic_bytes": dom.wl.bytes_moved(),
            "hbm": {k: hbm[k] for k in ("achieved", "peak", "peak_kind", "unit", "frac")}}


# ----------------------------------------------------------------- main ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=[n for n, _ in PARTS + EXTRA], default=None,
                    help="time a single part (for profiling); implies --no-e2e and --no-cpu-baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return reference_arm(args)

    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    from rank_markov_draft_vanillamarkov_b200 import _native as N
    from rank_markov_draft_vanillamarkov_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        torch.distributed.barrier()
    N.load()

    if args.only:
        wl = dict(PARTS + EXTRA)[args.only]
        p = Part(args.only, wl, device, seed_offset=1000 * rank)
        region, per = time_region([p], args.steps, args.warmup, world)
        if rank == 0:
            print(json.dumps({"only": args.only, "workload": wl.name, "us": per[args.only] * 1e6,
                              "gbps": wl.bytes_moved() / per[args.only] / 1e9, "steps": args.steps}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0

    parts = [Part(name, wl, device, seed_offset=1000 * rank) for name, wl in PARTS]
    extra = [] if args.no_extra else \
        [Part(name, wl, device, seed_offset=1000 * rank, min_bytes=2 * L2_BYTES) for name, wl in EXTRA]

    clocks = ClockSampler(local)
    clocks.start()
    region, per = time_region(parts, args.steps, args.warmup, world)
    launches = TIMED_LAUNCHES["last"]
    clk = clocks.stop()
    extra_per = time_region(extra, max(20, args.steps // 20), 3, world)[1] if extra else {}

    e2e = None
    if not args.no_e2e:
        e2e_sec, h2d, d2h = time_e2e(parts, args.e2e_steps, world)
        e2e = {"value": sum(p.rows for p in parts) * world * args.e2e_steps / e2e_sec, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    rows_step = sum(p.rows for p in parts)
    value = rows_step * world * args.steps / region
    hbm_peak, peak_kind = measured_peaks()
    partinfo = {}
    for p in parts + extra:
        t = per.get(p.name, extra_per.get(p.name))
        gbs = p.wl.bytes_moved() / t / 1e9
        info = {"us": t * 1e6, "rows_per_s": p.rows / t, "gbps": gbs, "frac_hbm": gbs / hbm_peak,
                "bytes": p.wl.bytes_moved(), "flops": p.wl.flops()}
        if p.wl.mode == "sample":
            info["blocks_per_s"] = p.wl.batch / t
        if p.wl.mode == "fused":  # compute-bound: the tensor pipe is its roofline
            tf_peak, tf_kind = measured_tensor_peak()
            info["tflops"] = p.wl.flops() / t / 1e12
            info["frac_tensor"] = info["tflops"] / tf_peak
            info["tensor_peak"] = tf_peak
            info["tensor_peak_kind"] = tf_kind
        partinfo[p.name] = info
    dom = max(parts, key=lambda p: per[p.name])
    tag = PROFILE_TAGS[dom.name]
    achieved = dom.wl.bytes_moved() / per[dom.name] / 1e9
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0
    for p in parts:  # the issue bound beside the HBM one, where a profile gives the instruction count
        iss = issue_roofline(PROFILE_TAGS[p.name], per[p.name], sm_mhz, sms)
        if iss:
            partinfo[p.name]["issue"] = iss
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": region / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_block(world),
        "sampled_blocks_per_s_m5": partinfo["greedy"]["blocks_per_s"] * world,
        "parts": partinfo,
        "roofline": roofline_block(dom, tag, achieved, hbm_peak, peak_kind, partinfo),
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inputs = [W.make_inputs(wl) for _, wl in PARTS]
        # Whole full-size steps until about 10 s of oracle time have passed.
        rows, steps, t0 = 0, 0, time.perf_counter()
        while steps == 0 or time.perf_counter() - t0 < 10.0:
            rows += oracle_full_step(inputs)
            steps += 1
        sec = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": rows / sec, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                                "threads": oracle_parallelism(),
                                "sample": f"{steps} full steps (all three parts at full size) through the fp64 oracle",
                                "seconds": sec}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
