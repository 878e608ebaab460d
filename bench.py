"""Benchmark of the OSDN forward pass (phase 1 scan + phase 2 chunked delta rule) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 1p3b|340m|long|varlen|decode]

One step is one ``osdn_fwd`` call -- the whole hot path: both phases, four kernels -- over one
batch of seeded synthetic inputs resident in HBM.  The default workload is the 1.3B-layer shape
(B=4, T=4096, H=16, d_k=d_v=128, bf16 I/O, APF on, eta=0.05); ``340m`` (B=8, T=2048, H=8, no
APF), ``long`` (B=1, T=65536, H=16, S_0 and d_0 passed in) and ``varlen`` (32 packed sequences
of U[128, 8192] tokens, H=16) are the other forward shapes; ``decode`` times ``osdn_step``.
Each timed step is bracketed by CUDA events on the launching stream, and a 256 MiB write
between steps flushes the 126 MB L2 (outside the events).  Prints one JSON line on rank 0.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch (independent
sequences: weak scaling, no data-path collective); the elapsed device time is the max over
ranks and ``value`` counts the tokens of all ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0 only), on a
bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FLUSH_BYTES = 256 << 20
# forward workloads: bench name -> (inputs.CONFIGS name, shape label, description)
FORWARD = {
    "1p3b": ("1p3b_apf", "1.3B-layer",
             "1.3B-layer OSDN token mixer (B=4, T=4096, H=16, d_k=d_v=128, APF)"),
    "340m": ("340m", "340M-layer",
             "340M-layer OSDN token mixer (B=8, T=2048, H=8, d_k=d_v=128, no APF)"),
    "long": ("long_ctx", "long-context",
             "long-context OSDN token mixer (B=1, T=65536, H=16, d_k=d_v=128, APF, S_0 and d_0 "
             "passed in)"),
    "varlen": ("varlen", "varlen",
               "packed variable-length OSDN token mixer (32 sequences of U[128, 8192] tokens, "
               "H=16, d_k=d_v=128, APF)"),
}
METRIC = "OSDN fwd tokens/s (scan+chunk) at 1.3B-layer shape; % of HBM/TC roofline"
# the kernels one bf16 osdn_fwd call with d_k = d_v = 128 launches, in order
FWD_KERNELS = ["precond_prep_kernel", "precond_chain_kernel", "wy_prep_kernel",
               "chunk_fwd_tc_kernel"]
FWD_SOURCES = ["osdn_lib.cu", "common.cuh", "watchdog.cuh", "tc_ptx.cuh", "tril_inverse.cuh",
               "chunk_walk.cuh", "scan_tc.cuh", "chunk_prep.cuh", "chunk_tc.cuh"]


def metric_name(label):
    return f"OSDN fwd tokens/s (scan+chunk) at {label} shape; % of HBM/TC roofline"


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_sha(names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "delta_rule_recurrent_osdn_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profile_record(name):
    """Key: value lines of a committed ncu summary (profiles/<name>.md), or None when the file
    is missing or was taken on other kernel sources (its recorded source hash differs)."""
    path = os.path.join(ROOT, "profiles", f"{name}.md")
    if not os.path.exists(path):
        return None
    rec = dict(re.findall(r"^(\w+):\s*(\S+)\s*$", open(path).read(), re.M))
    if rec.get("source_sha") != kernel_source_sha(FWD_SOURCES if name.startswith("fwd_")
                                                  else STEP_SOURCES):
        return None
    return rec


def fwd_algorithmic_bytes(inp, es=2):
    """Bytes the forward pass must move (the roofline's algorithmic bytes): q, k, v in and o out in the io
    dtype, beta (and r with APF) in fp32 per token-head; per (sequence, head) the final state
    S_T and d_T out in fp32, and S_0, d_0 in when given.  k~ is an intermediate, not counted."""
    th = inp.B * inp.T * inp.H
    per_th = (2 * inp.Dk + 2 * inp.Dv) * es + 4 + (4 if inp.r is not None else 0)
    per_nh = (inp.Dv * inp.Dk + inp.Dk) * 4 * (2 if inp.S0 is not None else 1)
    return th * per_th + inp.N * inp.H * per_nh


def fwd_flops(inp):
    """Chunk-form MMA FLOPs (the roofline's algorithmic tensor work): 5 * 2 * C * d + 3 * 2 * d_k * d_v per
    token-head."""
    return inp.B * inp.T * inp.H * (5 * 2 * inp.chunk * inp.Dk + 3 * 2 * inp.Dk * inp.Dv)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not getattr(self, "out", ""):
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    """(rank, world, local_rank); initialises NCCL only when launched by torchrun."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if n_gpus != world:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over the process group (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def oracle_sample(inp, m_tokens):
    """The first sequences (packed input: whole sequences; fixed length: the first m_tokens
    tokens of every sequence) of a batch, as the bounded sample the oracle is timed on."""
    from delta_rule_recurrent_osdn_b200 import inputs as W
    if inp.cu_seqlens is not None:
        cu = inp.cu_seqlens
        m = int(np.searchsorted(cu[1:], min(m_tokens, cu[-1]), side="left")) + 1
        sub = W.select(inp, seqs=list(range(min(m, inp.N))))
        return sub, int(sub.cu_seqlens[-1]), f"first {min(m, inp.N)} of {inp.N} packed sequences"
    tp = int(max(1, min(inp.T, m_tokens)))
    sub = W.select(inp)
    sub.q, sub.k, sub.v, sub.beta = inp.q[:, :tp], inp.k[:, :tp], inp.v[:, :tp], inp.beta[:, :tp]
    sub.r = None if inp.r is None else inp.r[:, :tp]
    return sub, inp.B * tp, f"first {tp} of {inp.T} tokens of all {inp.B} sequences"


def oracle_run(sub):
    from oracle import osdn_ref
    t0 = time.perf_counter()
    osdn_ref.fwd(sub.q, sub.k, sub.v, sub.beta, sub.r, sub.eta, sub.d0, sub.S0, sub.scale,
                 sub.cu_seqlens)
    return time.perf_counter() - t0


def oracle_rate(inp, seconds_target):
    """Oracle throughput (tokens/s over all heads) on a bounded sample of the batch sized to
    about `seconds_target` of CPU time; returns (rate, threads, sample description)."""
    from oracle import osdn_ref
    threads = osdn_ref.set_threads(0)
    probe, ptok, _ = oracle_sample(inp, 32)
    dt = oracle_run(probe)
    per_token = dt / max(ptok, 1)
    sub, tokens, desc = oracle_sample(inp, int(seconds_target / max(per_token, 1e-9) /
                                              (inp.B if inp.cu_seqlens is None else 1)))
    dt = oracle_run(sub)
    reps = 1
    if dt < seconds_target / 2:  # the whole batch is quick: repeat it
        reps = max(1, int(seconds_target / max(dt, 1e-6)))
        dt = sum(oracle_run(sub) for _ in range(reps))
    sample = (f"{desc} x {inp.H} heads ({tokens * inp.H} token-heads, fp64), {reps} run(s), "
              f"{dt:.1f} s")
    return tokens * reps / dt, threads, sample


def forward_inputs(args, seed=None):
    from delta_rule_recurrent_osdn_b200 import inputs as W
    name, label, desc = FORWARD[args.workload]
    return W.make_inputs(name, seed=seed), label, desc


def config_dict(inp, desc):
    cfg = {"workload": desc, "B": inp.B, "T": inp.T, "H": inp.H, "d_k": inp.Dk, "d_v": inp.Dv,
           "chunk": inp.chunk, "apf": inp.r is not None, "eta": inp.eta, "io": inp.io,
           "l2": "flushed between timed steps (256 MiB write)"}
    if inp.cu_seqlens is not None:
        cfg.update(num_seqs=inp.N, total_tokens=int(inp.cu_seqlens[-1]))
    if inp.S0 is not None:
        cfg["initial_state"] = "S_0 ~ N(0, 0.1^2), d_0 ~ U(0.5, 1.5)"
    return cfg


def bench_reference(args):
    """The oracle as the reference arm: rank 0 only, a bounded sample of the workload per
    step, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload == "decode":
        return bench_reference_decode(args)
    inp, label, desc = forward_inputs(args)
    rate, threads, sample = oracle_rate(inp, seconds_target=3.0)
    sub, tokens, sdesc = oracle_sample(inp, int(rate * 3.0 / (inp.B if inp.cu_seqlens is None
                                                              else 1)))
    for _ in range(args.warmup):
        oracle_run(sub)
    el = sum(oracle_run(sub) for _ in range(args.steps))
    value = tokens * args.steps / el
    line = {
        "impl": "reference", "metric": metric_name(label), "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(inp, desc),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{sdesc} x {inp.H} heads ({tokens * inp.H} token-heads, "
                                   f"fp64) per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def bench_ours(args):
    import torch
    from delta_rule_recurrent_osdn_b200 import inputs as W
    from delta_rule_recurrent_osdn_b200 import osdn

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp, label, desc = forward_inputs(args, seed=None if rank == 0 else 1000 + rank)
    d = W.to_torch(inp, dev)
    stream = torch.cuda.current_stream(dev)
    o = torch.empty_like(d["v"])
    N, H, Dk, Dv = inp.N, inp.H, inp.Dk, inp.Dv
    ST = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=dev)
    dT = torch.empty((N, H, Dk), dtype=torch.float32, device=dev)
    ws = torch.empty(osdn.osdn_fwd_workspace_bytes(inp.B, inp.T, H, Dk), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    launches_per_step = len(FWD_KERNELS)  # bf16, d_k = d_v = 128: both phases' two kernels

    def step():
        osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], inp.eta, d["d0"], d["S0"],
                      inp.scale, inp.chunk, d["cu_seqlens"], o=o, ST=ST, dT=dT, workspace=ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    if osdn.osdn_get_device_status() != osdn.OSDN_OK:
        raise RuntimeError("device status not OK after the timed region")
    step_ms = [e[0].elapsed_time(e[1]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    tokens = inp.B * inp.T
    value = world * tokens * args.steps / (total_ms / 1e3)

    # ---- end to end through the public API with host buffers (pinned): every step copies its
    #      inputs host -> device and o back inside the events; the L2 flush stays outside them
    names = [k_ for k_ in ("q", "k", "v", "beta", "r", "d0", "S0", "cu_seqlens")
             if d[k_] is not None]
    host = {k_: d[k_].cpu().pin_memory() for k_ in names}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    dev_in = {k_: torch.empty_like(d[k_]) for k_ in host}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host.numel() * o_host.element_size()

    def e2e_step():
        for k_, t in host.items():
            dev_in[k_].copy_(t, non_blocking=True)
        osdn.osdn_fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["beta"], dev_in.get("r"),
                      inp.eta, dev_in.get("d0"), dev_in.get("S0"), inp.scale, inp.chunk,
                      dev_in.get("cu_seqlens"), o=o, ST=ST, dT=dT, workspace=ws)
        o_host.copy_(o, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(3)
        e2e_ev[i][0].record(stream)
        e2e_step()
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
    e2e_value = world * tokens * args.steps / (e2e_ms / 1e3)

    if rank == 0:
        hbm, tc, kind = read_peaks()
        mean_ms = statistics.mean(step_ms)
        byts = fwd_algorithmic_bytes(inp)
        flops = fwd_flops(inp)
        achieved = byts / (mean_ms / 1e3) / 1e9
        t_hbm_us, t_tc_us = byts / (hbm * 1e9) * 1e6, flops / (tc * 1e12) * 1e6
        rec = profile_record(f"fwd_{FORWARD[args.workload][0]}")
        traffic = float(rec["dram_bytes_per_step"]) if rec and "dram_bytes_per_step" in rec \
            else None
        roof = {"bound": "hbm", "scope": "whole forward pass (one osdn_fwd call, 4 kernels)",
                "achieved": achieved, "peak": hbm, "peak_kind": f"{kind} hbm_gbs", "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic,
                "traffic_over_algorithmic": None if traffic is None else traffic / byts,
                "algorithmic_bytes_per_launch": byts,
                "hbm_floor_us": t_hbm_us, "tensor_floor_us": t_tc_us,
                "tensor_flops_per_launch": flops, "tensor_peak": tc,
                "tensor_peak_kind": f"{kind} bf16_tflops"}
        if rec and "kernel_shares" in rec:
            shares = {k_: float(v_) for k_, v_ in
                      (x.split("=") for x in rec["kernel_shares"].split(";"))}
            dom = max(shares, key=shares.get)
            roof["dominant_kernel"] = {"name": dom, "ncu_share": shares[dom],
                                       "ms_est": shares[dom] * mean_ms,
                                       "shares": shares}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, threads, sample = oracle_rate(inp, seconds_target=args.cpu_seconds)
            cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                   "sample": sample}
        line = {
            "metric": metric_name(label), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_dict(inp, desc), "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(), "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


STEP_SOURCES = ["common.cuh", "step.cuh"]
DECODE_METRIC = ("OSDN decode tokens/s (one recurrent step per sequence, 256 sequences x 16 heads, "
                 "d_k=d_v=128); % of HBM roofline")
DECODE = dict(B=256, T=8, H=16, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05, chunk=64, seed=7,
              init_state=True)


def decode_bytes_per_step(N, H, Dk, Dv, es=2):
    """HBM bytes of one decode step: the fp32 state read and written, d read and written,
    q, k, v in and o out in the io dtype, beta and r."""
    return N * H * (2 * Dv * Dk * 4 + 2 * Dk * 4 + (2 * Dk + 2 * Dv) * es + 8)


def bench_decode(args):
    """The decode path: ``osdn_step`` over a batch of sequences, one token each per step, the
    state carried in HBM (updated in place).  Tokens cycle through 8 seeded draws."""
    import torch
    from delta_rule_recurrent_osdn_b200 import inputs as W
    from delta_rule_recurrent_osdn_b200 import osdn

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = dict(DECODE)
    if rank:
        cfg["seed"] = 1000 + rank
    inp = W.make_inputs(cfg)
    d = W.to_torch(inp, dev)
    N, H, Dk, Dv, T = inp.N, inp.H, inp.Dk, inp.Dv, inp.T
    tok = [{k_: d[k_][:, t].contiguous() for k_ in ("q", "k", "v", "beta", "r")} for t in range(T)]
    S = d["S0"].clone()
    dd = d["d0"].clone()
    o = torch.empty_like(tok[0]["v"])
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(i):
        x = tok[i % T]
        osdn.osdn_step(x["q"], x["k"], x["v"], x["beta"], S, dd, x["r"], inp.eta, inp.scale, o=o)

    for i in range(args.warmup):
        flush.fill_(1)
        step(i)
    torch.cuda.synchronize(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            events[i][0].record(stream)
            step(i)
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    if osdn.osdn_get_device_status() != osdn.OSDN_OK:
        raise RuntimeError("device status not OK after the timed region")
    step_ms = [e[0].elapsed_time(e[1]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = world * N * args.steps / (total_ms / 1e3)

    # ---- end to end: the step's token data from pinned host memory, o back, copies timed
    host = [{k_: t.cpu().pin_memory() for k_, t in x.items()} for x in tok]
    dev_in = {k_: torch.empty_like(t) for k_, t in tok[0].items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host[0].values())
    d2h = o_host.numel() * o_host.element_size()

    def e2e_step(i):
        for k_, t in host[i % T].items():
            dev_in[k_].copy_(t, non_blocking=True)
        osdn.osdn_step(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["beta"], S, dd, dev_in["r"],
                       inp.eta, inp.scale, o=o)
        o_host.copy_(o, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(3)  # outside the events
        e2e_ev[i][0].record(stream)
        e2e_step(i)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
    e2e_value = world * N * args.steps / (e2e_ms / 1e3)

    if rank == 0:
        hbm, tc, kind = read_peaks()
        avg = statistics.mean(step_ms)
        byts = decode_bytes_per_step(N, H, Dk, Dv)
        achieved = byts / (avg / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": "step", "achieved": achieved, "peak": hbm,
                "peak_kind": f"{kind} hbm_gbs", "unit": "GB/s", "frac": achieved / hbm,
                "traffic": (lambda r: None if not r or "dram_bytes_per_launch" not in r else
                            float(r["dram_bytes_per_launch"]))(profile_record("step_decode")),
                "algorithmic_bytes_per_launch": byts, "kernel_ms": {"step": avg}}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            from oracle import osdn_ref as R
            t0 = time.perf_counter()
            reps = 0
            while True:
                R.fwd(inp.q[:, :1], inp.k[:, :1], inp.v[:, :1], inp.beta[:, :1], inp.r[:, :1],
                      inp.eta, inp.d0, inp.S0, inp.scale)
                reps += 1
                if time.perf_counter() - t0 > min(args.cpu_seconds, 5.0):
                    break
            dt = (time.perf_counter() - t0) / reps
            cpu = {"value": N / dt, "unit": "tokens/s", "cores": R.set_threads(0),
                   "kind": "oracle",
                   "sample": f"one step of all {N} sequences x {H} heads (fp64), {reps} run(s)"}
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"OSDN decode step, {N} sequences x {H} heads, d_k=d_v={Dk}, "
                                   "bf16 I/O, fp32 state, APF",
                       "N": N, "H": H, "d_k": Dk, "d_v": Dv, "io": "bf16", "apf": True,
                       "eta": inp.eta, "l2": "flushed between timed steps (256 MiB write)"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps, "clocks": clk.summary(),
            "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def bench_reference_decode(args):
    """The oracle as the reference arm of the decode workload: one token of every sequence per
    step (the oracle's token loop over a one-token batch), on the host cores."""
    from delta_rule_recurrent_osdn_b200 import inputs as W
    from oracle import osdn_ref as R
    inp = W.make_inputs(dict(DECODE))
    threads = R.set_threads(0)

    def step(i):
        t = i % inp.T
        R.fwd(inp.q[:, t:t + 1], inp.k[:, t:t + 1], inp.v[:, t:t + 1], inp.beta[:, t:t + 1],
              inp.r[:, t:t + 1], inp.eta, inp.d0, inp.S0, inp.scale)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = inp.N * args.steps / el
    line = {
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"OSDN decode step, {inp.N} sequences x {inp.H} heads, "
                               f"d_k=d_v={inp.Dk}, bf16 I/O, fp32 state, APF"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"one step of all {inp.N} sequences x {inp.H} heads (fp64) "
                                   "per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


BWD_METRIC = "OSDN bwd tokens/s (dq, dk, dv, dbeta, dr, deta, dS0, dd0) at 1.3B-layer shape"


def bench_bwd(args):
    """The backward pass (osdn_bwd) over the 1.3B-layer batch, given dL/do and dL/dS_T, dL/dd_T."""
    import torch
    from delta_rule_recurrent_osdn_b200 import inputs as W
    from delta_rule_recurrent_osdn_b200 import osdn

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_inputs("1p3b_apf", seed=None if rank == 0 else 1000 + rank)
    d = W.to_torch(inp, dev)
    rng = np.random.default_rng(123 + rank)
    dO = torch.from_numpy(rng.standard_normal(inp.v.shape).astype(np.float32)).to(dev, torch.bfloat16)
    N, H, Dk, Dv = inp.N, inp.H, inp.Dk, inp.Dv
    dST = torch.from_numpy((0.3 * rng.standard_normal((N, H, Dv, Dk))).astype(np.float32)).to(dev)
    ddT = torch.from_numpy(rng.standard_normal((N, H, Dk)).astype(np.float32)).to(dev)
    ws = torch.empty(osdn.LIB.osdn_bwd_workspace_bytes(0, inp.B, inp.T, H, Dk, Dv, osdn.OSDN_BF16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        return osdn.osdn_bwd(d["q"], d["k"], d["v"], d["beta"], dO, d["r"], inp.eta, d["d0"],
                             d["S0"], inp.scale, dST, ddT, workspace=ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world, dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    if osdn.osdn_get_device_status() != osdn.OSDN_OK:
        raise RuntimeError("device status not OK after the timed region")
    step_ms = [a.elapsed_time(b) for a, b in events]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    tokens = inp.B * inp.T
    value = world * tokens * args.steps / (total_ms / 1e3)
    if rank == 0:
        hbm, tc, kind = read_peaks()
        th = tokens * H
        # q, k, v, dO in (bf16), beta, r in; dq, dk, dv, dbeta, dr out (fp32); per (sequence,
        # head): dS_T, dd_T in and dS_0, dd_0 out (fp32)
        byts = th * ((2 * Dk + 2 * Dv) * 2 + 8 + (2 * Dk + Dv) * 4 + 8) + N * H * 2 * (Dv * Dk + Dk) * 4
        mean_ms = statistics.mean(step_ms)
        achieved = byts / (mean_ms / 1e3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            from oracle import osdn_ref as R
            threads = R.set_threads(0)
            sub, ntok, desc = oracle_sample(inp, 256)
            dO_np = dO.float().cpu().numpy()[:, :sub.T]
            t0 = time.perf_counter()
            R.bwd(sub.q, sub.k, sub.v, sub.beta, dO_np, sub.r, sub.eta, sub.d0, sub.S0, sub.scale)
            dt = time.perf_counter() - t0
            cpu = {"value": ntok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                   "sample": f"{desc} x {H} heads (fp64 gradient), {dt:.1f} s"}
        line = {
            "metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(config_dict(inp, "backward of the " + FORWARD["1p3b"][2]),
                           gradients="fp32"),
            "roofline": {"bound": "hbm", "scope": "whole backward pass (one osdn_bwd call)",
                         "achieved": achieved, "peak": hbm, "peak_kind": f"{kind} hbm_gbs",
                         "unit": "GB/s", "frac": achieved / hbm, "traffic": None,
                         "algorithmic_bytes_per_launch": byts},
            "cpu_baseline": cpu, "e2e": None, "gpu_launches": 5 * args.steps,
            "clocks": clk.summary(), "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=list(FORWARD) + ["decode", "bwd"], default="1p3b",
                    help="a forward-pass shape (default: the 1.3B layer), decode (osdn_step) or "
                         "bwd (osdn_bwd at the 1.3B-layer shape)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return bench_reference(args)
    if args.workload == "decode":
        return bench_decode(args)
    if args.workload == "bwd":
        return bench_bwd(args)
    return bench_ours(args)


if __name__ == "__main__":
    sys.exit(main())
