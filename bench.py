"""Benchmark of the OSDN forward pass (phase 1 scan + phase 2 chunked delta rule) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is the whole hot path over one batch of the 1.3B-layer workload (B=4, T=4096, H=16,
d_k=d_v=128, bf16 I/O, APF on, eta=0.05), seeded synthetic inputs resident in HBM.  Each
timed step is bracketed by CUDA events on the launching stream, and a 256 MiB write between
steps flushes the 126 MB L2 (outside the events).  Prints one JSON line on rank 0.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch (independent
sequences: weak scaling, no data-path collective); the elapsed device time is the max over
ranks and ``value`` counts the tokens of all ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0 only), on a
bounded prefix of the same batch per step.
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

METRIC = "OSDN fwd tokens/s (scan+chunk) at 1.3B-layer shape; % of HBM/TC roofline"
WORKLOAD = "1p3b_apf"
FLUSH_BYTES = 256 << 20
# Algorithmic HBM bytes per token-head (bf16 I/O, d_k = d_v = 128), by kernel:
#   scan : k in (256) + beta (4) + r (4) + k~ out (256)
#   chunk: q, k, k~, v in (1024) + beta (4) + o out (256)
#   fused forward (both phases in one kernel): q, k, v in (768) + beta, r (8) + o out (256)
ALGO_BYTES = {"scan": 520, "chunk": 1284, "fwd": 1032}


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


KERNEL_SOURCES = {"scan": ["common.cuh", "watchdog.cuh", "tc_ptx.cuh", "tril_inverse.cuh",
                           "chunk_walk.cuh", "scan_tc.cuh"],
                  "chunk": ["common.cuh", "watchdog.cuh", "tc_ptx.cuh", "tril_inverse.cuh",
                            "chunk_walk.cuh", "chunk_prep.cuh", "chunk_tc.cuh"],
                  "step": ["common.cuh", "step.cuh"]}


def profiled_traffic(kernel, workload=WORKLOAD):
    """DRAM bytes per launch from the committed ncu summary of this kernel, if it was taken on
    the current source (its recorded source hash matches); else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9.e+]+)", text)
    if not (m_sha and m_tr) or m_sha.group(1) != kernel_source_sha(KERNEL_SOURCES[kernel]):
        return None
    return float(m_tr.group(1))


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


def oracle_rate(inp, seconds_target, max_tokens=None):
    """Oracle throughput (tokens/s over all heads) on a prefix of the batch sized to about
    `seconds_target` of CPU time; returns (rate, threads, sample description, seconds)."""
    from delta_rule_recurrent_osdn_b200 import inputs as W  # noqa: F401
    from oracle import osdn_ref
    threads = osdn_ref.set_threads(0)

    def run(tp):
        q, k, v = inp.q[:, :tp], inp.k[:, :tp], inp.v[:, :tp]
        beta = inp.beta[:, :tp]
        r = None if inp.r is None else inp.r[:, :tp]
        t0 = time.perf_counter()
        osdn_ref.fwd(q, k, v, beta, r, inp.eta, inp.d0, inp.S0, inp.scale)
        return time.perf_counter() - t0

    probe = min(32, inp.T)
    dt = run(probe)
    tp = int(min(inp.T, max(probe, probe * seconds_target / max(dt, 1e-6))))
    if max_tokens:
        tp = min(tp, max_tokens)
    dt = run(tp)
    reps = 1
    if tp == inp.T and dt < seconds_target / 2:  # whole batch is quick: repeat it
        reps = max(1, int(seconds_target / max(dt, 1e-6)))
        dt = sum(run(tp) for _ in range(reps))
    tokens = inp.B * tp * reps
    sample = (f"first {tp} of {inp.T} tokens of all {inp.B} sequences x {inp.H} heads "
              f"({inp.B * tp * inp.H} token-heads, fp64), {reps} run(s), {dt:.1f} s")
    return tokens / dt, threads, sample, dt, tp


def bench_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from delta_rule_recurrent_osdn_b200 import inputs as W
    inp = W.make_inputs(WORKLOAD)
    rate, threads, sample, dt, tp = oracle_rate(inp, seconds_target=3.0)
    from oracle import osdn_ref

    def step():
        q, k, v = inp.q[:, :tp], inp.k[:, :tp], inp.v[:, :tp]
        r = None if inp.r is None else inp.r[:, :tp]
        osdn_ref.fwd(q, k, v, inp.beta[:, :tp], r, inp.eta, inp.d0, inp.S0, inp.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = inp.B * tp * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(inp),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample + " per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_dict(inp):
    return {"workload": "1.3B-layer OSDN token mixer (B=4, T=4096, H=16, d_k=d_v=128, APF)",
            "B": inp.B, "T": inp.T, "H": inp.H, "d_k": inp.Dk, "d_v": inp.Dv,
            "chunk": inp.chunk, "apf": inp.r is not None, "eta": inp.eta, "io": inp.io,
            "l2": "flushed between timed steps (256 MiB write)"}


def bench_ours(args):
    import torch
    from delta_rule_recurrent_osdn_b200 import inputs as W
    from delta_rule_recurrent_osdn_b200 import osdn

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(WORKLOAD, seed=None if rank == 0 else 1000 + rank)
    d = W.to_torch(inp, dev)
    stream = torch.cuda.current_stream(dev)
    kt = torch.empty_like(d["k"])
    o = torch.empty_like(d["v"])
    N, H, Dk, Dv = inp.N, inp.H, inp.Dk, inp.Dv
    ST = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=dev)
    dT = torch.empty((N, H, Dk), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    launches_per_step = 4  # per phase: a per-chunk pre-kernel and the sequential chain

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        osdn.osdn_precond_scan(d["k"], d["beta"], d["r"], d["eta"], d["d0"], k_tilde=kt, dT=dT)
        if ev:
            ev[1].record(stream)
        osdn.osdn_chunk_fwd(d["q"], d["k"], kt, d["v"], d["beta"], d["scale"], d["S0"],
                            d["chunk"], o=o, ST=ST)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            step(events[i])
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    if osdn.osdn_get_device_status() != osdn.OSDN_OK:
        raise RuntimeError("device status not OK after the timed region")
    scan_ms = [e[0].elapsed_time(e[1]) for e in events]
    chunk_ms = [e[1].elapsed_time(e[2]) for e in events]
    step_ms = [e[0].elapsed_time(e[2]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    tokens = inp.B * inp.T
    value = world * tokens * args.steps / (total_ms / 1e3)

    # ---- end to end through the public API with host buffers (pinned), copies timed
    host = {k_: d[k_].cpu().pin_memory() for k_ in ("q", "k", "v", "beta", "r")}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    dev_in = {k_: torch.empty_like(d[k_]) for k_ in host}
    ws = torch.empty(osdn.osdn_fwd_workspace_bytes(inp.B, inp.T, H, Dk), dtype=torch.uint8,
                     device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host.numel() * o_host.element_size()

    def e2e_step():
        for k_, t in host.items():
            dev_in[k_].copy_(t, non_blocking=True)
        osdn.osdn_fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["beta"], dev_in["r"],
                      inp.eta, None, None, inp.scale, inp.chunk, o=o, ST=ST, dT=dT, workspace=ws)
        o_host.copy_(o, non_blocking=True)

    for _ in range(max(3, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        flush.fill_(3)
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = world * tokens * args.steps / (e2e_ms / 1e3)

    if rank == 0:
        hbm, tc, kind = read_peaks()
        avg = {"scan": statistics.mean(scan_ms), "chunk": statistics.mean(chunk_ms)}
        dom = max(avg, key=avg.get)
        token_heads = tokens * H
        achieved = ALGO_BYTES[dom] * token_heads / (avg[dom] / 1e3) / 1e9
        traffic = profiled_traffic(dom)
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                "peak_kind": f"{kind} hbm_gbs", "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic,
                "algorithmic_bytes_per_launch": ALGO_BYTES[dom] * token_heads,
                "kernel_ms": avg, "whole_step_hbm_frac":
                    ALGO_BYTES["fwd"] * token_heads / (statistics.mean(step_ms) / 1e3) / 1e9 / hbm}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, threads, sample, _, _ = oracle_rate(inp, seconds_target=args.cpu_seconds)
            cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                   "sample": sample}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_dict(inp), "roofline": roof,
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
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        flush.fill_(3)
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = world * N * args.steps / (e2e_ms / 1e3)

    if rank == 0:
        hbm, tc, kind = read_peaks()
        avg = statistics.mean(step_ms)
        byts = decode_bytes_per_step(N, H, Dk, Dv)
        achieved = byts / (avg / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": "step", "achieved": achieved, "peak": hbm,
                "peak_kind": f"{kind} hbm_gbs", "unit": "GB/s", "frac": achieved / hbm,
                "traffic": profiled_traffic("step", "decode"),
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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["forward", "decode"], default="forward",
                    help="forward: the 1.3B-layer forward pass (default); decode: osdn_step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return bench_reference(args)
    if args.workload == "decode":
        return bench_decode(args)
    return bench_ours(args)


if __name__ == "__main__":
    sys.exit(main())
