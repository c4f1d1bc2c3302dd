#!/usr/bin/env python3
"""Throughput of the Lightning Attention-2 hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = la2_fwd + la2_bwd over one batch of the named workload (default:
the length-sweep point T = 131,072, B = 1, H = 32, d = e = 128, block 128),
inputs resident in HBM.  Prints one JSON line.  With a sweep workload the line
also carries `sweep`: tokens/s and TFLOP/s of the same step at every sweep
length and at the TNL-15B layer, timed in the same process, so one run shows
how flat the throughput is in T.
Under torchrun (N > 1) every rank runs its own replica (the path has no
exchange step), the timed region is bracketed by a barrier and device
synchronisation on every rank, and the slowest rank's time is reported.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (the pages ship no runnable reference).
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from causal_linear_attention_la2_b200 import inputs as I  # noqa: E402

METRIC = "fwd+bwd tokens/sec and TFLOP/s (fraction of bf16 TC peak) vs T, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


# ------------------------------------------------------------------ helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# the files that define la2_scan_ws, la2_state_ws and the launch plans
SCAN_SOURCES = ("ptx_sm100.cuh", "scan_ws_sm100.cuh", "la2_api.cu")


def kernel_source_hash() -> str:
    """Hash of the scan kernels' and the launch planner's sources: recorded
    DRAM traffic is used only while they are the ones that were profiled."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_linear_attention_la2_b200", "csrc")
    for name in sorted(SCAN_SOURCES):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def flops_per_token_head(w: I.Workload) -> float:
    """Credited fwd+bwd FLOPs per (token, head): 3 x (2 T_B (d + e) + 4 d e)."""
    return 3.0 * (2.0 * w.block * (w.d + w.e) + 4.0 * w.d * w.e)


def executed_flops_per_token_head(w: I.Workload) -> float:
    """Executed fwd+bwd FLOPs per (token, head) of the measurement plan: the
    forward's 2 T_B (d + e) + 4 d e and the backward's 2 T_B (3d + 3e) + 10 d e
    (which recomputes Q K^T, the states and dO V^T in each of its scans)."""
    fwd = 2.0 * w.block * (w.d + w.e) + 4.0 * w.d * w.e
    bwd = 2.0 * w.block * (3 * w.d + 3 * w.e) + 10.0 * w.d * w.e
    return fwd + bwd


def elem_bytes(w: I.Workload) -> int:
    """Bytes per input element."""
    return 2 if w.dtype == "bf16" else 4


OUT_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def out_bytes(out_dtype: str) -> int:
    """Bytes per output element (--out-dtype)."""
    return 2 if out_dtype == "bf16" else 4


def bwd_algorithmic_bytes(w: I.Workload) -> float:
    """la2_bwd reads q, k, v, dO and writes dq, dk, dv, each once, every tensor
    counted at the input element width (the per-token-head bytes of the
    measurement plan: w (2d + 2e) in, w (2d + e) out)."""
    return float(w.sequences) * w.T * elem_bytes(w) * (4 * w.d + 3 * w.e)


def bwd_written_bytes(w: I.Workload, ob: int = 4) -> float:
    """The same with the outputs at the width the kernel writes (ob bytes)."""
    return float(w.sequences) * w.T * (elem_bytes(w) * (2 * w.d + 2 * w.e) + ob * (2 * w.d + w.e))


def fwd_algorithmic_bytes(w: I.Workload, ob: int = 4) -> float:
    """la2_fwd reads q, k, v and writes o (ob bytes per element), each once."""
    return float(w.sequences) * w.T * (elem_bytes(w) * (2 * w.d + w.e) + ob * w.e)


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"la2_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = max(smax, float(parts[2]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- CPU oracle

class OracleSample:
    """Fwd+bwd of the fp64 oracle on a bounded sample of a workload.

    The sample is n sequences (b, h), each its first P positions (P = T when
    whole sequences fit the time budget).  A sequence carries the per-head work
    of its positions, so n sequences of P positions stand for n * P / H tokens
    of the metric; the oracle's cost per position does not depend on T (it is a
    linear-time recurrence), so a prefix measures the same rate.
    """

    def __init__(self, w: I.Workload, x, target_s: float):
        import oracle
        oracle.build()
        self.oracle = oracle
        self.w = w
        self.cores = len(os.sched_getaffinity(0))
        B, H = w.B, w.H
        self.lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :],
                                   (B, H)).reshape(-1)
        self.q, self.k, self.v, self.do = (x[n].reshape(B * H, w.T, -1)
                                           for n in ("q", "k", "v", "do"))
        # calibrate on one sequence per core and a short prefix, then size the
        # sample (positions first, then sequences) to about target_s.  The
        # oracle hands its threads sequences in chunks of about 1 GiB of
        # float64, so a prefix is kept short enough that every chunk still
        # holds a sequence for each core.
        n, P = self.cores, min(w.T, 1024)
        dt = self.run(n, P)
        per_pos = max(dt, 1e-4) / (n * P)
        want = max(1, int(target_s / per_pos))
        p_cap = max(1024, (1 << 30) // (8 * self.cores * 4 * (w.d + w.e)))
        P = min(w.T, p_cap, max(P, want // n))
        n = min(64 * self.cores, max(n, want // P))
        self.n, self.P = n, P

    def run(self, n=None, P=None):
        n = self.n if n is None else n
        P = self.P if P is None else P
        idx = np.arange(n) % (self.w.B * self.w.H)
        t = torch.from_numpy(idx)
        qs, ks, vs, ds = (z[t, :P] for z in (self.q, self.k, self.v, self.do))
        t0 = time.perf_counter()
        self.oracle.forward(qs, ks, vs, self.lam[idx], nthreads=self.cores)
        self.oracle.backward(qs, ks, vs, self.lam[idx], ds, nthreads=self.cores)
        return time.perf_counter() - t0

    def rate(self):
        dt = self.run()
        tokens = self.n * self.P / self.w.H
        what = "whole sequences" if self.P == self.w.T else f"sequences, first {self.P} positions each,"
        return {"value": tokens / dt, "unit": "tokens/s", "cores": self.cores, "kind": "oracle",
                "sample": f"{self.n} {what} (b,h) of T={self.w.T}, d={self.w.d}, e={self.w.e}: "
                          f"{tokens:.0f} token-equivalents in {dt:.2f} s"}


def oracle_rate(w: I.Workload, x, target_s: float = 12.0):
    return OracleSample(w, x, target_s).rate()


# -------------------------------------------------------------- main paths

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, w, world, rank):
    if rank != 0:
        return 0
    x = I.make_workload_inputs(w, seed=args.seed)
    # each step is one bounded sample; the whole run stays within a few minutes
    per_step = min(args.ref_seconds, 150.0 / max(1, args.steps))
    sample = OracleSample(w, x, per_step)  # its calibration run doubles as warm-up
    rates = []
    base = None
    for _ in range(max(1, args.steps)):
        r = sample.rate()
        rates.append(r["value"])
        base = r
    value = statistics.median(rates)
    base = dict(base, value=value)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.tokens / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, args):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "e": w.e,
            "block": w.block, "layout": getattr(args, "layout", "bhtd"),
            "global_batch": w.B * args.gpus, "seq_len": w.T,
            "parallelism": f"replicas{args.gpus}",
            "out_dtype": getattr(args, "out_dtype", "f32"),
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)"}


def run_decode(args, world, rank, local):
    """One recurrent decode step (la2_decode) per timed step: one new token for
    each of B*H sequences, state [B, H, d, e] fp32 read and written in place.
    Roofline: HBM, with the state's read and write plus q, k, v in and o out."""
    from causal_linear_attention_la2_b200 import la2
    la2.load()
    dw = I.DECODE_WORKLOADS[args.decode_workload]
    B, H, d, e = dw.B, dw.H, dw.d, dw.e
    dev = torch.device("cuda", local)
    g = torch.Generator().manual_seed(args.seed)
    x = I.make_inputs(B, H, args.steps + args.warmup + 2, d, e, dw.dtype, seed=args.seed)
    lam = x["lam"].to(dev)
    state = (torch.randn(B, H, d, e, generator=g) * 0.1).to(dev)
    tok = [{n: x[n][:, :, t].contiguous().to(dev) for n in ("q", "k", "v")}
           for t in range(args.steps + args.warmup + 2)]
    out = torch.empty(B, H, e, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for t in range(args.warmup):
        flush.fill_(0.0)
        la2.la2_decode(tok[t]["q"], tok[t]["k"], tok[t]["v"], lam, state, out=out)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    launches = 0
    barrier(world)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(float(i))
        t = args.warmup + i
        s, e_ = ev[i]
        s.record(stream)
        la2.la2_decode(tok[t]["q"], tok[t]["k"], tok[t]["v"], lam, state, out=out)
        launches += la2.la2_last_launch_count()
        e_.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop() if clocks else None
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / len(ev), world)
    # end to end: q, k, v of the token from pinned host memory in, o back out
    hq = {n: tok[0][n].cpu().pin_memory() for n in ("q", "k", "v")}
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(5):
        dq_, dk_, dv_ = (hq[n].to(dev, non_blocking=True) for n in ("q", "k", "v"))
        la2.la2_decode(dq_, dk_, dv_, lam, state, out=out)
        hout.copy_(out, non_blocking=True)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / 5, world)
    if rank != 0:
        return 0
    pk, pk_kind = peaks()
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    esz = 2 if dw.dtype == "bf16" else 4
    step_bytes = B * H * (2 * d * e * 4 + (2 * d + e) * esz + e * 4)
    achieved = step_bytes / (step_ms * 1e-3) / 1e9
    value = B * world / (step_ms * 1e-3)
    line = {
        "metric": "decode tokens/s (one new token per sequence, all heads, per la2_decode step)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dw.dtype, "data": "synthetic",
        "config": {"workload": dw.name, "B": B, "H": H, "d": d, "e": e,
                   "state_bytes": B * H * d * e * 4, "parallelism": f"replicas{args.gpus}",
                   "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)"},
        "token_heads_per_s": value * H,
        "roofline": {"bound": "hbm", "kernel": "la2_decode_kernel", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": None,
                     "peak_kind": f"{pk_kind} hbm_gbs"},
        "e2e": {"value": B * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hq.values()),
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "gpu_launches": launches, "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        n = max(1, min(B * H, 256))
        qs = tok[0]["q"].reshape(B * H, d)[:n].float().cpu().numpy()
        ks = tok[0]["k"].reshape(B * H, d)[:n].float().cpu().numpy()
        vs = tok[0]["v"].reshape(B * H, e)[:n].float().cpu().numpy()
        st = state.reshape(B * H, d, e)[:n].cpu().numpy().astype(np.float64)
        lam_n = np.resize(x["lam"].numpy().astype(np.float64), n)
        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < min(args.ref_seconds, 5.0):
            oracle.decode_step(qs, ks, vs, lam_n, st)
            reps += 1
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * n / H / dt, "unit": "tokens/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"{reps} decode steps of {n} sequences (b, h), d={d}, "
                                          f"e={e}, in {dt:.2f} s"}
    print(json.dumps(line), flush=True)
    return 0


def time_steps(la2, fwd, bwd, stream, flush, steps, warmup):
    """CUDA-event times of `steps` fwd and bwd calls after `warmup` untimed
    ones, the L2 flushed (outside the events) before each unless flush is
    None; returns the per-step fwd and bwd times in ms and the kernels
    launched in the timed steps."""
    for _ in range(warmup):
        if flush is not None:
            flush.fill_(0.0)
        fwd()
        bwd()
    torch.cuda.synchronize()
    assert la2.la2_device_status(reset=True) == 0, "kernel reported a device fault in warm-up"
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launches = 0
    for i in range(steps):
        if flush is not None:
            flush.fill_(float(i))
        s, m, e = ev[i]
        s.record(stream)
        fwd()
        launches += la2.la2_last_launch_count()
        m.record(stream)
        bwd()
        launches += la2.la2_last_launch_count()
        e.record(stream)
    torch.cuda.synchronize()
    assert la2.la2_device_status(reset=True) == 0, "kernel reported a device fault"
    return [s.elapsed_time(m) for s, m, _ in ev], [m.elapsed_time(e) for _, m, e in ev], launches


def step_line(w, fwd_ms, bwd_ms, tc, hbm, world=1, ob=4):
    """tokens/s, credited TFLOP/s and roofline figures of one workload's step."""
    f = sum(fwd_ms) / len(fwd_ms)
    b = sum(bwd_ms) / len(bwd_ms)
    step_ms = f + b
    tflops = flops_per_token_head(w) * w.T * w.sequences * world / (step_ms * 1e-3) / 1e12
    return {"tokens_per_s": w.tokens * world / (step_ms * 1e-3), "ms_per_step": step_ms,
            "fwd_ms": f, "bwd_ms": b, "tflops": tflops, "tc_frac": tflops / (tc * world),
            "bwd_hbm_frac": bwd_algorithmic_bytes(w) / (b * 1e-3) / 1e9 / hbm,
            "bwd_hbm_frac_as_written": bwd_written_bytes(w, ob) / (b * 1e-3) / 1e9 / hbm}


def sweep_lines(la2, w, dev_in, dev_out, lam_sweep, dev, stream, flush, args, tc, hbm):
    """The same fwd+bwd step at every sweep length (and at the TNL-15B layer),
    with block 128 and 256, on views of the resident inputs: every sweep point has B T = 131,072, and
    its inputs drawn by the recipe are the same flat buffers reshaped (T =
    92,160, B = 1, and the 15B layer take a prefix of them)."""
    lines = []
    cases = [I.sweep_workload(T, w.block) for T in I.SWEEP_T] + [I.WORKLOADS["tnl15b"]]
    # the pages' other block size for the sweep (T_B = 256: the phase-serial kernel)
    cases += [I.sweep_workload(T, 256) for T in I.SWEEP_T if w.block != 256]
    for ws in cases:
        if ws.d != w.d or ws.e != w.e:
            continue
        nq, nv = ws.sequences * ws.T * ws.d, ws.sequences * ws.T * ws.e
        shp_q, shp_v = (ws.B, ws.H, ws.T, ws.d), (ws.B, ws.H, ws.T, ws.e)
        q, k = (t.reshape(-1)[:nq].view(shp_q) for t in dev_in[:2])
        v, do = (t.reshape(-1)[:nv].view(shp_v) for t in dev_in[2:])
        out = dev_out[0].reshape(-1)[:nv].view(shp_v)
        dq, dk = (t.reshape(-1)[:nq].view(shp_q) for t in dev_out[1:3])
        dv = dev_out[3].reshape(-1)[:nv].view(shp_v)
        lam = lam_sweep if ws.H == w.H else torch.from_numpy(ws.decays().copy()).to(dev)

        od = OUT_TORCH[args.out_dtype]

        def fwd():
            la2.la2_fwd_ex(q, k, v, lam, out=out, block=ws.block, out_dtype=od)

        def bwd():
            la2.la2_bwd_ex(q, k, v, lam, do, dq=dq, dk=dk, dv=dv, block=ws.block, out_dtype=od)

        fm, bm, _ = time_steps(la2, fwd, bwd, stream, flush, args.sweep_steps, 3)
        ent = {"workload": ws.name, "B": ws.B, "T": ws.T, "H": ws.H, "block": ws.block}
        ent.update(step_line(ws, fm, bm, tc, hbm, ob=out_bytes(args.out_dtype)))
        lines.append(ent)
    return lines


def bwd_kernel_label(la2, w) -> str:
    """The kernels of one la2_bwd call, the roofline's unit of measurement."""
    if w.dtype != "bf16":
        return "la2_scan_f32 (la2_bwd launch)"
    if w.block != 128:
        return "la2_scan_blk (la2_bwd launch)"
    plans = la2.la2_plan_info(w.B, w.H, w.T, w.d, w.e, w.block, is_bwd=True)
    if any(p["prepass_ctas"] > 0 for p in plans):
        return "la2_bwd call: la2_state_ws pre-pass + la2_scan_ws"
    return "la2_scan_ws (la2_bwd launch)"


def run_ours(args, w, world, rank, local):
    from causal_linear_attention_la2_b200 import la2
    la2.load()
    dev = torch.device("cuda", local)
    x = I.make_workload_inputs(w, seed=args.seed)
    lay = args.layout
    if lay == "bthd":  # [B, T, H, D]: the model-native layout
        x = dict(x, **{n: x[n].transpose(1, 2).contiguous() for n in ("q", "k", "v", "do")})
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    od = OUT_TORCH[args.out_dtype]
    ob = out_bytes(args.out_dtype)
    o = dict(dtype=od, device=dev)
    out = torch.empty(v.shape, **o)
    dq, dk, dv = torch.empty(q.shape, **o), torch.empty(k.shape, **o), torch.empty(v.shape, **o)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd(qq=q, kk=k, vv=v):
        la2.la2_fwd_ex(qq, kk, vv, lam, lay, out=out, block=w.block, out_dtype=od)

    def bwd(qq=q, kk=k, vv=v, dd=do):
        la2.la2_bwd_ex(qq, kk, vv, lam, dd, lay, dq=dq, dk=dk, dv=dv, block=w.block, out_dtype=od)

    for _ in range(args.warmup):
        flush.fill_(0.0)
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    assert la2.la2_device_status(reset=True) == 0, "kernel reported a device fault in warm-up"

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    fwd_ms, bwd_ms, launches = time_steps(la2, fwd, bwd, stream, flush, args.steps, 0)
    barrier(world)
    clk = clocks.stop() if clocks else None
    step_ms = max_over_ranks(sum(fwd_ms) / len(fwd_ms) + sum(bwd_ms) / len(bwd_ms), world)
    # the same steps back to back without the L2 flush (context only: every
    # workload but tiny_f32 holds more than the 126 MB L2)
    nf_f, nf_b, _ = time_steps(la2, fwd, bwd, stream, None, args.steps, 1)
    step_ms_no_flush = max_over_ranks(sum(nf_f) / len(nf_f) + sum(nf_b) / len(nf_b), world)

    # end to end through the public API: pinned host in -> device -> host out.
    # The four outputs are read back into one pinned buffer, one after the
    # other (every byte still crosses PCIe; the host copy is not kept).
    hosts = {n: x[n].pin_memory() for n in ("q", "k", "v", "do")}
    hout = torch.empty(max(t.numel() for t in (out, dq, dk, dv)), dtype=od, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in hosts.values())
    d2h = sum(t.numel() * t.element_size() for t in (out, dq, dk, dv))
    e2e_steps = max(2, min(args.steps, 5))

    def e2e_step():
        qd, kd, vd, dd = (hosts[n].to(dev, non_blocking=True) for n in ("q", "k", "v", "do"))
        fwd(qd, kd, vd)
        bwd(qd, kd, vd, dd)
        for dsrc in (out, dq, dk, dv):
            hout[:dsrc.numel()].copy_(dsrc.reshape(-1), non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / e2e_steps, world)
    barrier(world)
    del hosts, hout

    if rank != 0:
        return 0

    pk, pk_kind = peaks()
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tc_sus = float(pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    tokens_per_step = w.tokens * world
    value = tokens_per_step / (step_ms * 1e-3)
    bwd_avg_ms = sum(bwd_ms) / len(bwd_ms)
    achieved = bwd_algorithmic_bytes(w) / (bwd_avg_ms * 1e-3) / 1e9
    written = bwd_written_bytes(w, ob) / (bwd_avg_ms * 1e-3) / 1e9
    traffic = None
    try:
        with open(PROFILE_TRAFFIC) as f:
            t = json.load(f)
        ent = t.get(w.name, {})
        if ent.get("source_hash") == kernel_source_hash():
            traffic = ent.get("bwd_dram_bytes_per_call")
    except (OSError, ValueError):
        pass
    tflops = flops_per_token_head(w) * w.T * w.sequences * world / (step_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic", "config": workload_config(w, args),
        "tflops": tflops, "tc_frac": tflops / (tc * world), "tc_peak_tflops": tc,
        "tc_frac_sustained": tflops / (tc_sus * world), "tc_peak_sustained_tflops": tc_sus,
        "tflops_executed": executed_flops_per_token_head(w) * w.T * w.sequences * world / (step_ms * 1e-3) / 1e12,
        "ms_per_step_no_l2_flush": step_ms_no_flush,
        "fwd_ms": sum(fwd_ms) / len(fwd_ms), "bwd_ms": bwd_avg_ms,
        "roofline": {"bound": "hbm", "kernel": bwd_kernel_label(la2, w),
                     "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "peak_kind": f"{pk_kind} hbm_gbs",
                     "bytes": "q, k, v, dO in and dq, dk, dv out, each once at the input width",
                     "out_dtype": args.out_dtype,
                     "achieved_as_written": written, "frac_as_written": written / hbm},
        "e2e": {"value": tokens_per_step / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if w.dtype == "bf16":
        # the launch plans the two calls ran (schedule, segments, CTAs, pre-pass)
        line["plan"] = {"fwd": la2.la2_plan_info(w.B, w.H, w.T, w.d, w.e, w.block),
                        "bwd": la2.la2_plan_info(w.B, w.H, w.T, w.d, w.e, w.block, is_bwd=True)}
    if (world == 1 and lay == "bhtd" and w.name.startswith("sweep_") and args.sweep_steps > 0
            and w.B * w.T == 131072):
        line["sweep"] = sweep_lines(la2, w, (q, k, v, do), (out, dq, dk, dv), lam, dev, stream,
                                    flush, args, tc, hbm)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_rate(w, x, target_s=args.ref_seconds)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="sweep_T131072_blk128", choices=sorted(I.WORKLOADS))
    ap.add_argument("--sweep-steps", type=int, default=5,
                    help="timed steps per entry of the sweep object (0: leave it out)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layout", default="bhtd", choices=["bhtd", "bthd"],
                    help="tensor layout of the fwd+bwd step: [B,H,T,D] or [B,T,H,D]")
    ap.add_argument("--mode", default="train", choices=["train", "decode"],
                    help="train: la2_fwd + la2_bwd (the default line); decode: la2_decode steps")
    ap.add_argument("--decode-workload", default="decode_tnl15b", choices=sorted(I.DECODE_WORKLOADS))
    ap.add_argument("--out-dtype", default="f32", choices=sorted(OUT_TORCH),
                    help="element type of o, dq, dk, dv (bf16 needs bf16 inputs)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")
    w = I.WORKLOADS[args.workload]
    if w.dtype != "bf16":
        args.out_dtype = "f32"
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return run_reference(args, w, world, rank)
        if args.mode == "decode":
            return run_decode(args, world, rank, local)
        return run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
