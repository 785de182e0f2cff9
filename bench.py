#!/usr/bin/env python
"""Benchmark of the gated modal long convolution (prefill + O(1) decode) on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
filter materialisation, filter spectrum, FFT long convolution with gating and
prompt -> state reduction over a B x L prompt (one hyena_prefill call), then T
decode steps (one hyena_decode_step call each, replayed from a CUDA graph).
Default workload: the mid-size operator, B=8, L=4096, Dch=1024, H=8, d=16,
bf16 activations, complex fp32 state, FFT length 8192, 256 decode steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU: the
sequences are independent, so the data-parallel shards need no collective;
timing is the max over ranks.  Rank 0 prints one JSON line.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and prefill tokens/s on 1 B200; % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ multi-rank plumbing
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(
        os.environ.get("LOCAL_RANK", 0))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def reduce_max(x: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ roofline bookkeeping
def algorithmic_bytes(w):
    """Bytes the method must move (DRAM), per prefill call and per decode launch."""
    a = w.act_bytes
    prefill = w.B * w.L * w.Dch * 4 * a + w.B * w.d * w.Dch * 8
    decode = w.B * w.Dch * (4 * a + 16 * w.d)
    return prefill, decode


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))[workload][kernel]
    except Exception:
        return None
    if d.get("source_hash") != source_hash(d.get("sources", [])):
        return None
    return d.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def gpu_id_for(device) -> str:
    import torch
    try:
        pr = torch.cuda.get_device_properties(device)
        return "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[device.index] if vis else str(device.index)


# ------------------------------------------------------------------ CPU (oracle) timing
class OracleSample:
    """Inputs of the workload drawn once; the fp64 oracle (recurrent mode: prompt then
    T decode tokens) is timed on the first `channels` channels of every sequence."""

    def __init__(self, w, layer: int = 0):
        import torch

        from distilled_ssm_decode_b200 import workloads as W
        self.w = w
        self.p = W.params(w, layer)
        q, k, v = W.prefill_inputs(w, layer)
        if w.T:
            dec = [W.decode_inputs(w, t, layer) for t in range(w.T)]
            q = torch.cat([q, torch.stack([x[0] for x in dec], 1)], 1)
            k = torch.cat([k, torch.stack([x[1] for x in dec], 1)], 1)
            v = torch.cat([v, torch.stack([x[2] for x in dec], 1)], 1)
        self.qkv = (q, k, v)

    def run(self, channels: int):
        """Returns (seconds, token-equivalents processed)."""
        import oracle
        from distilled_ssm_decode_b200 import workloads as W
        w = self.w
        qs, ks, vs = (W.to_f64(t[:, :, :channels].contiguous()) for t in self.qkv)
        ch = w.Dch // w.H
        heads = [c // ch for c in range(channels)]
        t0 = time.perf_counter()
        oracle.recurrent(qs, ks, vs, self.p.lam[heads], self.p.R[heads], self.p.Dskip[heads],
                         H=channels)
        dt = time.perf_counter() - t0
        return dt, w.B * (w.L + w.T) * channels / w.Dch

    def calibrate(self, target_s: float) -> int:
        dt, _ = self.run(16)
        c = int(16 * target_s / max(dt, 1e-4))
        return max(16, min(self.w.Dch, c))


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args):
    rank, world = dist_init("gloo")
    if rank != 0:
        return 0
    import oracle
    from distilled_ssm_decode_b200 import workloads as W
    oracle.build()
    w = W.WORKLOADS[args.workload]
    sample = OracleSample(w)
    channels = sample.calibrate(1.0)
    for _ in range(args.warmup):
        sample.run(channels)
    total, tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, t = sample.run(channels)
        total += dt
        tok += t
    value = tok / total
    cores = oracle.threads()
    desc = (f"fp64 oracle, recurrent mode: all {w.B} sequences x first {channels} of {w.Dch} "
            f"channels, {w.L}-token prompt + {w.T} decode tokens per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    return {"workload": (f"{w.name}: B={w.B} L={w.L} Dch={w.Dch} H={w.H} d={w.d} "
                         f"{w.dtype} activations, complex fp32 state, FFT length {w.fft_len}, "
                         f"{w.T} decode steps"),
            "B": w.B, "L": w.L, "Dch": w.Dch, "H": w.H, "d": w.d, "fft_len": w.fft_len,
            "decode_steps": w.T, "activations": w.dtype, "parallelism": "data-parallel replicas"}


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    from distilled_ssm_decode_b200 import build, ops
    from distilled_ssm_decode_b200 import workloads as W
    build.build()
    ops.lib()

    w = W.WORKLOADS[args.workload]
    p = W.params(w)
    lam, R, D = p.lam_f32().to(dev), p.R_f32().to(dev), p.Dskip_f32().to(dev)
    q_h, k_h, v_h = W.prefill_inputs(w)
    dec_h = [W.decode_inputs(w, t) for t in range(w.T)]
    dq_h = torch.stack([x[0] for x in dec_h])
    dk_h = torch.stack([x[1] for x in dec_h])
    dv_h = torch.stack([x[2] for x in dec_h])
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    dq, dk, dv = dq_h.to(dev), dk_h.to(dev), dv_h.to(dev)
    y = torch.empty_like(q)
    ydec = torch.empty_like(dq)
    state = torch.empty((w.B, w.d, w.Dch, 2), dtype=torch.float32, device=dev)
    ws = torch.empty(ops.prefill_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d, w.fft_len),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)

    def prefill():
        ops.prefill(q, k, v, lam, R, D, w.fft_len, y=y, state=state, workspace=ws)

    def decode_all():
        for t in range(w.T):
            ops.decode_step(dq[t], dk[t], dv[t], lam, R, D, state, y=ydec[t])

    with torch.cuda.stream(stream):
        prefill()
        decode_all()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        decode_all()
    torch.cuda.synchronize(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        prefill()
        if ev is not None:
            ev[1].record(stream)
        g.replay()
        if ev is not None:
            ev[2].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)

    # ---- timed region (device-resident inputs)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_id_for(dev))
    clocks.start()
    time.sleep(0.3)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clk = clocks.stop()
    elapsed_ms = reduce_max(t_start.elapsed_time(t_end), dev)
    pre_ms = reduce_max(sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps, dev)
    dec_ms = reduce_max(sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps, dev)
    ms_per_step = elapsed_ms / args.steps

    tokens_step = w.B * (w.L + w.T)
    value = world * tokens_step / (ms_per_step / 1e3)
    pre_tok = world * w.B * w.L / (pre_ms / 1e3)
    dec_tok = world * w.B * w.T / (dec_ms / 1e3)
    peak, peak_src = load_peaks()
    pb, db = algorithmic_bytes(w)
    pre_gbs = pb / (pre_ms / 1e3) / 1e9
    dec_launch_ms = dec_ms / max(w.T, 1)
    dec_gbs = db / (dec_launch_ms / 1e3) / 1e9
    roof_pre = {"kernel": "hyena_prefill (filter + spectrum + fused FFT conv/gate/state)",
                "bound": "hbm", "achieved": pre_gbs, "peak": peak, "unit": "GB/s",
                "frac": pre_gbs / peak, "peak_source": peak_src,
                "algorithmic_bytes": pb, "launch_ms": pre_ms,
                "traffic": ncu_traffic("prefill_fused", w.name)}
    roof_dec = {"kernel": "hyena_decode_step", "bound": "hbm", "achieved": dec_gbs, "peak": peak,
                "unit": "GB/s", "frac": dec_gbs / peak, "peak_source": peak_src,
                "algorithmic_bytes": db, "launch_ms": dec_launch_ms,
                "traffic": ncu_traffic("decode", w.name)}
    dominant = roof_dec if dec_ms > pre_ms else roof_pre

    # ---- end to end: host (pinned) inputs, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.pin_memory()  # noqa: E731
        qp, kp, vp = pin(q_h), pin(k_h), pin(v_h)
        dqp, dkp, dvp = pin(dq_h), pin(dk_h), pin(dv_h)
        yp, ydp = torch.empty_like(qp).pin_memory(), torch.empty_like(dqp).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in (qp, kp, vp, dqp, dkp, dvp))
        bo = yp.numel() * yp.element_size() + ydp.numel() * ydp.element_size()

        def e2e_step():
            for dst, src in ((q, qp), (k, kp), (v, vp), (dq, dqp), (dk, dkp), (dv, dvp)):
                dst.copy_(src, non_blocking=True)
            step()
            yp.copy_(y, non_blocking=True)
            ydp.copy_(ydec, non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(max(1, min(args.warmup, 3))):
                e2e_step()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(args.steps):
                e2e_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = reduce_max(a.elapsed_time(b), dev) / args.steps
        e2e = {"value": world * tokens_step / (e2e_ms / 1e3), "unit": "tokens/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}

    # ---- CPU baseline: the oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        sample = OracleSample(w)
        channels = sample.calibrate(12.0)
        dt, tok = sample.run(channels)
        cpu = {"value": tok / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
               "sample": (f"fp64 oracle, recurrent mode, one step on all {w.B} sequences x first "
                          f"{channels} of {w.Dch} channels ({w.L}-token prompt + {w.T} decode "
                          f"tokens); {dt:.1f} s")}

    if rank == 0:
        cfg = workload_config(w)
        cfg["l2"] = ("prefill inputs larger than L2 (3 x %d MiB); decode state %.1f MiB stays "
                     "L2-resident between steps, as in real decoding"
                     % (q.numel() * q.element_size() >> 20, state.numel() * 4 / 2 ** 20))
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic", "config": cfg,
                "prefill": {"tokens_per_s": pre_tok, "ms": pre_ms, "hbm_frac": pre_gbs / peak},
                "decode": {"tokens_per_s": dec_tok, "ms_per_token_step": dec_launch_ms,
                           "hbm_frac": dec_gbs / peak},
                "roofline": dominant, "roofline_all": [roof_pre, roof_dec],
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": args.steps * (3 + w.T), "clocks": clk}
        print(json.dumps(line), flush=True)
    del g
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mid_bf16")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
