#!/usr/bin/env python
"""Benchmark of the gated modal long convolution (prefill + O(1) decode) on B200.

Default line: the 1.3B-shaped generation workload, 24 independent operator layers, each
B=64, L=512, Dch=2048, H=16, d=16, bf16 activations, complex fp32 state.  One step = the
chunked tensor-core prefill of every layer's 512-token prompt (one launch), then 512 decode
tokens, each one grouped decode launch over all 24 layers (replayed from a CUDA graph).  The
same run adds sub-records, each timed on its own: the tiny fp32 operator (FFT prefill and 32
decode steps), the mid-size operator (prefill and decode), the long prefill (65536 tokens,
with its end-to-end time) and the decode batch sweep at B = 1, 16, 64, 256 and 1024.  Every
sub-record carries its roofline entries.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-subrecords] ...

Under torchrun (N > 1) every rank runs the headline workload on its own GPU: sequences and
layers are independent, so the data-parallel replicas need no collective; timing is the max
over ranks and rank 0 prints one JSON line (sub-records are single-GPU figures, N = 1 only).
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and prefill tokens/s on 1 B200; % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "gen1p3b_bf16"


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


LEAD_SPIN_CYCLES = 4_000_000       # ~2 ms at the B200's clock


def source_hash(paths) -> str:
    """Hash of the kernel sources with C/C++ comments removed and white space collapsed: a capture
    stays valid across comment and layout edits and is dropped as soon as any code changes."""
    h = hashlib.sha256()
    for p in paths:
        text = open(os.path.join(ROOT, p), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.json, keyed by
    workload name and batch), or None if there is none or the kernel source changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))[workload][kernel]
    except Exception:
        return None
    if d.get("source_hash") != source_hash(d.get("sources", [])):
        return None
    return d.get("bytes_per_launch")


def roof(kernel, nbytes, launch_ms, peak, peak_src, traffic=None, total_ms=None, note=None):
    """Roofline entry: algorithmic bytes of one launch over its measured duration."""
    gbs = nbytes / (launch_ms / 1e3) / 1e9
    r = {"kernel": kernel, "bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
         "frac": gbs / peak, "peak_source": peak_src, "algorithmic_bytes": nbytes,
         "launch_ms": launch_ms, "total_ms": launch_ms if total_ms is None else total_ms,
         "traffic": traffic}
    if note:
        r["note"] = note
    return r


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


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


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

    def calibrate(self, target_s: float):
        """(channels, repeats): a sample of about target_s seconds of oracle work.  When the
        whole workload takes less than that, it is run `repeats` times."""
        dt, _ = self.run(16)
        c = int(16 * target_s / max(dt, 1e-4))
        c = max(16, min(self.w.Dch, c))
        reps = 1
        if c == self.w.Dch:
            dt_all, _ = self.run(c)
            reps = max(1, int(round(target_s / max(dt_all, 1e-4))))
        return c, reps

    def run_reps(self, channels: int, reps: int):
        total, tok = 0.0, 0.0
        for _ in range(reps):
            dt, t = self.run(channels)
            total += dt
            tok += t
        return total, tok


def oracle_baseline(w, nl: int, target_s: float):
    """The fp64 oracle on the host cores: tokens/s of the whole workload (layer 0 timed, divided by
    the layer count), with a description of the sample."""
    import oracle
    oracle.build()
    sample = OracleSample(w)
    channels, reps = sample.calibrate(target_s)
    dt, tok = sample.run_reps(channels, reps)
    desc = (f"fp64 oracle, recurrent mode: {reps} pass(es) over all {w.B} sequences x first {channels} of "
            f"{w.Dch} channels ({w.L}-token prompt + {w.T} decode tokens), {dt:.1f} s"
            + (f"; layer 0 only, tokens/s divided by {nl} layers" if nl > 1 else ""))
    return {"value": tok / dt / nl, "unit": "tokens/s", "cores": oracle.threads(), "cpu_model": cpu_model(),
            "kind": "oracle", "sample": desc}, sample, channels, reps


# ------------------------------------------------------------------ the line's config (both arms)
def line_config(w, nl: int):
    layers = f", {nl} independent layers" if nl > 1 else ""
    return {"workload": (f"{w.name}: B={w.B} L={w.L} Dch={w.Dch} H={w.H} d={w.d} {w.dtype} activations, "
                         f"complex fp32 state, FFT length {w.fft_len}, {w.T} decode steps{layers}"),
            "B": w.B, "L": w.L, "Dch": w.Dch, "H": w.H, "d": w.d, "fft_len": w.fft_len,
            "decode_steps": w.T, "layers": nl, "activations": w.dtype,
            "parallelism": "data-parallel replicas",
            "l2": "inputs larger than L2 (prefill q,k,v per call; decode states of the batch-256+ and "
                  "multi-layer workloads)"}


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args):
    rank, world = dist_init("gloo")
    if rank != 0:
        return 0
    import oracle
    from distilled_ssm_decode_b200 import workloads as W
    oracle.build()
    w = W.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(B=args.batch)
    nl = args.layers or w.layers
    sample = OracleSample(w)
    channels, reps = sample.calibrate(1.0)
    for _ in range(args.warmup):
        sample.run_reps(channels, reps)
    total, tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, t = sample.run_reps(channels, reps)
        total += dt
        tok += t
    value = tok / total / nl
    desc = (f"fp64 oracle, recurrent mode: all {w.B} sequences x first {channels} of {w.Dch} "
            f"channels, {w.L}-token prompt + {w.T} decode tokens, {reps} pass(es) per step"
            + (f"; layer 0 only, tokens/s divided by {nl} layers" if nl > 1 else ""))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": line_config(w, nl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ shared timing helpers
def timed_steps(stream, dev, steps: int, warmup: int, step, nsec: int, lead_spin: bool = True):
    """Run `warmup` untimed steps, then `steps` timed ones on `stream`.  step(ev) records
    ev[0..nsec] around its sections.  Returns (elapsed ms of all steps, [mean ms per section])."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step(None)
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nsec + 1)] for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        if lead_spin:
            # a short GPU spin ahead of the start event, so that the first step's launches are queued
            # while the GPU is busy: the timed region then holds device work only, as every later step
            # does (each is queued while the previous one runs)
            torch.cuda._sleep(LEAD_SPIN_CYCLES)
        t_start.record(stream)
        for i in range(steps):
            step(evs[i])
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    elapsed = reduce_max(t_start.elapsed_time(t_end), dev)
    secs = [reduce_max(sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps, dev) for j in range(nsec)]
    return elapsed, secs


def make_pinned(shape, dtype):
    import torch
    return torch.empty(shape, dtype=dtype, pin_memory=True)


def fir_baseline(ops, W, w, q, k, v, dq, dk, dv, lam, R, D, stream, dev, nsteps, modal_step_ms,
                 prefill_ms, peak, layers=1):
    """Generation without the distilled recurrence, on the same inputs: each token convolves the
    cached history with the long filter (O(t) per token).  Times `nsteps` tokens after the
    prompt (CUDA graph; `layers` launches per token over one shared history, so every launch
    streams it from DRAM like a layer of its own would); the re-prefill cost per token is at
    least one prefill of the prompt."""
    import torch
    t_max = w.L + nsteps
    h = ops.filter_from_modes(lam, R, D, t_max)
    u = ops.fir_cache_prompt(k, v, t_max)
    y = torch.empty((w.B, w.Dch), dtype=w.torch_dtype, device=dev)

    def run():
        for t in range(nsteps):
            i = t % dq.shape[0]
            for _ in range(layers):
                ops.fir_decode_step(dq[i], dk[i], dv[i], h, u, w.L + t, y=y)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        a.record(stream)
        for _ in range(3):
            g.replay()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / 3 / nsteps
    t_mid = w.L + (nsteps - 1) / 2
    hist_bytes = layers * w.B * w.Dch * (t_mid * 4 + 4 * w.act_bytes + 4)
    del g
    return {"fir_decode": {"what": (f"cached-activation long convolution per token (no distillation), tokens "
                                    f"{w.L}..{w.L + nsteps - 1}" + (f", {layers} layers" if layers > 1 else "")),
                           "ms_per_token_step": ms, "tokens_per_s": w.B / (ms / 1e3),
                           "hbm_frac": hist_bytes / (ms / 1e3) / 1e9 / peak,
                           "modal_decode_speedup": ms / modal_step_ms},
            "reprefill_per_token": {"what": "lower bound: one chunked prefill of the prompt per generated token",
                                    "ms_per_token_step": prefill_ms, "modal_decode_speedup": prefill_ms / modal_step_ms}}


# ------------------------------------------------------------------ one-layer workloads
def measure_single(args, w, dev, steps: int, warmup: int, e2e_steps: int, with_fft_route: bool,
                   with_baselines: bool, with_e2e: bool):
    """Prefill (chunked route when supported, else FFT) and T decode steps of one workload.
    Returns a record with separate prefill and decode figures, each with its roofline entry."""
    import torch

    from distilled_ssm_decode_b200 import ops
    from distilled_ssm_decode_b200 import workloads as W
    _, world, _ = dist_env()
    has_pre, has_dec = w.L > 0, w.T > 0
    use_chunked = has_pre and args.prefill != "fft" and ops.lib().hyena_prefill_chunked_workspace_bytes(
        w.B, w.L, w.Dch, w.H, w.d) > 0
    if args.prefill == "chunked" and has_pre and not use_chunked:
        raise SystemExit(f"chunked prefill does not support workload {w.name}")
    p = W.params(w)
    lam, R, D = p.lam_f32().to(dev), p.R_f32().to(dev), p.Dskip_f32().to(dev)
    stream = torch.cuda.Stream(dev)
    state = torch.empty((w.B, w.d, w.Dch, 2), dtype=torch.float32, device=dev)
    key = f"{w.name}/B{w.B}"

    # ---- inputs (resident in HBM before the timed region)
    host = {}
    if has_pre:
        host["q"], host["k"], host["v"] = W.prefill_inputs(w)
        q, k, v = host["q"].to(dev), host["k"].to(dev), host["v"].to(dev)
        y = torch.empty_like(q)
        ws = torch.empty(max(1, ops.prefill_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d, w.fft_len)),
                         dtype=torch.uint8, device=dev)
        if use_chunked:
            ws_c = torch.empty(ops.prefill_chunked_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d),
                               dtype=torch.uint8, device=dev)
    else:
        state.copy_(torch.view_as_real(W.initial_state(w)).to(dev))
    if has_dec:
        pool = w.T if w.B * w.Dch * w.T <= (1 << 26) else 32
        if pool == w.T:
            dec = [W.decode_inputs(w, t) for t in range(w.T)]
            host["dq"] = torch.stack([x[0] for x in dec])
            host["dk"] = torch.stack([x[1] for x in dec])
            host["dv"] = torch.stack([x[2] for x in dec])
            dq, dk, dv = host["dq"].to(dev), host["dk"].to(dev), host["dv"].to(dev)
        else:
            dq, dk, dv = W.decode_pool_device(w, pool, device=dev)
        ydec = torch.empty((w.T, w.B, w.Dch), dtype=w.torch_dtype, device=dev)

    def prefill_fft():
        ops.prefill(q, k, v, lam, R, D, w.fft_len, y=y, state=state, workspace=ws)

    # which FFT route the library takes for these tensors (tensor cores for bf16 at 4096..16384)
    fft_tc = has_pre and ops.prefill_uses_tensor_cores(q, k, v, w.H, w.d, w.fft_len, y=y)
    fft_label = ("hyena_prefill (filter + spectrum + tensor-core FFT conv/gate/state)" if fft_tc
                 else "hyena_prefill (filter + spectrum + fused FFT conv/gate/state)")
    fft_kernel = "prefill_monarch" if fft_tc else "prefill_fused"

    def prefill_chunked():
        ops.prefill_chunked(q, k, v, lam, R, D, y=y, state=state, workspace=ws_c)

    prefill = prefill_chunked if use_chunked else prefill_fft

    def decode_all():
        for t in range(w.T):
            i = t % dq.shape[0]
            ops.decode_step(dq[i], dk[i], dv[i], lam, R, D, state, y=ydec[t])

    g = None
    with torch.cuda.stream(stream):
        if has_pre:
            prefill()
        if has_dec:
            decode_all()
    torch.cuda.synchronize(dev)
    if has_dec:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            decode_all()
        torch.cuda.synchronize(dev)

    def step(ev):
        if ev is not None:
            ev[0].record(stream)
        if has_pre:
            prefill()
        if ev is not None:
            ev[1].record(stream)
        if has_dec:
            g.replay()
        if ev is not None:
            ev[2].record(stream)

    elapsed_ms, (pre_ms, dec_ms) = timed_steps(stream, dev, steps, warmup, step, 2)
    ms_per_step = elapsed_ms / steps
    peak, peak_src = load_peaks()
    pb, db = algorithmic_bytes(w)
    rec = {"workload": line_config(w, 1)["workload"], "steps": steps, "warmup": warmup,
           "ms_per_step": ms_per_step,
           "value": world * w.B * (w.L + w.T) / (ms_per_step / 1e3), "unit": "tokens/s"}
    roofs = []
    if has_pre:
        name = "hyena_prefill_chunked (tcgen05 chunked conv/gate/state)" if use_chunked else fft_label
        r = roof(name, pb, pre_ms, peak, peak_src,
                 ncu_traffic("prefill_chunk" if use_chunked else fft_kernel, key))
        roofs.append(r)
        rec["prefill"] = {"route": "chunked" if use_chunked else ("fft, tensor cores" if fft_tc else "fft"),
                          "tokens_per_s": world * w.B * w.L / (pre_ms / 1e3), "ms": pre_ms,
                          "hbm_frac": r["frac"], "roofline": r,
                          "inputs": "q, k, v of %d MiB each (larger than L2)" % (w.B * w.L * w.Dch * w.act_bytes >> 20)}
        if use_chunked:
            err = ops.chunked_error(ws_c, w.B, w.L, w.Dch, w.H, w.d)
            if err:
                raise SystemExit(f"chunked prefill kernel reported error {err}")
    if has_dec:
        launch_ms = dec_ms / w.T
        st_mib = state.numel() * 4 / 2 ** 20
        l2_res = st_mib < 100
        note = (f"the {st_mib:.1f} MiB state stays in L2 between steps, so a step reads no DRAM and is bound by "
                "launch and L2 latency; the HBM fraction is not its bound") if l2_res else None
        r = roof("hyena_decode_step", db, launch_ms, peak, peak_src, ncu_traffic("decode", key), dec_ms, note)
        roofs.append(r)
        rec["decode"] = {"tokens_per_s": world * w.B * w.T / (dec_ms / 1e3), "ms_per_token_step": launch_ms,
                         "hbm_frac": r["frac"], "roofline": r,
                         "state": "%.1f MiB, %s" % (st_mib, "L2-resident between steps" if l2_res else "larger than L2"),
                         "inputs": ("%d distinct input sets, cycled" % dq.shape[0]) if dq.shape[0] != w.T
                         else "one input set per step"}
    # the FFT route (zero-padded FFT long convolution) timed on the same inputs
    if has_pre and use_chunked and with_fft_route:
        def fstep(ev):
            if ev is not None:
                ev[0].record(stream)
            prefill_fft()
            if ev is not None:
                ev[1].record(stream)
        _, (fms,) = timed_steps(stream, dev, steps, 3, fstep, 1)
        r = roof(fft_label, pb, fms, peak, peak_src, ncu_traffic(fft_kernel, key))
        rec["prefill_fft_route"] = {"fft_len": w.fft_len, "tensor_cores": bool(fft_tc),
                                    "tokens_per_s": world * w.B * w.L / (fms / 1e3),
                                    "ms": fms, "hbm_frac": r["frac"], "roofline": r}
    rec["roofline_all"] = roofs
    rec["roofline"] = max(roofs, key=lambda x: x["total_ms"])
    rec["launches_per_step"] = (0 if not has_pre else (2 if use_chunked else (3 if w.fft_len <= 16384 else 8))) + w.T
    if has_pre and has_dec and with_baselines:
        rec["baselines"] = fir_baseline(ops, W, w, q, k, v, dq, dk, dv, lam, R, D, stream, dev, w.T,
                                        dec_ms / w.T, pre_ms, peak)

    # ---- end to end: host (pinned) inputs, copies inside the timed region.  Every step copies its
    # inputs in from pinned host memory and its results (prefill y and every decode y) out to
    # pinned host memory.  Two buffer sets let step i+1's inputs travel in, and step i-1's results
    # travel out, while step i computes (copy-in, compute and copy-out streams; PCIe is full duplex).
    if with_e2e and all(x in host for x in ("q", "k", "v")) and (not has_dec or "dq" in host):
        pins = {n: t.pin_memory() for n, t in host.items()}
        sets = []
        for j in range(2):
            bs = {n: torch.empty_like(t, device=dev) for n, t in host.items()}
            bs["y"] = torch.empty_like(bs["q"])
            bs["state"] = torch.empty_like(state)
            if has_dec:
                bs["ydec"] = torch.empty_like(ydec)
            bs["yp"] = torch.empty_like(pins["q"]).pin_memory()
            bs["ydp"] = torch.empty(tuple(ydec.shape), dtype=ydec.dtype).pin_memory() if has_dec else None
            sets.append(bs)
        bi = sum(t.numel() * t.element_size() for t in pins.values())
        bo = sets[0]["yp"].numel() * sets[0]["yp"].element_size() + \
            (sets[0]["ydp"].numel() * sets[0]["ydp"].element_size() if has_dec else 0)

        def compute(bs):
            if use_chunked:
                ops.prefill_chunked(bs["q"], bs["k"], bs["v"], lam, R, D, y=bs["y"], state=bs["state"],
                                    workspace=ws_c)
            else:
                ops.prefill(bs["q"], bs["k"], bs["v"], lam, R, D, w.fft_len, y=bs["y"], state=bs["state"],
                            workspace=ws)
            if has_dec:
                bs["graph"].replay()

        if has_dec:       # one decode graph per buffer set
            for bs in sets:
                def dec(bs=bs):
                    for t in range(w.T):
                        ops.decode_step(bs["dq"][t], bs["dk"][t], bs["dv"][t], lam, R, D, bs["state"],
                                        y=bs["ydec"][t])
                with torch.cuda.stream(stream):
                    dec()
                torch.cuda.synchronize(dev)
                bs["graph"] = torch.cuda.CUDAGraph()
                with torch.cuda.graph(bs["graph"], stream=stream):
                    dec()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        done_c = [ev(), ev()]       # compute on set j finished (its inputs may be overwritten)
        done_o = [ev(), ev()]       # results of set j copied out (its outputs may be overwritten)
        for e in done_c + done_o:
            e.record(stream)

        def e2e_run(n, t0=None, t1=None):
            for i in range(n):
                j = i % 2
                bs = sets[j]
                s_in.wait_event(done_c[j])
                if t0 is not None and i == 0:
                    t0.record(s_in)
                with torch.cuda.stream(s_in):
                    for name in pins:
                        bs[name].copy_(pins[name], non_blocking=True)
                got = ev()
                got.record(s_in)
                stream.wait_event(got)
                stream.wait_event(done_o[j])
                with torch.cuda.stream(stream):
                    compute(bs)
                done_c[j].record(stream)
                s_out.wait_event(done_c[j])
                with torch.cuda.stream(s_out):
                    bs["yp"].copy_(bs["y"], non_blocking=True)
                    if has_dec:
                        bs["ydp"].copy_(bs["ydec"], non_blocking=True)
                done_o[j].record(s_out)
            if t1 is not None:
                t1.record(s_out)

        e2e_run(3)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        e2e_run(e2e_steps, a, b)
        torch.cuda.synchronize(dev)
        e2e_ms = reduce_max(a.elapsed_time(b), dev) / e2e_steps
        if use_chunked:
            err = ops.chunked_error(ws_c, w.B, w.L, w.Dch, w.H, w.d)
            if err:
                raise SystemExit(f"chunked prefill kernel reported error {err} (end-to-end run)")
        rec["e2e"] = {"value": world * w.B * (w.L + w.T) / (e2e_ms / 1e3), "unit": "tokens/s",
                      "ms_per_step": e2e_ms, "steps": e2e_steps, "h2d_bytes_per_step": bi,
                      "d2h_bytes_per_step": bo,
                      "overlap": "two buffer sets; copy-in, compute and copy-out streams"}
        for bs in sets:
            bs.pop("graph", None)
    del g
    return rec


# ------------------------------------------------------------------ multi-layer workload
def measure_layers(args, w, nl: int, dev, steps: int, warmup: int, e2e_steps: int, with_baselines: bool,
                   with_e2e: bool, clocks=None):
    """Every layer of a multi-layer workload: per step, the chunked prefill of each layer's prompt,
    then T decode steps, each one grouped launch over all layers (CUDA graph).  Inputs are drawn on
    the device (seeded); each layer has its own parameters, state and activations."""
    import torch

    from distilled_ssm_decode_b200 import ops
    from distilled_ssm_decode_b200 import workloads as W
    _, world, _ = dist_env()
    if ops.lib().hyena_prefill_chunked_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d) == 0:
        raise SystemExit(f"chunked prefill does not support workload {w.name}")
    ps = [W.params(w, layer=l) for l in range(nl)]
    lams = [p.lam_f32().to(dev) for p in ps]
    Rs = [p.R_f32().to(dev) for p in ps]
    Ds = [p.Dskip_f32().to(dev) for p in ps]
    states = [torch.empty((w.B, w.d, w.Dch, 2), dtype=torch.float32, device=dev) for _ in range(nl)]
    qkv = [W.prefill_inputs_device(w, l, device=dev) for l in range(nl)]
    ys = [torch.empty_like(x[0]) for x in qkv]
    ws = torch.empty(ops.prefill_chunked_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d), dtype=torch.uint8,
                     device=dev)
    # every layer's prefill in one launch (the layers' work items share the persistent grid)
    pset = ops.PrefillLayerSet([x[0] for x in qkv], [x[1] for x in qkv], [x[2] for x in qkv], ys, states,
                               lams, Rs, Ds)
    ws_all = torch.empty(pset.workspace_bytes(), dtype=torch.uint8, device=dev)
    pool = 8
    dpool = [W.decode_pool_device(w, pool, device=dev, layer=l) for l in range(nl)]
    ydec = torch.empty((w.T, nl, w.B, w.Dch), dtype=w.torch_dtype, device=dev)
    ls = ops.LayerSet(lams, Rs, Ds, states)
    stream = torch.cuda.Stream(dev)

    # workspaces of the end-to-end leg's per-layer calls
    pws = [ws, torch.empty_like(ws)]

    def prefill_all():
        ops.prefill_chunked_layers(pset, workspace=ws_all)

    def decode_all():
        for t in range(w.T):
            i = t % pool
            ops.decode_step_layers(ls, [dpool[l][0][i] for l in range(nl)], [dpool[l][1][i] for l in range(nl)],
                                   [dpool[l][2][i] for l in range(nl)], [ydec[t][l] for l in range(nl)])

    with torch.cuda.stream(stream):
        prefill_all()
        decode_all()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        decode_all()
    torch.cuda.synchronize(dev)

    def step(ev):
        if ev is not None:
            ev[0].record(stream)
        prefill_all()
        if ev is not None:
            ev[1].record(stream)
        g.replay()
        if ev is not None:
            ev[2].record(stream)

    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    elapsed_ms, (pre_ms, dec_ms) = timed_steps(stream, dev, steps, warmup, step, 2)
    clk = clocks.stop() if clocks is not None else None
    ms_per_step = elapsed_ms / steps
    err = pset.error(ws_all)
    if err:
        raise SystemExit(f"chunked prefill kernel reported error {err}")

    peak, peak_src = load_peaks()
    key = f"{w.name}/B{w.B}"
    pb, db = algorithmic_bytes(w)
    dec_launch_ms = dec_ms / w.T
    r_pre = roof(f"hyena_prefill_chunked_layers ({nl} layers per launch)", pb * nl, pre_ms, peak, peak_src,
                 ncu_traffic("prefill_chunk_layers", key))
    t_dec = ncu_traffic("decode_layers", key)
    r_dec = roof(f"hyena_decode_step_layers ({nl} layers per launch)", db * nl, dec_launch_ms, peak, peak_src,
                 t_dec, dec_ms)
    rec = {"workload": line_config(w, nl)["workload"], "steps": steps, "warmup": warmup,
           "ms_per_step": ms_per_step,
           "value": world * w.B * (w.L + w.T) / (ms_per_step / 1e3), "unit": "tokens/s",
           "prefill": {"route": "chunked", "tokens_per_s": world * w.B * w.L / (pre_ms / 1e3), "ms": pre_ms,
                       "hbm_frac": r_pre["frac"], "roofline": r_pre,
                       "inputs": "q, k, v of %d MiB per layer (larger than L2), drawn on the device"
                                 % (w.B * w.L * w.Dch * w.act_bytes >> 20)},
           "decode": {"tokens_per_s": world * w.B * w.T / (dec_ms / 1e3), "ms_per_token_step": dec_launch_ms,
                      "hbm_frac": r_dec["frac"], "roofline": r_dec,
                      "state": "%d MiB over %d layers (larger than L2)" % (nl * states[0].numel() * 4 >> 20, nl),
                      "inputs": f"{pool} distinct device-drawn input sets per layer, cycled"},
           "roofline_all": [r_pre, r_dec], "roofline": max([r_pre, r_dec], key=lambda x: x["total_ms"]),
           "launches_per_step": 2 + w.T, "clocks": clk}
    if with_baselines:
        q0, k0, v0 = qkv[0]
        dq0, dk0, dv0 = dpool[0]
        # tokens around the middle of the generation: history of ~L + T/2 tokens per layer
        wl = w.with_(L=w.L + w.T // 2)
        k_hist = torch.cat([k0, dk0.transpose(0, 1).repeat(1, w.T // 2 // pool + 1, 1)[:, :w.T // 2]], 1)
        v_hist = torch.cat([v0, dv0.transpose(0, 1).repeat(1, w.T // 2 // pool + 1, 1)[:, :w.T // 2]], 1)
        rec["baselines"] = fir_baseline(ops, W, wl, None, k_hist.contiguous(), v_hist.contiguous(), dq0, dk0,
                                        dv0, lams[0], Rs[0], Ds[0], stream, dev, 8, dec_launch_ms, pre_ms, peak,
                                        layers=nl)
        del k_hist, v_hist
    del g

    # ---- end to end through the C ABI: every step copies every layer's prompt q, k, v in from pinned
    # host memory and its y out, then every decode token's q, k, v of all layers in and its y out.
    # Prefill: one call per layer (hyena_prefill_chunked) on two device buffer sets, so layer l+1's
    # prompt travels in while layer l computes and layer l-1's y travels out.  Decode: blocks of S tokens, two device blocks; a block's inputs
    # (S tokens x all layers, one copy) travel in while the previous block decodes (CUDA graph per
    # device block), and its outputs travel out after it.
    if with_e2e:
        S = 64
        nblk = (w.T + S - 1) // S
        # host memory (pinned): the prompts of 4 layers, which the 24 layers' copies cycle through (each
        # layer's prompt still crosses PCIe every step; the pool only bounds pinned memory, ~4 GB per
        # GPU in all); one block of S decode tokens' inputs, tiled from the device input pool and copied
        # in for every block; outputs to two prompt-y buffers and two decode-y blocks, alternating
        P = min(4, nl)
        hp = [[make_pinned(t.shape, t.dtype) for t in qkv[l]] for l in range(P)]
        for l in range(P):
            for j in range(3):
                hp[l][j].copy_(qkv[l][j])
        hblk = make_pinned((S, nl, 3, w.B, w.Dch), w.torch_dtype)
        for t in range(S):
            for l in range(nl):
                for j in range(3):
                    hblk[t, l, j].copy_(dpool[l][j][t % pool])
        hy = [make_pinned(qkv[0][0].shape, w.torch_dtype) for _ in range(2)]
        hyd = [make_pinned((S, nl, w.B, w.Dch), w.torch_dtype) for _ in range(2)]
        dset = [[torch.empty_like(qkv[0][0]) for _ in range(4)] for _ in range(2)]     # q, k, v, y
        dblk = [torch.empty((S, nl, 3, w.B, w.Dch), dtype=w.torch_dtype, device=dev) for _ in range(2)]
        dyb = [torch.empty((S, nl, w.B, w.Dch), dtype=w.torch_dtype, device=dev) for _ in range(2)]
        torch.cuda.synchronize(dev)

        def dec_block(j):
            for t in range(S):
                ops.decode_step_layers(ls, [dblk[j][t, l, 0] for l in range(nl)], [dblk[j][t, l, 1] for l in range(nl)],
                                       [dblk[j][t, l, 2] for l in range(nl)], [dyb[j][t, l] for l in range(nl)])
        graphs = []
        for j in range(2):
            with torch.cuda.stream(stream):
                dec_block(j)
            torch.cuda.synchronize(dev)
            gj = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gj, stream=stream):
                dec_block(j)
            graphs.append(gj)
        torch.cuda.synchronize(dev)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        pc, po = [ev(), ev()], [ev(), ev()]       # prompt set j: computed / y copied out
        dc, do = [ev(), ev()], [ev(), ev()]       # decode block j: decoded / y copied out
        for e in pc + po + dc + do:
            e.record(stream)
        bi = nl * 3 * qkv[0][0].numel() * w.act_bytes + nblk * S * nl * 3 * w.B * w.Dch * w.act_bytes
        bo = nl * qkv[0][0].numel() * w.act_bytes + nblk * S * nl * w.B * w.Dch * w.act_bytes

        def e2e_step():
            for l in range(nl):
                j = l % 2
                s_in.wait_event(pc[j])
                with torch.cuda.stream(s_in):
                    for x in range(3):
                        dset[j][x].copy_(hp[l % P][x], non_blocking=True)
                got = ev()
                got.record(s_in)
                stream.wait_event(got)
                stream.wait_event(po[j])
                with torch.cuda.stream(stream):
                    ops.prefill_chunked(dset[j][0], dset[j][1], dset[j][2], lams[l], Rs[l], Ds[l], y=dset[j][3],
                                        state=states[l], workspace=pws[j])
                pc[j].record(stream)
                s_out.wait_event(pc[j])
                with torch.cuda.stream(s_out):
                    hy[j].copy_(dset[j][3], non_blocking=True)
                po[j].record(s_out)
            for bk in range(nblk):
                j = bk % 2
                s_in.wait_event(dc[j])
                with torch.cuda.stream(s_in):
                    dblk[j].copy_(hblk, non_blocking=True)
                got = ev()
                got.record(s_in)
                stream.wait_event(got)
                stream.wait_event(do[j])
                with torch.cuda.stream(stream):
                    graphs[j].replay()
                dc[j].record(stream)
                s_out.wait_event(dc[j])
                with torch.cuda.stream(s_out):
                    hyd[j].copy_(dyb[j], non_blocking=True)
                do[j].record(s_out)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize(dev)
        s_in.wait_stream(torch.cuda.current_stream(dev))
        a.record(s_in)
        for _ in range(e2e_steps):
            e2e_step()
        s_out.wait_stream(stream)
        s_out.wait_stream(s_in)
        b.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = reduce_max(a.elapsed_time(b), dev) / e2e_steps
        for wsx in pws:
            err = ops.chunked_error(wsx, w.B, w.L, w.Dch, w.H, w.d)
            if err:
                raise SystemExit(f"chunked prefill kernel reported error {err} (end-to-end run)")
        rec["e2e"] = {"value": world * w.B * (w.L + w.T) / (e2e_ms / 1e3), "unit": "tokens/s",
                      "ms_per_step": e2e_ms, "steps": e2e_steps, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                      "overlap": (f"prompt: two device buffer sets, layer l+1 copied in while layer l computes; "
                                  f"decode: blocks of {S} tokens x {nl} layers, two device blocks; copy-in, compute "
                                  f"and copy-out streams"),
                      "host_buffers": (f"pinned prompts of {P} layers, cycled over the {nl} layers' copies; one "
                                       f"pinned block of {S} tokens' decode inputs, copied in for each of the "
                                       f"{nblk} blocks; outputs to two alternating pinned buffers")}
        del graphs
    return rec


# ------------------------------------------------------------------ our arm
SUBRECORDS = [
    # (name, workload, batch override, steps, e2e, fft route, baselines)
    ("tiny_f32", "tiny_f32", 0, None, True, False, False),
    ("mid_bf16", "mid_bf16", 0, None, True, True, True),
    ("long_prefill_bf16", "long_prefill_bf16", 0, None, True, True, False),
    ("decode_sweep_bf16/B1", "decode_sweep_bf16", 1, 5, False, False, False),
    ("decode_sweep_bf16/B16", "decode_sweep_bf16", 16, 5, False, False, False),
    ("decode_sweep_bf16/B64", "decode_sweep_bf16", 64, 5, False, False, False),
    ("decode_sweep_bf16/B256", "decode_sweep_bf16", 256, 5, False, False, False),
    ("decode_sweep_bf16/B1024", "decode_sweep_bf16", 1024, 5, False, False, False),
]


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
    if args.batch:
        w = w.with_(B=args.batch)
    nl = args.layers or w.layers
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    clocks = ClockSampler(gpu_id_for(dev))
    if nl > 1:
        head = measure_layers(args, w, nl, dev, args.steps, args.warmup, e2e_steps, not args.no_baselines,
                              not args.no_e2e, clocks)
        clk = head.pop("clocks")
    else:
        clocks.start()
        time.sleep(0.3)
        head = measure_single(args, w, dev, args.steps, args.warmup, e2e_steps, not args.no_fft_route,
                              not args.no_baselines, not args.no_e2e)
        clk = clocks.stop()
    torch.cuda.synchronize(dev)

    # sub-records: the other workloads, each timed on its own (1 GPU only)
    subs = None
    if world == 1 and not args.no_subrecords and args.workload == DEFAULT_WORKLOAD and not args.batch:
        subs = {}
        for name, wl, batch, steps, e2e, fft, base in SUBRECORDS:
            ws = W.WORKLOADS[wl]
            if batch:
                ws = ws.with_(B=batch)
            st = steps or args.steps
            subs[name] = measure_single(args, ws, dev, st, args.warmup, e2e_steps, fft and not args.no_fft_route,
                                        base and not args.no_baselines, e2e and not args.no_e2e)
            torch.cuda.empty_cache()

    cpu = None
    if world == 1 and not args.no_cpu_baseline and w.L > 0:
        cpu, _, _, _ = oracle_baseline(w, nl, 12.0)

    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded; drawn on the device for the multi-layer workload)" if nl > 1 else "synthetic (seeded)",
                "config": line_config(w, nl),
                "value_definition": "(prompt + generated) tokens per second through every layer: "
                                    "B x (L + T) tokens per step / step time, summed over GPUs",
                "prefill": head.get("prefill"), "decode": head.get("decode"),
                "roofline": head["roofline"], "roofline_all": head["roofline_all"],
                "cpu_baseline": cpu, "e2e": head.get("e2e"),
                "gpu_launches": args.steps * head["launches_per_step"], "clocks": clk}
        for k in ("prefill_fft_route", "baselines"):
            if k in head:
                line[k] = head[k]
        if subs is not None:
            line["subrecords"] = subs
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_truncation(args):
    """Filter error of modal truncation against the number of kept modes, per workload: the l2
    norm of the tap error relative to the full filter's (taps j >= 1) and the l1 bound relative to
    its value with every mode dropped (GPU kernel through the C ABI)."""
    import torch
    from distilled_ssm_decode_b200 import build, ops
    from distilled_ssm_decode_b200 import workloads as W
    build.build()
    out = {"metric": "modal truncation: relative filter error vs kept modes", "workloads": {}}
    for name in ("mid_bf16", "gen1p3b_bf16", "long_prefill_bf16"):
        w = W.WORKLOADS[name]
        p = W.params(w)
        lam, R = p.lam_f32().cuda(), p.R_f32().cuda()
        _, _, _, b0, e0 = ops.modal_truncate(lam, R, 0)
        rows = []
        for k in range(1, w.d + 1):
            _, _, _, b, e = ops.modal_truncate(lam, R, k)
            rel = (e / e0).cpu().numpy()
            rb = (b / b0).cpu().numpy()
            rows.append({"k": k, "l2_rel_mean": float(rel.mean()), "l2_rel_max": float(rel.max()),
                         "l1_bound_rel_max": float(rb.max())})
        out["workloads"][name] = {"H": w.H, "d": w.d, "poles": f"|lambda| ~ U[{w.rmin}, {w.rmax}]",
                                  "rows": rows}
    print(json.dumps(out), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size")
    ap.add_argument("--prefill", choices=["auto", "chunked", "fft"], default="auto",
                    help="prefill route: chunked tensor-core evaluation (auto when supported) or FFT")
    ap.add_argument("--fft-cuda-cores", action="store_true",
                    help="run the FFT route's transforms on the CUDA cores also where the tensor-core "
                         "route applies (bf16 at FFT lengths 4096..16384); for comparisons")
    ap.add_argument("--no-fft-route", action="store_true",
                    help="skip the extra timing of the FFT route when the chunked route is used")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5, help="timed end-to-end steps (at most --steps)")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="only the headline workload (the default run adds the other workloads' records)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip the undistilled (FIR / re-prefill) decode baselines")
    ap.add_argument("--truncation", action="store_true",
                    help="print the modal-truncation error table instead of benchmarking")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers of a multi-layer workload to run (default: all; 1 = one layer)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.truncation:
        return run_truncation(args)
    if args.fft_cuda_cores:
        from distilled_ssm_decode_b200 import ops
        ops.lib().hyena_test_fft_tensor_cores(0)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
