"""GPU parity of the chunked tensor-core prefill (tcgen05) against the fp64 oracle.

The chunked route regroups the causal convolution into 64-token chunks with the
recurrent state carried between them; its outputs must match the oracle's
direct convolution and prompt state within the bf16 tolerance (2e-2 of
max|oracle|).  Shapes cover ragged prompts, prompts shorter than one chunk,
several 128-channel tiles and heads, d from 1 to 16, and sequences split into
many segments (which exercises the cross-segment state look-back).  Every run
also checks the kernel's error word (0 = no bounded wait gave up).
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, column_params, dev_params, gather_columns, rel_err, sample_columns, state_c128

pytestmark = pytest.mark.gpu

# The chunked route rounds its tensor-core operands to bf16 (u = k v, the taps, the powers and the
# carried state; relative 2^-9 each) and accumulates in fp32.  Measured on B200 over every case
# below and the full-size workloads: max|y - oracle| / max|oracle| from 2.8e-3 to 6.5e-3 (the FFT
# route on the same inputs: 1.3e-3 to 3.3e-3, its bf16 output rounding), and the prompt state from
# 1.6e-3 to 3.9e-3 (FFT route ~1e-7).  Besides the bf16 bar (2e-2) every case must stay within
# these measured margins, so a change that loses accuracy shows even while the bar still holds.
Y_MARGIN = 1e-2
S_MARGIN = 6e-3


def _check_errors(record_property, ey, es):
    record_property("chunked_y_err", float(ey))
    record_property("chunked_state_err", float(es))
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)
    assert ey <= Y_MARGIN and es <= S_MARGIN, (ey, es)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _run(q, k, v, p):
    lam, R, D = dev_params(p)
    y, s, ws = ops.prefill_chunked(q.cuda(), k.cuda(), v.cuda(), lam, R, D)
    B, L, Dch = q.shape
    err = ops.chunked_error(ws, B, L, Dch, lam.shape[0], lam.shape[1])
    assert err == 0, f"kernel error word {err}"
    return y.cpu(), state_c128(s)


CASES = [
    # B, L, Dch, H, d
    (1, 64, 128, 1, 16),      # one full chunk
    (1, 1, 128, 1, 16),       # single token
    (2, 63, 256, 2, 8),       # shorter than a chunk, two heads
    (2, 65, 256, 1, 16),      # one chunk + 1 token; a head spans two channel tiles
    (3, 300, 128, 1, 4),      # ragged, d = 4
    (1, 1000, 384, 3, 1),     # d = 1
    (1, 4096, 128, 1, 16),    # one tile: the sequence is split into many segments (look-back)
    (2, 2048, 256, 2, 12),    # d not a multiple of 8
    (2, 300, 128, 2, 16),     # 64-channel heads (64-channel tiles), ragged
    (1, 4096, 128, 2, 16),    # 64-channel tiles, sequences split into segments (look-back)
    (3, 1000, 192, 3, 5),     # 64-channel heads, three of them
    # state-only passes of 2, 3, 7 and 10 chunks before the look-back: the two product issuers
    # take alternate chunks of these passes (an even count, an odd count, both with a single
    # chunk left over at the end)
    (1, 8192, 128, 2, 16),
    (1, 12000, 128, 2, 16),
    (1, 20000, 192, 3, 16),
    (3, 5000, 384, 6, 8),
]


@pytest.mark.parametrize("B,L,Dch,H,d", CASES)
def test_chunked_small_cases_full_compare(oracle, record_property, B, L, Dch, H, d):
    w = W.Workload(300 + L + d, "case", B=B, L=L, Dch=Dch, H=H, d=d, dtype="bf16", fft_len=0, T=0)
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    y, s = _run(q, k, v, p)
    qf, kf, vf = W.to_f64(q), W.to_f64(k), W.to_f64(v)
    if L <= 1024:
        h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, L)
        y_ref = oracle.conv_direct(qf, kf, vf, h, H=H)
        s_ref = oracle.prompt_state(kf, vf, p.lam, H=H)
    else:
        y_ref, s_ref = oracle.recurrent(qf, kf, vf, p.lam, p.R, p.Dskip, H=H)
    ey, es = rel_err(y.double().numpy(), y_ref), rel_err(s, s_ref)
    _check_errors(record_property, ey, es)


@pytest.mark.parametrize("name,ncols", [("mid_bf16", 24), ("gen1p3b_bf16", 32)])
def test_chunked_full_size_sampled(oracle, record_property, name, ncols):
    w = W.WORKLOADS[name]
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    y, s = _run(q, k, v, p)
    rng = np.random.default_rng(7)
    bc = sample_columns(rng, w.B, w.Dch, ncols)
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, [c for _, c in bc])
    qc, kc, vc = gather_columns(q, bc), gather_columns(k, bc), gather_columns(v, bc)
    h = oracle.filter_from_modes(lam_c, R_c, D_c, w.L)
    y_ref = oracle.conv_direct(qc, kc, vc, h, H=len(bc))
    s_ref = oracle.prompt_state(kc, vc, lam_c, H=len(bc))
    ey = rel_err(gather_columns(y, bc), y_ref)
    es = rel_err(np.stack([s[b, :, c] for b, c in bc], -1)[None], s_ref)
    _check_errors(record_property, ey, es)


def test_chunked_matches_fft_route():
    """Both prefill routes compute the same operator: outputs agree within the bf16 bar."""
    w = W.WORKLOADS["mid_bf16"]
    p = W.params(w)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, B=2, L=2048, Dch=256))
    lam, R, D = dev_params(p.__class__(p.lam[:2], p.R[:2], p.Dskip[:2]))
    y1, s1, _ = ops.prefill_chunked(q, k, v, lam, R, D)
    with ops.fft_tensor_cores(False):
        y2, s2 = ops.prefill(q, k, v, lam, R, D, 4096)
    # the CUDA-core FFT route is fp32 throughout (state ~1e-7 of the oracle), so this measures the
    # chunked route's own error (bf16 operands): within the bf16 bar and the measured margins
    assert rel_err(y1.cpu().double().numpy(), y2.cpu().double().numpy()) <= Y_MARGIN
    assert rel_err(state_c128(s1), state_c128(s2)) <= S_MARGIN


def test_chunked_is_deterministic():
    w = W.WORKLOADS["gen1p3b_bf16"]
    p = W.params(w)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, B=4, L=512, Dch=256))
    lam, R, D = dev_params(p.__class__(p.lam[:2], p.R[:2], p.Dskip[:2]))
    y1, s1, _ = ops.prefill_chunked(q, k, v, lam, R, D)
    y2, s2, _ = ops.prefill_chunked(q, k, v, lam, R, D)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_chunked_unsupported_shapes_are_rejected():
    lam = torch.zeros(2, 4, 2, device="cuda")
    D = torch.zeros(2, device="cuda")
    x32 = torch.zeros(1, 64, 256, device="cuda")
    with pytest.raises(ops.HyenaError) as e:
        ops.prefill_chunked(x32, x32, x32, lam, lam, D)          # fp32 activations
    assert e.value.status == -5
    x = torch.zeros(1, 64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.HyenaError) as e:
        ops.prefill_chunked(x, x, x, lam, lam, D)                # 32 channels per head
    assert e.value.status == -5


def test_chunked_long_prefill_full_size_sampled(oracle, record_property):
    """The long-prefill workload as the bench runs it (B=1, L=65536, Dch=768, 12 heads of 64
    channels, |lambda| up to 0.999, sequences split into segments joined by the look-back):
    24 sampled channels against the oracle's recurrence over the whole prompt."""
    w = W.WORKLOADS["long_prefill_bf16"]
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    y, s = _run(q, k, v, p)
    rng = np.random.default_rng(11)
    bc = sample_columns(rng, w.B, w.Dch, 24)
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, [c for _, c in bc])
    qc, kc, vc = gather_columns(q, bc), gather_columns(k, bc), gather_columns(v, bc)
    y_ref, s_ref = oracle.recurrent(qc, kc, vc, lam_c, R_c, D_c, H=len(bc))
    ey = rel_err(gather_columns(y, bc), y_ref)
    es = rel_err(np.stack([s[b, :, c] for b, c in bc], -1)[None], s_ref)
    _check_errors(record_property, ey, es)


def test_chunked_is_deterministic_with_many_items():
    """1024 items on the persistent grid (the 1.3B-shaped layer): each CTA's first item has a fixed
    ticket, the rest are handed out by counters, so which CTA takes which item (and switches heads
    when) varies from run to run; the outputs must not: repeated runs are bitwise identical."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    p = W.params(w)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, B=64, L=512))
    lam, R, D = dev_params(p)
    y1, s1, ws = ops.prefill_chunked(q, k, v, lam, R, D)
    for _ in range(3):
        y2, s2, _ = ops.prefill_chunked(q, k, v, lam, R, D, workspace=ws)
        assert torch.equal(y1, y2) and torch.equal(s1, s2)
    assert ops.chunked_error(ws, w.B, w.L, w.Dch, w.H, w.d) == 0


@pytest.mark.parametrize("B,L,Dch,H", [(1, 65536, 768, 12), (1, 20000, 192, 3)])
def test_chunked_is_deterministic_with_segments(B, L, Dch, H):
    """Sequences split into segments (the long-prefill shape: 12 segments of 86 chunks; and 45
    segments of 7): which predecessor a look-back finds with an inclusive state, and when the two
    product issuers finish their shares of a state-only pass, vary from run to run; the outputs
    must not: repeated runs are bitwise identical."""
    w = W.Workload(400 + H, "segments", B=B, L=L, Dch=Dch, H=H, d=16, dtype="bf16", fft_len=0, T=0)
    p = W.params(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    q, k, v = (torch.randn((B, L, Dch), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    lam, R, D = dev_params(p)
    y1, s1, ws = ops.prefill_chunked(q, k, v, lam, R, D)
    for _ in range(3):
        y2, s2, _ = ops.prefill_chunked(q, k, v, lam, R, D, workspace=ws)
        assert torch.equal(y1, y2) and torch.equal(s1, s2)
    assert ops.chunked_error(ws, B, L, Dch, H, 16) == 0


def test_chunked_empty_inputs():
    lam = torch.zeros(2, 4, 2, device="cuda")
    D = torch.zeros(2, device="cuda")
    # empty prompt: the state is zero
    x = torch.empty(2, 0, 128, dtype=torch.bfloat16, device="cuda")
    s = torch.full((2, 4, 128, 2), 7.0, device="cuda")
    ops.prefill_chunked(x, x, x, lam, lam, D, state=s)
    assert torch.all(s == 0)
    # no sequences: nothing to do
    x = torch.empty(0, 64, 128, dtype=torch.bfloat16, device="cuda")
    ops.prefill_chunked(x, x, x, lam, lam, D, state=torch.empty(0, 4, 128, 2, device="cuda"))
    torch.cuda.synchronize()


def test_chunked_degenerate_poles(oracle, record_property):
    """Poles at 0 (lambda^0 = 1 only: a two-tap filter, no carry beyond one token) and poles at
    |lambda| = 0.9999 (almost no decay over the 3000-token prompt, sequence split into segments)
    mixed in one head; every element against the oracle's recurrence."""
    w = W.Workload(777, "case", B=1, L=3000, Dch=128, H=1, d=6, dtype="bf16", fft_len=0, T=0)
    p = W.params(w)
    lam = p.lam.copy()
    lam[0, 0] = 0.0
    lam[0, 1] = 0.0
    lam[0, 2] = np.complex64(0.9999 * np.exp(0.3j))
    lam[0, 3] = np.complex64(-0.9999)
    p = W.Params(lam.astype(np.complex64).astype(np.complex128), p.R, p.Dskip)
    q, k, v = W.prefill_inputs(w)
    y, s = _run(q, k, v, p)
    y_ref, s_ref = oracle.recurrent(W.to_f64(q), W.to_f64(k), W.to_f64(v), p.lam, p.R, p.Dskip, H=1)
    ey, es = rel_err(y.double().numpy(), y_ref), rel_err(s, s_ref)
    _check_errors(record_property, ey, es)


def test_mid_workload_flow_chunked_then_decode(oracle):
    """The default benchmark's flow at full size (B=8, L=4096, Dch=1024, H=8, d=16): chunked
    prefill, then 8 decode steps from its state; 24 sampled channels against the oracle's
    recurrence over prompt + generated tokens."""
    w = W.WORKLOADS["mid_bf16"]
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    _, s, ws = ops.prefill_chunked(q.cuda(), k.cuda(), v.cuda(), lam, R, D)
    T = 8
    bc = sample_columns(np.random.default_rng(5), w.B, w.Dch, 24)
    ib = torch.tensor([b for b, _ in bc]); ic = torch.tensor([c for _, c in bc])
    ys, qs, ks, vs = [], [], [], []
    for t in range(T):
        a, b, c = W.decode_inputs(w, t)
        ys.append(ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu()[ib, ic])
        qs.append(a[ib, ic]); ks.append(b[ib, ic]); vs.append(c[ib, ic])
    assert ops.chunked_error(ws, w.B, w.L, w.Dch, w.H, w.d) == 0
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, [c for _, c in bc])
    qa = np.concatenate([gather_columns(q, bc), W.to_f64(torch.stack(qs))[None]], 1)
    ka = np.concatenate([gather_columns(k, bc), W.to_f64(torch.stack(ks))[None]], 1)
    va = np.concatenate([gather_columns(v, bc), W.to_f64(torch.stack(vs))[None]], 1)
    y_ref, s_ref = oracle.recurrent(qa, ka, va, lam_c, R_c, D_c, H=len(bc))
    assert rel_err(torch.stack(ys).double().numpy()[None], y_ref[:, w.L:]) <= TOL["bf16"]


ERR_LOOKBACK = 2


def test_chunked_lookback_timeout_reports_error_and_recovers(oracle):
    """Failure detection without a GPU fault: the test hook stops one segment's completion word from
    ever being posted and bounds the wait for it to 5 ms.  The call must return with error word 2
    (a look-back gave up) instead of hanging, and the next normal call on the same stream and
    workspace must pass parity."""
    w = W.Workload(301, "lookback", B=1, L=4096, Dch=128, H=1, d=16, dtype="bf16", fft_len=0, T=0)
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ops.test_chunked_inject(0, 0.005)          # item 0: segment 0 of the first sequence
    try:
        _, _, ws = ops.prefill_chunked(qd, kd, vd, lam, R, D)
        torch.cuda.synchronize()
    finally:
        ops.test_chunked_inject(-1, 0.0)
    assert ops.chunked_error(ws, w.B, w.L, w.Dch, w.H, w.d) == ERR_LOOKBACK
    y, s, _ = ops.prefill_chunked(qd, kd, vd, lam, R, D, workspace=ws)
    assert ops.chunked_error(ws, w.B, w.L, w.Dch, w.H, w.d) == 0
    y_ref, s_ref = oracle.recurrent(W.to_f64(q), W.to_f64(k), W.to_f64(v), p.lam, p.R, p.Dskip, H=w.H)
    ey, es = rel_err(y.cpu().double().numpy(), y_ref), rel_err(state_c128(s), s_ref)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)


def _hold_sms_lib():
    """Build (once) and load the test helper that occupies SMs for a bounded time."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = os.path.join(root, "tests", "gpu_aux", "hold_sms.cu")
    out = os.path.join(root, "_build", "libhyena_test_hold_sms.so")
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(out), exist_ok=True)
        nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler",
                        "-fPIC", "-o", out, src], check=True, capture_output=True)
    lib = ctypes.CDLL(out)
    lib.hold_sms.argtypes = [ctypes.c_int, ctypes.c_ulonglong, ctypes.c_int, ctypes.c_void_p]
    lib.sm_count.argtypes = []
    return lib


@pytest.mark.parametrize("B,L,Dch,H", [(1, 20000, 192, 3), (1, 65536, 768, 12)])
def test_chunked_segments_progress_with_most_sms_busy(B, L, Dch, H):
    """Sequences split into segments, launched while a kernel on another stream holds all but 12 SMs
    for 20 ms: the items that wait for earlier segments must only ever wait on work that is running,
    so the call completes with error word 0 and the same bits as an uncontended run."""
    aux = _hold_sms_lib()
    w = W.Workload(500 + H, "busy", B=B, L=L, Dch=Dch, H=H, d=16, dtype="bf16", fft_len=0, T=0)
    p = W.params(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(13)
    q, k, v = (torch.randn((B, L, Dch), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    lam, R, D = dev_params(p)
    y1, s1, ws = ops.prefill_chunked(q, k, v, lam, R, D)
    torch.cuda.synchronize()
    nsm = aux.sm_count()
    assert nsm > 12
    busy, work = torch.cuda.Stream(), torch.cuda.Stream()
    y2, s2 = torch.empty_like(y1), torch.empty_like(s1)
    ws2 = torch.empty_like(ws)
    assert aux.hold_sms(nsm - 12, 20_000_000, 160 * 1024, ctypes.c_void_p(busy.cuda_stream)) == 0
    with torch.cuda.stream(work):
        ops.prefill_chunked(q, k, v, lam, R, D, y=y2, state=s2, workspace=ws2)
    torch.cuda.synchronize()
    assert ops.chunked_error(ws2, B, L, Dch, H, 16) == 0
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


@pytest.mark.parametrize("nl,B,L,Dch,hd_ch,d", [(3, 2, 300, 256, 128, 16), (2, 1, 4096, 128, 64, 16),
                                                  (5, 1, 65, 192, 64, 5)])
def test_chunked_layers_match_oracle(oracle, record_property, nl, B, L, Dch, hd_ch, d):
    """Several independent layers in one launch (their work items share the persistent grid; with one
    sequence and 64-channel heads the sequences are split into segments): every layer's y and
    state against the oracle."""
    H = Dch // hd_ch
    w = W.Workload(700 + L + d, "layers", B=B, L=L, Dch=Dch, H=H, d=d, dtype="bf16", fft_len=0, T=0)
    ps = [W.params(w, layer=l) for l in range(nl)]
    qkv = [W.prefill_inputs(w, layer=l) for l in range(nl)]
    dev = [dev_params(p) for p in ps]
    qs, ks, vs = ([x[j].cuda() for x in qkv] for j in range(3))
    ys = [torch.empty_like(q) for q in qs]
    sts = [torch.empty((B, d, Dch, 2), device="cuda") for _ in range(nl)]
    ls = ops.PrefillLayerSet(qs, ks, vs, ys, sts, [x[0] for x in dev], [x[1] for x in dev], [x[2] for x in dev])
    ws = ops.prefill_chunked_layers(ls)
    assert ls.error(ws) == 0
    for l in range(nl):
        qf, kf, vf = (W.to_f64(t) for t in qkv[l])
        y_ref, s_ref = oracle.recurrent(qf, kf, vf, ps[l].lam, ps[l].R, ps[l].Dskip, H=H)
        ey, es = rel_err(ys[l].cpu().double().numpy(), y_ref), rel_err(state_c128(sts[l]), s_ref)
        _check_errors(record_property, ey, es)


def test_chunked_layers_equal_single_layer_calls_1p3b():
    """The 24 layers of the 1.3B-shaped workload in one launch give the same bits as 24 single-layer
    calls (the same plan: 128-channel tiles, sequences not split)."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    nl = w.layers
    ps = [W.params(w, layer=l) for l in range(nl)]
    dev = [dev_params(p) for p in ps]
    qkv = [W.prefill_inputs_device(w, l) for l in range(nl)]
    ys = [torch.empty_like(x[0]) for x in qkv]
    sts = [torch.empty((w.B, w.d, w.Dch, 2), device="cuda") for _ in range(nl)]
    ls = ops.PrefillLayerSet([x[0] for x in qkv], [x[1] for x in qkv], [x[2] for x in qkv], ys, sts,
                             [x[0] for x in dev], [x[1] for x in dev], [x[2] for x in dev])
    ws = ops.prefill_chunked_layers(ls)
    assert ls.error(ws) == 0
    for l in range(nl):
        y1, s1, ws1 = ops.prefill_chunked(*qkv[l], *dev[l])
        assert ops.chunked_error(ws1, w.B, w.L, w.Dch, w.H, w.d) == 0
        assert torch.equal(y1, ys[l]) and torch.equal(s1, sts[l]), l


def test_chunked_layers_lookback_timeout_and_empty_prompt():
    """The grouped launch shares the single-layer error path: with one item's completion word
    suppressed (test hook, 5 ms bound) a split-sequence launch of two layers ends with error word 2,
    and the next normal call passes; an empty prompt writes zero states for every layer."""
    nl, B, L, Dch, H, d = 2, 1, 4096, 64, 1, 8
    w = W.Workload(711, "layers", B=B, L=L, Dch=Dch, H=H, d=d, dtype="bf16", fft_len=0, T=0)
    ps = [W.params(w, layer=l) for l in range(nl)]
    dev = [dev_params(p) for p in ps]
    g = torch.Generator(device="cuda")
    g.manual_seed(21)
    qs, ks, vs = ([torch.randn((B, L, Dch), generator=g, device="cuda").to(torch.bfloat16) for _ in range(nl)]
                  for _ in range(3))
    ys = [torch.empty_like(q) for q in qs]
    sts = [torch.empty((B, d, Dch, 2), device="cuda") for _ in range(nl)]
    ls = ops.PrefillLayerSet(qs, ks, vs, ys, sts, [x[0] for x in dev], [x[1] for x in dev], [x[2] for x in dev])
    ops.test_chunked_inject(0, 0.005)
    try:
        ws = ops.prefill_chunked_layers(ls)
        torch.cuda.synchronize()
    finally:
        ops.test_chunked_inject(-1, 0.0)
    assert ls.error(ws) == ERR_LOOKBACK
    ops.prefill_chunked_layers(ls, workspace=ws)
    assert ls.error(ws) == 0
    for l in range(nl):
        y1, s1, _ = ops.prefill_chunked(qs[l], ks[l], vs[l], *dev[l])
        assert rel_err(ys[l].cpu().double().numpy(), y1.cpu().double().numpy()) <= Y_MARGIN
    empty = [torch.empty((B, 0, Dch), dtype=torch.bfloat16, device="cuda") for _ in range(nl)]
    sts0 = [torch.full((B, d, Dch, 2), 7.0, device="cuda") for _ in range(nl)]
    ls0 = ops.PrefillLayerSet(empty, empty, empty, empty, sts0, [x[0] for x in dev], [x[1] for x in dev],
                              [x[2] for x in dev])
    ops.prefill_chunked_layers(ls0)
    torch.cuda.synchronize()
    assert all(torch.all(st == 0) for st in sts0)
