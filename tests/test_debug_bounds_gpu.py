"""Bounds-checked tier: tiny shapes through the bounds-checked build of the library.

libhyena_b200_dbg.so is the library compiled with -DHYENA_DEBUG_BOUNDS: every kernel checks the
index of each global load and store against the extent its arguments give that buffer, records
the first one out of range and skips it (no trap, no fault).  This tier runs every entry point on
the smallest and most ragged shapes (L in {1, 2, 3, 17}, d in {1, 2}, one or two sequences, odd
channel counts where the entry point takes them), checks that no access was out of range, and
checks the results against the fp64 oracle as the release tests do.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, dev_params, rel_err, state_c128

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()
    path = build.build(debug_bounds=True)
    with ops.using_library(path):
        st, _ = ops.bounds_check()
        assert st == 0            # a bounds-checked build, with no record yet
        yield


def _clean():
    torch.cuda.synchronize()
    st, rec = ops.bounds_check()
    assert st == 0, f"out-of-range access recorded: file {rec[0]}, line {rec[1]}, index {rec[2]}, extent {rec[3]}"


def _case(B, L, Dch, H, d, dtype, seed):
    w = W.Workload(600 + seed, "tiny", B=B, L=L, Dch=Dch, H=H, d=d, dtype=dtype, fft_len=0, T=0)
    return w, W.params(w)


SHAPES = [(B, L, Dch, H, d) for (B, Dch, H) in ((1, 2, 1), (2, 6, 3), (1, 5, 5), (2, 8, 2))
          for L in (1, 2, 3, 17) for d in (1, 2)]


@pytest.mark.parametrize("B,L,Dch,H,d", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fft_prefill_then_decode_in_bounds(dbg, oracle, B, L, Dch, H, d, dtype):
    w, p = _case(B, L, Dch, H, d, dtype, L * 7 + d)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    N = max(64, 1 << (2 * L - 1).bit_length())
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, N)
    T = 3
    steps = [W.decode_inputs(w, t) for t in range(T)]
    yd = [ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s) for a, b, c in steps]
    _clean()
    qa = np.concatenate([W.to_f64(q), W.to_f64(torch.stack([a for a, _, _ in steps], 1))], 1)
    ka = np.concatenate([W.to_f64(k), W.to_f64(torch.stack([b for _, b, _ in steps], 1))], 1)
    va = np.concatenate([W.to_f64(v), W.to_f64(torch.stack([c for _, _, c in steps], 1))], 1)
    h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, L + T)
    y_ref = oracle.conv_direct(qa, ka, va, h, H=H)
    got = np.concatenate([y.cpu().double().numpy(), torch.stack([t.cpu() for t in yd], 1).double().numpy()], 1)
    assert rel_err(got, y_ref) <= TOL[dtype]


@pytest.mark.parametrize("L", [1, 2, 3, 17])
@pytest.mark.parametrize("d", [1, 2])
def test_chunked_prefill_in_bounds(dbg, oracle, L, d):
    B, Dch, H = 2, 128, 2
    w, p = _case(B, L, Dch, H, d, "bf16", 50 + L * 3 + d)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    y, s, ws = ops.prefill_chunked(q.cuda(), k.cuda(), v.cuda(), lam, R, D)
    _clean()
    assert ops.chunked_error(ws, B, L, Dch, H, d) == 0
    qf, kf, vf = W.to_f64(q), W.to_f64(k), W.to_f64(v)
    y_ref = oracle.conv_direct(qf, kf, vf, oracle.filter_from_modes(p.lam, p.R, p.Dskip, L), H=H)
    s_ref = oracle.prompt_state(kf, vf, p.lam, H=H)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["bf16"]
    assert rel_err(state_c128(s), s_ref) <= TOL["bf16"]


def test_chunked_prefill_segments_in_bounds(dbg, oracle):
    """A sequence split into segments (look-back, published states) in the bounds-checked build."""
    B, L, Dch, H, d = 1, 3000, 128, 1, 2
    w, p = _case(B, L, Dch, H, d, "bf16", 99)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    y, s, ws = ops.prefill_chunked(q.cuda(), k.cuda(), v.cuda(), lam, R, D)
    _clean()
    assert ops.chunked_error(ws, B, L, Dch, H, d) == 0
    y_ref, s_ref = oracle.recurrent(W.to_f64(q), W.to_f64(k), W.to_f64(v), p.lam, p.R, p.Dskip, H=H)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["bf16"]
    assert rel_err(state_c128(s), s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("L", [1, 17])
def test_long_fft_route_and_state_in_bounds(dbg, oracle, L):
    """The four-step FFT route (transform longer than 16384 points) and the standalone prompt
    state on a tiny prompt."""
    B, Dch, H, d = 1, 4, 2, 2
    w, p = _case(B, L, Dch, H, d, "f32", 70 + L)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, 32768)
    s2 = ops.prompt_state(k.cuda(), v.cuda(), lam, H)
    _clean()
    qf, kf, vf = W.to_f64(q), W.to_f64(k), W.to_f64(v)
    y_ref = oracle.conv_direct(qf, kf, vf, oracle.filter_from_modes(p.lam, p.R, p.Dskip, L), H=H)
    s_ref = oracle.prompt_state(kf, vf, p.lam, H=H)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["f32"]
    assert rel_err(state_c128(s), s_ref) <= TOL["f32"]
    assert rel_err(state_c128(s2), s_ref) <= TOL["f32"]


@pytest.mark.parametrize("t", [0, 1, 16])
def test_fir_filter_spectrum_truncate_in_bounds(dbg, oracle, t):
    B, L, Dch, H, d = 2, 17, 6, 3, 2
    w, p = _case(B, L, Dch, H, d, "f32", 80 + t)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    t_max = t + 1
    h = ops.filter_from_modes(lam, R, D, t_max)
    spec = ops.filter_spectrum(h, 64)
    u = ops.fir_cache_prompt(k[:, :t].contiguous().cuda(), v[:, :t].contiguous().cuda(), t_max)
    y = ops.fir_decode_step(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(), v[:, t].contiguous().cuda(),
                            h, u, t)
    kept, lo, ro, bound, err = ops.modal_truncate(lam, R, 1)
    _clean()
    h_ref = oracle.filter_from_modes(p.lam, p.R, p.Dskip, t_max)
    assert rel_err(h.cpu().double().numpy(), h_ref) <= 1e-6
    y_ref = oracle.conv_direct(W.to_f64(q[:, :t + 1]), W.to_f64(k[:, :t + 1]), W.to_f64(v[:, :t + 1]), h_ref, H=H)
    assert rel_err(y.cpu().double().numpy(), y_ref[:, t]) <= TOL["f32"]
    assert spec.shape[-1] == 33 and kept.shape == (H, 1) and bound.shape == (H,) and err.shape == (H,)


def test_decode_layers_in_bounds(dbg):
    """The grouped decode over 3 layers, against the one-layer decode (in the same build)."""
    B, Dch, H, d = 2, 6, 3, 2
    ws = [_case(B, 1, Dch, H, d, "bf16", 90 + l) for l in range(3)]
    pars = [dev_params(p) for _, p in ws]
    g = torch.Generator().manual_seed(5)
    st = [torch.randn((B, d, Dch, 2), generator=g).cuda() for _ in range(3)]
    xs = [[torch.randn((B, Dch), generator=g).to(torch.bfloat16).cuda() for _ in range(3)] for _ in range(3)]
    ref_st = [s.clone() for s in st]
    ref = [ops.decode_step(x[0], x[1], x[2], *par, s) for x, par, s in zip(xs, pars, ref_st)]
    ls = ops.LayerSet([p[0] for p in pars], [p[1] for p in pars], [p[2] for p in pars], st)
    ys = [torch.empty((B, Dch), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ops.decode_step_layers(ls, [x[0] for x in xs], [x[1] for x in xs], [x[2] for x in xs], ys)
    _clean()
    for a, b in zip(ys, ref):
        assert rel_err(a.cpu().double().numpy(), b.cpu().double().numpy()) <= 1e-2
    for a, b in zip(st, ref_st):
        assert rel_err(a.cpu().double().numpy(), b.cpu().double().numpy()) <= 1e-5


@pytest.mark.parametrize("L", [1, 17, 3000])
def test_chunked_layers_in_bounds(dbg, oracle, L):
    """Three layers in one launch (with L = 3000 and one 64-channel head per layer the sequences are
    split into segments: look-back across the layers' items) in the bounds-checked build."""
    nl, B, Dch, H, d = 3, 1, 64, 1, 2
    cases = [_case(B, L, Dch, H, d, "bf16", 200 + 10 * l + L % 7) for l in range(nl)]
    qkv = [W.prefill_inputs(w) for w, _ in cases]
    dev = [dev_params(p) for _, p in cases]
    qs, ks, vs = ([x[j].cuda() for x in qkv] for j in range(3))
    ys = [torch.empty_like(q) for q in qs]
    sts = [torch.empty((B, d, Dch, 2), device="cuda") for _ in range(nl)]
    ls = ops.PrefillLayerSet(qs, ks, vs, ys, sts, [x[0] for x in dev], [x[1] for x in dev], [x[2] for x in dev])
    ws = ops.prefill_chunked_layers(ls)
    _clean()
    assert ls.error(ws) == 0
    for l, (w, p) in enumerate(cases):
        qf, kf, vf = (W.to_f64(t) for t in qkv[l])
        y_ref, s_ref = oracle.recurrent(qf, kf, vf, p.lam, p.R, p.Dskip, H=H)
        assert rel_err(ys[l].cpu().double().numpy(), y_ref) <= TOL["bf16"]
        assert rel_err(state_c128(sts[l]), s_ref) <= TOL["bf16"]
