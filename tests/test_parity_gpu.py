"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Same seeded inputs on both sides.  Bar (per output tensor):
max|gpu - oracle| <= tol * max|oracle|, tol = 1e-4 (fp32 activations) or
2e-2 (bf16 activations, complex fp32 state).  Small cases compare every
element; the full-size workloads compare sampled (batch, channel) columns that
the oracle evaluates on their own (columns are independent).
"""
import json
import os

import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import (TOL, column_params, dev_params, gather_columns, rel_err, sample_columns,
                         state_c128)

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()
    torch.cuda.init()


def _random_case(seed, B, L, Dch, H, d, dtype, rmin=0.5, rmax=0.95):
    w = W.Workload(100 + seed, "case", B=B, L=L, Dch=Dch, H=H, d=d, dtype=dtype,
                   fft_len=0, T=0, rmin=rmin, rmax=rmax)
    return w, W.params(w)


# ---------------------------------------------------------------- filter (a1) and spectrum (a2)
@pytest.mark.parametrize("name,L", [("tiny_f32", 256), ("mid_bf16", 4096),
                                    ("long_prefill_bf16", 65536)])
def test_filter_parity(oracle, name, L):
    w = W.WORKLOADS[name]
    p = W.params(w)
    lam, R, D = dev_params(p)
    h = ops.filter_from_modes(lam, R, D, L).cpu().double().numpy()
    ref = oracle.filter_from_modes(p.lam, p.R, p.Dskip, L)
    assert rel_err(h, ref) <= 1e-6


def test_filter_zero_pole_is_two_tap(oracle):
    H, d, L = 2, 3, 9
    lam = torch.zeros(H, d, 2)
    R = torch.randn(H, d, 2, generator=torch.Generator().manual_seed(0))
    D = torch.tensor([0.5, -1.25])
    h = ops.filter_from_modes(lam.cuda(), R.cuda(), D.cuda(), L).cpu()
    assert torch.equal(h[:, 0], D)
    torch.testing.assert_close(h[:, 1], R[..., 0].sum(1), rtol=1e-6, atol=1e-6)
    assert torch.all(h[:, 2:] == 0)


@pytest.mark.parametrize("name,L,N,bins", [("tiny_f32", 256, 512, None),
                                           ("mid_bf16", 4096, 8192, 64),
                                           ("long_prefill_bf16", 65536, 131072, 64),
                                           ("tiny_f32", 50, 64, None)])
def test_spectrum_parity(oracle, name, L, N, bins):
    w = W.WORKLOADS[name]
    p = W.params(w)
    lam, R, D = dev_params(p)
    h = ops.filter_from_modes(lam, R, D, L)
    spec = ops.filter_spectrum(h, N).cpu().to(torch.complex128).numpy()
    hh = h.cpu().double().numpy()
    if bins is None:
        ref = oracle.spectrum(hh, N)
        got = spec
    else:
        rng = np.random.default_rng(N)
        sel = np.unique(np.concatenate([[0, 1, N // 2], rng.integers(0, N // 2 + 1, size=bins)]))
        ref = oracle.spectrum(hh, N, bins=sel)
        got = spec[:, sel]
    assert rel_err(got, ref) <= 1e-5


# ---------------------------------------------------------------- prefill (a3-a6)
def test_prefill_tiny_f32_full(oracle):
    w = W.WORKLOADS["tiny_f32"]
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, w.fft_len)
    h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, w.L)
    y_ref = oracle.conv_direct(W.to_f64(q), W.to_f64(k), W.to_f64(v), h, H=w.H)
    s_ref = oracle.prompt_state(W.to_f64(k), W.to_f64(v), p.lam, H=w.H)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["f32"]
    assert rel_err(state_c128(s), s_ref) <= TOL["f32"]


def _prefill_sampled(oracle, w, ncols, seed, direct=True):
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, w.fft_len)
    y = y.cpu()
    s = state_c128(s)
    rng = np.random.default_rng(seed)
    bc = sample_columns(rng, w.B, w.Dch, ncols)
    cols = [c for _, c in bc]
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, cols)
    qc, kc, vc = gather_columns(q, bc), gather_columns(k, bc), gather_columns(v, bc)
    if direct:
        h = oracle.filter_from_modes(lam_c, R_c, D_c, w.L)
        y_ref = oracle.conv_direct(qc, kc, vc, h, H=len(bc))
        s_ref = oracle.prompt_state(kc, vc, lam_c, H=len(bc))
    else:
        y_ref, s_ref = oracle.recurrent(qc, kc, vc, lam_c, R_c, D_c, H=len(bc))
    y_got = gather_columns(y, bc)
    s_got = np.stack([s[b, :, c] for b, c in bc], axis=-1)[None]
    return rel_err(y_got, y_ref), rel_err(s_got, s_ref)


def test_prefill_mid_bf16_full_size(oracle):
    ey, es = _prefill_sampled(oracle, W.WORKLOADS["mid_bf16"], ncols=24, seed=2)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)


def test_prefill_gen_layer_full_size(oracle):
    w = W.WORKLOADS["gen1p3b_bf16"]
    ey, es = _prefill_sampled(oracle, w, ncols=48, seed=3)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)


def test_prefill_long_four_step_full_size(oracle):
    w = W.WORKLOADS["long_prefill_bf16"]
    ey, es = _prefill_sampled(oracle, w, ncols=16, seed=4, direct=False)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)


EDGE = [
    # B, L, Dch, H, d, fft_len, dtype
    (1, 1, 2, 1, 1, 1, "f32"),        # single token, fft raised internally
    (1, 2, 4, 2, 2, 4, "f32"),
    (2, 3, 6, 2, 3, 8, "f32"),        # 3 channels per head: unpaired path
    (1, 17, 8, 4, 8, 64, "f32"),      # ragged prompt
    (1, 100, 4, 1, 20, 1024, "f32"),  # d > 16, fft_len >> 2L
    (2, 257, 12, 3, 5, 1024, "bf16"),  # ragged, odd d
    (1, 8192, 4, 2, 16, 16384, "bf16"),   # largest fused transform
    (1, 9000, 4, 1, 16, 32768, "f32"),    # smallest four-step transform, ragged L
    (1, 5000, 6, 3, 4, 16384, "bf16"),    # odd channels per head at a long length
    (3, 64, 32, 1, 64, 128, "f32"),       # d at the maximum
]


@pytest.mark.parametrize("B,L,Dch,H,d,N,dt", EDGE)
def test_prefill_edge_cases(oracle, B, L, Dch, H, d, N, dt):
    w, p = _random_case(L + Dch + d, B, L, Dch, H, d, dt)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, N)
    qf, kf, vf = W.to_f64(q), W.to_f64(k), W.to_f64(v)
    if L <= 4096:
        h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, L)
        y_ref = oracle.conv_direct(qf, kf, vf, h, H=H)
        s_ref = oracle.prompt_state(kf, vf, p.lam, H=H)
    else:
        y_ref, s_ref = oracle.recurrent(qf, kf, vf, p.lam, p.R, p.Dskip, H=H)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL[dt]
    assert rel_err(state_c128(s), s_ref) <= TOL[dt]


def test_prefill_empty_prompt_gives_zero_state():
    w, p = _random_case(1, 2, 0, 8, 2, 4, "bf16")
    lam, R, D = dev_params(p)
    q = torch.empty(2, 0, 8, dtype=torch.bfloat16, device="cuda")
    s = torch.full((2, 4, 8, 2), 7.0, device="cuda")
    _, s = ops.prefill(q, q, q, lam, R, D, 1, state=s)
    assert torch.all(s == 0)


def test_prefill_is_deterministic():
    w = W.WORKLOADS["mid_bf16"]
    p = W.params(w)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, B=2, L=1024, Dch=256))
    lam, R, D = dev_params(p)
    y1, s1 = ops.prefill(q, k, v, lam, R, D, 2048)
    y2, s2 = ops.prefill(q, k, v, lam, R, D, 2048)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_prompt_state_standalone(oracle):
    w = W.WORKLOADS["mid_bf16"]
    p = W.params(w)
    _, k, v = W.prefill_inputs(w, B=2, L=4096, Dch=64)
    lam, _, _ = dev_params(p)
    s = ops.prompt_state(k.cuda(), v.cuda(), lam, H=w.H)
    ref = oracle.prompt_state(W.to_f64(k), W.to_f64(v), p.lam, H=w.H)
    assert rel_err(state_c128(s), ref) <= 1e-4


# ---------------------------------------------------------------- decode (a7)
def test_prefill_then_decode_tiny_f32_equals_full_convolution(oracle):
    """GPU prompt state + GPU decode steps = the direct convolution over L+T tokens."""
    w = W.WORKLOADS["tiny_f32"]
    p = W.params(w)
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    _, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, w.fft_len)
    ys, dq, dk, dv = [], [], [], []
    for t in range(w.T):
        a, b, c = W.decode_inputs(w, t)
        dq.append(a); dk.append(b); dv.append(c)
        ys.append(ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu())
    y_dec = torch.stack(ys, 1).double().numpy()
    qa = np.concatenate([W.to_f64(q), W.to_f64(torch.stack(dq, 1))], 1)
    ka = np.concatenate([W.to_f64(k), W.to_f64(torch.stack(dk, 1))], 1)
    va = np.concatenate([W.to_f64(v), W.to_f64(torch.stack(dv, 1))], 1)
    h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, w.L + w.T)
    y_full = oracle.conv_direct(qa, ka, va, h, H=w.H)
    assert rel_err(y_dec, y_full[:, w.L:]) <= TOL["f32"]
    _, s_ref = oracle.recurrent(qa, ka, va, p.lam, p.R, p.Dskip, H=w.H)
    assert rel_err(state_c128(s), s_ref) <= TOL["f32"]


SWEEP_STEPS = {1: 1024, 16: 256, 64: 64, 256: 8, 1024: 4}


@pytest.mark.parametrize("B", [1, 16, 64, 256, 1024])
def test_decode_sweep_parity(oracle, B):
    w = W.WORKLOADS["decode_sweep_bf16"]
    p = W.params(w)
    lam, R, D = dev_params(p)
    T = SWEEP_STEPS[B]
    s0 = W.initial_state(w, B=B)
    s = torch.view_as_real(s0).contiguous().cuda()
    rng = np.random.default_rng(B)
    full = B * w.Dch <= 64 * 4096 and T * B <= 4096
    bc = None if full else sample_columns(rng, B, w.Dch, 64)
    ys, ins = [], []
    for t in range(T):
        a, b, c = W.decode_inputs(w, t, B=B)
        y = ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu()
        if full:
            ys.append(y); ins.append((a, b, c))
        else:
            idx_b = torch.tensor([x for x, _ in bc]); idx_c = torch.tensor([x for _, x in bc])
            ys.append(y[idx_b, idx_c]); ins.append(tuple(z[idx_b, idx_c] for z in (a, b, c)))
    y_gpu = torch.stack(ys, -2).double().numpy()       # [B][T][Dch] (full) or [T][ncol] (sampled)
    qs = W.to_f64(torch.stack([i[0] for i in ins], -2))
    ks = W.to_f64(torch.stack([i[1] for i in ins], -2))
    vs = W.to_f64(torch.stack([i[2] for i in ins], -2))
    s0c = s0.to(torch.complex128).numpy()
    if full:
        y_ref, s_ref = oracle.recurrent(qs, ks, vs, p.lam, p.R, p.Dskip, H=w.H, state=s0c)
        assert rel_err(y_gpu, y_ref) <= TOL["bf16"]
        assert rel_err(state_c128(s), s_ref) <= TOL["bf16"]
    else:
        cols = [c for _, c in bc]
        lam_c, R_c, D_c = column_params(p, w.H, w.Dch, cols)
        # columns as channels of one sequence: [1][T][ncol]
        qs1, ks1, vs1 = qs[None], ks[None], vs[None]
        st0 = np.stack([s0c[b, :, c] for b, c in bc], -1)[None]
        y_ref, s_ref = oracle.recurrent(qs1, ks1, vs1, lam_c, R_c, D_c, H=len(bc), state=st0)
        assert rel_err(y_gpu[None], y_ref) <= TOL["bf16"]
        sg = state_c128(s)
        s_got = np.stack([sg[b, :, c] for b, c in bc], -1)[None]
        assert rel_err(s_got, s_ref) <= TOL["bf16"]


def test_decode_gen_layer_after_prefill(oracle):
    """1.3B-shaped layer: GPU prefill of the 512-token prompt, then decode steps, sampled columns."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    p = W.params(w)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    _, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, w.fft_len)
    T = 8
    rng = np.random.default_rng(33)
    bc = sample_columns(rng, w.B, w.Dch, 32)
    ib = torch.tensor([b for b, _ in bc]); ic = torch.tensor([c for _, c in bc])
    ys, qs, ks, vs = [], [], [], []
    for t in range(T):
        a, b, c = W.decode_inputs(w, t)
        ys.append(ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu()[ib, ic])
        qs.append(a[ib, ic]); ks.append(b[ib, ic]); vs.append(c[ib, ic])
    cols = [c for _, c in bc]
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, cols)
    qa = np.concatenate([gather_columns(q, bc), W.to_f64(torch.stack(qs))[None]], 1)
    ka = np.concatenate([gather_columns(k, bc), W.to_f64(torch.stack(ks))[None]], 1)
    va = np.concatenate([gather_columns(v, bc), W.to_f64(torch.stack(vs))[None]], 1)
    y_ref, s_ref = oracle.recurrent(qa, ka, va, lam_c, R_c, D_c, H=len(bc))
    y_gpu = torch.stack(ys).double().numpy()[None]
    assert rel_err(y_gpu, y_ref[:, w.L:]) <= TOL["bf16"]
    sg = state_c128(s)
    assert rel_err(np.stack([sg[b, :, c] for b, c in bc], -1)[None], s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("B,Dch,H", [(8, 1024, 8), (16, 2048, 16), (2, 1024, 8), (16, 4096, 32), (17, 4096, 32)])
def test_decode_launch_shapes(oracle, B, Dch, H):
    """Channel-pair counts that select the launch shapes not covered by the sweep workload
    (4096 pairs: 8 lanes x 2 modes; 16384: 4 lanes x 2 modes; 1024: 16 lanes x 1 mode), including
    the mid-size workload's B=8, Dch=1024, and both sides of the bound of the early parameter loads
    on the 2-lane shape (32768 pairs: early; 34816: at first use); 6 steps from a random state,
    every element compared."""
    w = W.Workload(600 + B, "case", B=B, L=0, Dch=Dch, H=H, d=16, dtype="bf16", fft_len=0, T=0,
                   random_state0=True)
    p = W.params(w)
    lam, R, D = dev_params(p)
    s0 = W.initial_state(w)
    s = torch.view_as_real(s0).contiguous().cuda()
    steps = [W.decode_inputs(w, t) for t in range(6)]
    ys = [ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu() for a, b, c in steps]
    qs, ks, vs = (W.to_f64(torch.stack([x[i] for x in steps], 1)) for i in range(3))
    y_ref, s_ref = oracle.recurrent(qs, ks, vs, p.lam, p.R, p.Dskip, H=H, state=s0.to(torch.complex128).numpy())
    assert rel_err(torch.stack(ys, 1).double().numpy(), y_ref) <= TOL["bf16"]
    assert rel_err(state_c128(s), s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("B,Dch,H,d,dt", [(3, 64, 2, 64, "f32"), (2, 256, 4, 64, "bf16"), (5, 96, 3, 33, "bf16")])
def test_decode_many_modes(oracle, B, Dch, H, d, dt):
    """Mode counts up to the maximum (64) and an odd one above 32: every element, 5 steps."""
    w = W.Workload(650 + d, "case", B=B, L=0, Dch=Dch, H=H, d=d, dtype=dt, fft_len=0, T=0, random_state0=True)
    p = W.params(w)
    lam, R, D = dev_params(p)
    s0 = W.initial_state(w)
    s = torch.view_as_real(s0).contiguous().cuda()
    steps = [W.decode_inputs(w, t) for t in range(5)]
    ys = [ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu() for a, b, c in steps]
    qs, ks, vs = (W.to_f64(torch.stack([x[i] for x in steps], 1)) for i in range(3))
    y_ref, s_ref = oracle.recurrent(qs, ks, vs, p.lam, p.R, p.Dskip, H=H, state=s0.to(torch.complex128).numpy())
    assert rel_err(torch.stack(ys, 1).double().numpy(), y_ref) <= TOL[dt]
    assert rel_err(state_c128(s), s_ref) <= TOL[dt]


@pytest.mark.parametrize("Dch,H,dt", [(9, 3, "f32"), (6, 2, "bf16"), (7, 7, "bf16")])
def test_decode_scalar_layouts(oracle, Dch, H, dt):
    """Odd channel counts take the one-channel-per-thread kernel."""
    w, p = _random_case(Dch * 10 + H, 3, 0, Dch, H, 5, dt)
    lam, R, D = dev_params(p)
    g = np.random.default_rng(Dch)
    s0 = (g.normal(size=(3, 5, Dch)) + 1j * g.normal(size=(3, 5, Dch))).astype(np.complex64)
    s = torch.view_as_real(torch.from_numpy(s0)).contiguous().cuda()
    a, b, c = W.decode_inputs(w.with_(B=3, Dch=Dch), 0)
    y = ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu()
    y_ref, s_ref = oracle.recurrent(W.to_f64(a)[:, None], W.to_f64(b)[:, None], W.to_f64(c)[:, None],
                                    p.lam, p.R, p.Dskip, H=H, state=s0.astype(np.complex128))
    assert rel_err(y.double().numpy(), y_ref[:, 0]) <= TOL[dt]
    assert rel_err(state_c128(s), s_ref) <= 1e-5


def test_golden_hand_example_on_gpu():
    g = json.load(open(GOLD))["real_pole"]
    lam = torch.tensor(g["lam"], dtype=torch.float32).cuda()
    R = torch.tensor(g["R"], dtype=torch.float32).cuda()
    D = torch.tensor(g["Dskip"], dtype=torch.float32).cuda()
    k = torch.tensor(g["k"]).reshape(1, 3, 1)
    v = torch.tensor(g["v"]).reshape(1, 3, 1)
    q = torch.tensor(g["q"]).reshape(1, 3, 1)
    y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, 8)
    torch.testing.assert_close(y.cpu().ravel(), torch.tensor(g["y"]), rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(s.cpu().ravel(), torch.tensor(g["state"]), rtol=1e-6, atol=1e-6)
    dd = g["decode"]
    one = lambda x: torch.full((1, 1), float(x)).cuda()  # noqa: E731
    yd = ops.decode_step(one(dd["q"]), one(dd["k"]), one(dd["v"]), lam, R, D, s)
    assert abs(yd.item() - dd["y"]) < 1e-5
    torch.testing.assert_close(s.cpu().ravel(), torch.tensor(dd["state"]), rtol=1e-6, atol=1e-6)
