"""GPU parity of the undistilled decode baseline (cached-activation long convolution).

hyena_fir_decode_step emits token t as q_t * sum_{j<=t} h_{t-j} u_j over the cached history, the
way generation works without the distilled recurrence.  Its outputs must match the oracle's direct
convolution (the plain definition) and, within the same tolerance, the modal route: chunked or FFT
prefill followed by hyena_decode_step.  Tolerance per output tensor: 1e-4 of max|oracle| for fp32
activations, 2e-2 for bf16.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, column_params, dev_params, gather_columns, rel_err, sample_columns

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _inputs(w, T):
    q, k, v = W.prefill_inputs(w)
    steps = [W.decode_inputs(w, t) for t in range(T)]
    qa = torch.cat([q, torch.stack([s[0] for s in steps], 1)], 1)
    ka = torch.cat([k, torch.stack([s[1] for s in steps], 1)], 1)
    va = torch.cat([v, torch.stack([s[2] for s in steps], 1)], 1)
    return (q, k, v), steps, (qa, ka, va)


def _fir_run(w, p, prompt, steps, t_max):
    lam, R, D = dev_params(p)
    h = ops.filter_from_modes(lam, R, D, t_max)
    u = ops.fir_cache_prompt(prompt[1].cuda(), prompt[2].cuda(), t_max)
    ys = []
    for t, (a, b, c) in enumerate(steps):
        ys.append(ops.fir_decode_step(a.cuda(), b.cuda(), c.cuda(), h, u, w.L + t).cpu())
    torch.cuda.synchronize()
    return torch.stack(ys, 1), u


@pytest.mark.parametrize("B,L,Dch,H,d,dt,T", [
    (2, 40, 64, 4, 8, "f32", 10),
    (3, 77, 96, 3, 5, "bf16", 9),      # Dch not a multiple of 32
    (1, 0, 32, 1, 4, "f32", 12),       # no prompt: the history starts empty
    (2, 300, 160, 5, 16, "bf16", 33),  # long enough for the unrolled history loop and its tail
])
def test_fir_small_full_compare(oracle, B, L, Dch, H, d, dt, T):
    w = W.Workload(500 + L + T, "case", B=B, L=L, Dch=Dch, H=H, d=d, dtype=dt, fft_len=0, T=T)
    p = W.params(w)
    prompt, steps, (qa, ka, va) = _inputs(w, T)
    t_max = L + T + 3
    y_fir, u = _fir_run(w, p, prompt, steps, t_max)
    h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, L + T)
    y_ref = oracle.conv_direct(W.to_f64(qa), W.to_f64(ka), W.to_f64(va), h, H=H)[:, L:]
    assert rel_err(y_fir.double().numpy(), y_ref) <= TOL[dt]
    # the cache holds k v, rounded once to fp32, for every token seen (exact for bf16 inputs)
    u_ref = (ka.float() * va.float()).double().numpy()
    assert np.array_equal(u[:, :L + T].cpu().double().numpy(), u_ref)


def test_fir_matches_modal_decode():
    """The two decode routes compute the same operator: FIR over the history and the modal
    recurrence from the prefill state agree within the bf16 bar."""
    w = W.Workload(560, "case", B=4, L=256, Dch=256, H=2, d=16, dtype="bf16", fft_len=512, T=16)
    p = W.params(w)
    prompt, steps, _ = _inputs(w, w.T)
    y_fir, _ = _fir_run(w, p, prompt, steps, w.L + w.T)
    lam, R, D = dev_params(p)
    _, s = ops.prefill(*(x.cuda() for x in prompt), lam, R, D, w.fft_len)
    y_mod = torch.stack([ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s).cpu()
                         for a, b, c in steps], 1)
    assert rel_err(y_fir.double().numpy(), y_mod.double().numpy()) <= TOL["bf16"]


def test_fir_gen_layer_full_size_sampled(oracle):
    """One 1.3B-shaped layer (B=64, 512-token prompt, Dch=2048): 4 FIR steps, sampled columns."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    p = W.params(w)
    T = 4
    prompt, steps, (qa, ka, va) = _inputs(w, T)
    y_fir, _ = _fir_run(w, p, prompt, steps, w.L + w.T)
    bc = sample_columns(np.random.default_rng(9), w.B, w.Dch, 32)
    lam_c, R_c, D_c = column_params(p, w.H, w.Dch, [c for _, c in bc])
    h = oracle.filter_from_modes(lam_c, R_c, D_c, w.L + T)
    y_ref = oracle.conv_direct(gather_columns(qa, bc), gather_columns(ka, bc), gather_columns(va, bc), h,
                               H=len(bc))[:, w.L:]
    ib = torch.tensor([b for b, _ in bc]); ic = torch.tensor([c for _, c in bc])
    y_gpu = y_fir[ib, :, ic].transpose(0, 1).double().numpy()[None]
    assert rel_err(y_gpu, y_ref) <= TOL["bf16"]
