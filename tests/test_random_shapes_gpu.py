"""Seeded random shapes through every route, against the fp64 oracle.

The fixed cases elsewhere cover the edges that the layouts suggest (one token, ragged prompts, one
channel per head, odd heads, segment counts).  This sweep draws 24 more shapes from a fixed seed, so
that combinations nobody thought of also run: B in 1..3, prompt lengths 1..3000, 1..4 heads with
1..80 channels each (multiples of 64 for the chunked route), d in 1..16, bf16 and fp32, and 1..6 decode
steps after each prefill.  Every output is compared with the oracle's recurrence over prompt and
generated tokens.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, dev_params, rel_err, state_c128

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _shapes():
    rng = np.random.default_rng(20261202)
    out = []
    for i in range(24):
        route = ["fft", "chunked", "fft"][i % 3]
        B = int(rng.integers(1, 4))
        L = int(rng.choice([1, 2, 63, 64, 65, int(rng.integers(3, 3000))]))
        H = int(rng.integers(1, 5))
        ch = 64 * int(rng.integers(1, 3)) if route == "chunked" else int(rng.integers(1, 81))
        d = int(rng.integers(1, 17))
        dtype = "bf16" if route == "chunked" else ["f32", "bf16"][int(rng.integers(0, 2))]
        T = int(rng.integers(1, 7))
        out.append((route, B, L, H * ch, H, d, dtype, T))
    return out


@pytest.mark.parametrize("route,B,L,Dch,H,d,dtype,T", _shapes())
def test_random_shape_prefill_then_decode(oracle, route, B, L, Dch, H, d, dtype, T):
    w = W.Workload(800 + L % 97 + d, "rand", B=B, L=L, Dch=Dch, H=H, d=d, dtype=dtype, fft_len=0, T=0)
    p = W.params(w)
    lam, R, D = dev_params(p)
    q, k, v = W.prefill_inputs(w)
    if route == "chunked":
        y, s, ws = ops.prefill_chunked(q.cuda(), k.cuda(), v.cuda(), lam, R, D)
        assert ops.chunked_error(ws, B, L, Dch, H, d) == 0
    else:
        y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, max(64, 1 << (2 * L - 1).bit_length()))
    s_pre = state_c128(s)
    steps = [W.decode_inputs(w, t) for t in range(T)]
    yd = [ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, s) for a, b, c in steps]
    torch.cuda.synchronize()
    qa = np.concatenate([W.to_f64(q), W.to_f64(torch.stack([a for a, _, _ in steps], 1))], 1)
    ka = np.concatenate([W.to_f64(k), W.to_f64(torch.stack([b for _, b, _ in steps], 1))], 1)
    va = np.concatenate([W.to_f64(v), W.to_f64(torch.stack([c for _, _, c in steps], 1))], 1)
    y_ref, _ = oracle.recurrent(qa, ka, va, p.lam, p.R, p.Dskip, H=H)
    _, s_ref = oracle.recurrent(W.to_f64(q), W.to_f64(k), W.to_f64(v), p.lam, p.R, p.Dskip, H=H)
    got = np.concatenate([y.cpu().double().numpy(), torch.stack([t.cpu() for t in yd], 1).double().numpy()], 1)
    tol = TOL[dtype]
    assert rel_err(got, y_ref) <= tol, rel_err(got, y_ref)
    assert rel_err(s_pre, s_ref) <= tol, rel_err(s_pre, s_ref)
