"""Checkpoint / resume of generation through the recurrent state.

The distilled operator's whole context after a prompt is the O(d) recurrent state per
channel ("Laughing Hyena Distillery", nubint.ai review, "Main findings": O(d) memory per
channel instead of a cache that grows with the sequence).  So a generation can be stopped
after any token, its state copied to host memory, and resumed later in a fresh device
buffer.  These tests run prefill -> decode, stop, move the state through the host into a
new buffer (and, for the multi-layer entry point, into buffers of a new layer set), go on
decoding, and require the outputs and the final state to be bit-identical to a run that
never stopped: the resumed kernels see exactly the same numbers.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import dev_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _decode(steps, lam, R, D, state):
    return [ops.decode_step(a.cuda(), b.cuda(), c.cuda(), lam, R, D, state) for a, b, c in steps]


@pytest.mark.parametrize("route,wl,B,L,Dch,T,stop", [
    ("fft", "tiny_f32", 1, 256, 64, 12, 5),
    ("chunked", "mid_bf16", 2, 1000, 256, 10, 4),
    ("fft", "mid_bf16", 2, 700, 256, 6, 0),          # checkpoint right after the prompt
])
def test_resume_from_host_state_is_bit_identical(route, wl, B, L, Dch, T, stop):
    w = W.WORKLOADS[wl]
    H = max(1, Dch // (w.Dch // w.H))
    p = W.params(w, H=H)
    lam, R, D = dev_params(p)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, B=B, L=L, Dch=Dch))
    steps = [W.decode_inputs(w, t, B=B, Dch=Dch) for t in range(T)]

    def prefill():
        if route == "chunked":
            y, s, ws = ops.prefill_chunked(q, k, v, lam, R, D)
            assert ops.chunked_error(ws, B, L, Dch, H, w.d) == 0
            return y, s
        return ops.prefill(q, k, v, lam, R, D, 1 << (2 * L - 1).bit_length())

    # uninterrupted
    y_a, s_a = prefill()
    yd_a = _decode(steps, lam, R, D, s_a)
    # interrupted after `stop` tokens: the state goes to host memory and back into a new buffer
    y_b, s_b = prefill()
    yd_b = _decode(steps[:stop], lam, R, D, s_b)
    torch.cuda.synchronize()
    host = s_b.cpu().numpy().copy()
    del s_b
    torch.cuda.empty_cache()
    s_c = torch.from_numpy(host).cuda()
    yd_b += _decode(steps[stop:], lam, R, D, s_c)
    assert torch.equal(y_a, y_b)
    for a, b in zip(yd_a, yd_b):
        assert torch.equal(a, b)
    assert torch.equal(s_a, s_c)


def test_resume_multi_layer_decode_in_new_layer_set():
    """24 layers of the 1.3B shape at a small batch: stop the grouped decode after a few tokens,
    save every layer's state to host, rebuild the layer set on fresh buffers and continue."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    nl, B, T, stop = 24, 2, 8, 3
    ps = [W.params(w, layer=l) for l in range(nl)]
    lams, Rs, Ds = zip(*(dev_params(p) for p in ps))
    g = torch.Generator().manual_seed(3)
    s0 = [torch.randn((B, w.d, w.Dch, 2), generator=g).cuda() for _ in range(nl)]
    x = [[torch.randn((nl, B, w.Dch), generator=g).to(torch.bfloat16).cuda() for _ in range(3)] for _ in range(T)]

    def run(states, ts):
        ls = ops.LayerSet(list(lams), list(Rs), list(Ds), states)
        out = []
        for t in ts:
            y = torch.empty((nl, B, w.Dch), dtype=torch.bfloat16, device="cuda")
            ops.decode_step_layers(ls, list(x[t][0]), list(x[t][1]), list(x[t][2]), list(y))
            out.append(y)
        return out

    sa = [s.clone() for s in s0]
    ya = run(sa, range(T))
    sb = [s.clone() for s in s0]
    yb = run(sb, range(stop))
    torch.cuda.synchronize()
    host = [s.cpu().numpy().copy() for s in sb]
    del sb
    sc = [torch.from_numpy(h).cuda() for h in host]
    yb += run(sc, range(stop, T))
    for a, b in zip(ya, yb):
        assert torch.equal(a, b)
    for a, c in zip(sa, sc):
        assert torch.equal(a, c)
    assert np.isfinite(host[0]).all()
