"""GPU parity of the grouped decode step (hyena_decode_step_layers) against the fp64 oracle.

Several independent operator layers advance by one token in a single launch; each layer has
its own parameters, state and activations.  Every layer must match the oracle's recurrence
for that layer alone (tolerance per output tensor as in the other parity tests: 1e-4 of
max|oracle| for fp32 activations, 2e-2 for bf16).  Small cases compare every element; the
1.3B-shaped workload (24 layers x B=64 x Dch=2048, d=16) compares sampled columns of every
layer after a few steps from a random state.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, column_params, dev_params, rel_err, sample_columns, state_c128

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _layer_inputs(w, layers, T, B):
    """Per layer: params, initial state (complex64 [B][d][Dch]) and T steps of (q, k, v)."""
    out = []
    for l in range(layers):
        p = W.params(w, layer=l)
        s0 = W.initial_state(w, B=B, layer=l)
        steps = [W.decode_inputs(w, t, layer=l, B=B) for t in range(T)]
        out.append((p, s0, steps))
    return out


def _run_layers(w, data, T, B):
    lams, Rs, Ds, states = [], [], [], []
    for p, s0, _ in data:
        lam, R, D = dev_params(p)
        lams.append(lam); Rs.append(R); Ds.append(D)
        states.append(torch.view_as_real(s0).contiguous().cuda())
    ls = ops.LayerSet(lams, Rs, Ds, states)
    ys = []
    for t in range(T):
        qs = [d[2][t][0].cuda() for d in data]
        ks = [d[2][t][1].cuda() for d in data]
        vs = [d[2][t][2].cuda() for d in data]
        yo = [torch.empty_like(q) for q in qs]
        ops.decode_step_layers(ls, qs, ks, vs, yo)
        ys.append([y.cpu() for y in yo])
    torch.cuda.synchronize()
    return ys, states


@pytest.mark.parametrize("layers,B,Dch,H,d,dt", [
    (3, 2, 64, 4, 8, "f32"),
    (5, 3, 128, 2, 16, "bf16"),
    (1, 1, 8, 1, 3, "bf16"),
    (7, 4, 96, 3, 5, "f32"),
])
def test_layers_small_full_compare(oracle, layers, B, Dch, H, d, dt):
    w = W.Workload(400 + layers, "case", B=B, L=0, Dch=Dch, H=H, d=d, dtype=dt, fft_len=0, T=0)
    T = 6
    data = _layer_inputs(w, layers, T, B)
    ys, states = _run_layers(w, data, T, B)
    for l, (p, s0, steps) in enumerate(data):
        qs = W.to_f64(torch.stack([st[0] for st in steps], 1))
        ks = W.to_f64(torch.stack([st[1] for st in steps], 1))
        vs = W.to_f64(torch.stack([st[2] for st in steps], 1))
        y_ref, s_ref = oracle.recurrent(qs, ks, vs, p.lam, p.R, p.Dskip, H=H,
                                        state=s0.to(torch.complex128).numpy())
        y_gpu = torch.stack([ys[t][l] for t in range(T)], 1).double().numpy()
        assert rel_err(y_gpu, y_ref) <= TOL[dt], l
        assert rel_err(state_c128(states[l]), s_ref) <= TOL[dt], l


def test_layers_match_single_layer_steps():
    """Grouped and one-layer-at-a-time steps compute the same operator (bf16 bar)."""
    w = W.Workload(450, "case", B=4, L=0, Dch=256, H=2, d=16, dtype="bf16", fft_len=0, T=0)
    data = _layer_inputs(w, 4, 3, 4)
    ys, states = _run_layers(w, data, 3, 4)
    for l, (p, s0, steps) in enumerate(data):
        lam, R, D = dev_params(p)
        s = torch.view_as_real(s0).contiguous().cuda()
        for t in range(3):
            y1 = ops.decode_step(*(x.cuda() for x in steps[t]), lam, R, D, s).cpu()
            assert rel_err(ys[t][l].double().numpy(), y1.double().numpy()) <= TOL["bf16"]
        assert rel_err(state_c128(states[l]), state_c128(s)) <= 1e-5


def test_layers_gen1p3b_full_size_sampled(oracle):
    """All 24 layers of the 1.3B-shaped workload (B=64, Dch=2048, H=16, d=16, bf16) from a
    random N(0,1) state, 3 grouped steps; 16 sampled columns of every layer."""
    w = W.WORKLOADS["gen1p3b_bf16"]
    layers, T, B = w.layers, 3, w.B
    data = _layer_inputs(w, layers, T, B)
    ys, states = _run_layers(w, data, T, B)
    rng = np.random.default_rng(24)
    for l, (p, s0, steps) in enumerate(data):
        bc = sample_columns(rng, B, w.Dch, 16)
        ib = torch.tensor([b for b, _ in bc]); ic = torch.tensor([c for _, c in bc])
        qs = W.to_f64(torch.stack([st[0][ib, ic] for st in steps]))[None]
        ks = W.to_f64(torch.stack([st[1][ib, ic] for st in steps]))[None]
        vs = W.to_f64(torch.stack([st[2][ib, ic] for st in steps]))[None]
        lam_c, R_c, D_c = column_params(p, w.H, w.Dch, [c for _, c in bc])
        s0c = s0.to(torch.complex128).numpy()
        st0 = np.stack([s0c[b, :, c] for b, c in bc], -1)[None]
        y_ref, s_ref = oracle.recurrent(qs, ks, vs, lam_c, R_c, D_c, H=len(bc), state=st0)
        y_gpu = torch.stack([ys[t][l][ib, ic] for t in range(T)]).double().numpy()[None]
        assert rel_err(y_gpu, y_ref) <= TOL["bf16"], l
        sg = state_c128(states[l])
        assert rel_err(np.stack([sg[b, :, c] for b, c in bc], -1)[None], s_ref) <= TOL["bf16"], l


def test_layers_rejects_bad_arguments():
    w = W.Workload(460, "case", B=2, L=0, Dch=64, H=2, d=4, dtype="bf16", fft_len=0, T=0)
    data = _layer_inputs(w, 2, 1, 2)
    lams, Rs, Ds, states = [], [], [], []
    for p, s0, _ in data:
        lam, R, D = dev_params(p)
        lams.append(lam); Rs.append(R); Ds.append(D)
        states.append(torch.view_as_real(s0).contiguous().cuda())
    ls = ops.LayerSet(lams, Rs, Ds, states)
    q = [data[l][2][0][0].cuda() for l in range(2)]
    y = [torch.empty_like(x) for x in q]
    odd = [torch.zeros(2, 63, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(ops.HyenaError) as e:          # Dch odd: the grouped step needs channel pairs
        ops.decode_step_layers(ls, odd, odd, odd, [torch.empty_like(x) for x in odd])
    assert e.value.status in (-2, -5)
    mis = [torch.zeros(2 * 64 + 1, dtype=torch.bfloat16, device="cuda")[1:].view(2, 64) for _ in range(2)]
    with pytest.raises(ops.HyenaError) as e:          # activations not aligned to a channel pair
        ops.decode_step_layers(ls, mis, q, q, y)
    assert e.value.status == -3


def test_layers_flow_chunked_prefill_then_grouped_decode(oracle):
    """The 24-layer benchmark's flow on 3 small layers: each layer's chunked prefill, then grouped
    decode steps over all layers from those states; every element against the oracle."""
    w = W.Workload(480, "case", B=2, L=300, Dch=128, H=2, d=8, dtype="bf16", fft_len=0, T=0)
    layers, T = 3, 4
    ps = [W.params(w, layer=l) for l in range(layers)]
    prompts = [W.prefill_inputs(w, layer=l) for l in range(layers)]
    steps = [[W.decode_inputs(w, t, layer=l) for t in range(T)] for l in range(layers)]
    lams, Rs, Ds, states = [], [], [], []
    for l in range(layers):
        lam, R, D = dev_params(ps[l])
        _, s, _ = ops.prefill_chunked(*(x.cuda() for x in prompts[l]), lam, R, D)
        lams.append(lam); Rs.append(R); Ds.append(D); states.append(s)
    ls = ops.LayerSet(lams, Rs, Ds, states)
    ys = []
    for t in range(T):
        yo = [torch.empty(w.B, w.Dch, dtype=torch.bfloat16, device="cuda") for _ in range(layers)]
        ops.decode_step_layers(ls, [steps[l][t][0].cuda() for l in range(layers)],
                               [steps[l][t][1].cuda() for l in range(layers)],
                               [steps[l][t][2].cuda() for l in range(layers)], yo)
        ys.append([y.cpu() for y in yo])
    for l in range(layers):
        qa = np.concatenate([W.to_f64(prompts[l][0]), W.to_f64(torch.stack([x[0] for x in steps[l]], 1))], 1)
        ka = np.concatenate([W.to_f64(prompts[l][1]), W.to_f64(torch.stack([x[1] for x in steps[l]], 1))], 1)
        va = np.concatenate([W.to_f64(prompts[l][2]), W.to_f64(torch.stack([x[2] for x in steps[l]], 1))], 1)
        y_ref, s_ref = oracle.recurrent(qa, ka, va, ps[l].lam, ps[l].R, ps[l].Dskip, H=w.H)
        y_gpu = torch.stack([ys[t][l] for t in range(T)], 1).double().numpy()
        assert rel_err(y_gpu, y_ref[:, w.L:]) <= TOL["bf16"], l
        assert rel_err(state_c128(states[l]), s_ref) <= TOL["bf16"], l
