"""FFT prefill on the tensor cores (bf16 activations; FFT lengths 4096, 8192, 16384, and the
inner 8192-point rows of the four-step route beyond).

hyena_prefill runs these calls with each transform factored as 64 x 64 x (N/4096): the two
64-point DFT stages are dense matrix products on the tensor cores (bf16 operands, fp32
accumulation), the twiddles, the small DFT over the last factor and the spectral product run
in fp32 on the CUDA cores.  These tests compare it element by element with the fp64 oracle (the
direct causal convolution with the modal filter, and the prompt state by its sum) over ragged
prompt lengths, several channel groups, heads of 2 to 8 channels and d from 1 to 64; they check
that the call really took the tensor-core route (its rounding differs from the CUDA-core route's
on the same inputs), that it is deterministic, that its error word stays 0, and that its
bounds-checked build makes no out-of-range access.
"""
import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W
from parity_util import TOL, dev_params, rel_err, state_c128

pytestmark = pytest.mark.gpu

# measured margins asserted besides the bf16 bar (the errors are printed by the conftest summary):
# y carries the bf16 rounding of u, of the DFT matrix and of three intermediate operands; the
# state is summed in fp32 from fp32 u while the window fits the 1024-token fp32 copy
Y_MARGIN = 1e-2
S_MARGIN = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from distilled_ssm_decode_b200 import build
    build.build()


def _case(seed, B, L, Dch, H, d, rmin=0.5, rmax=0.95):
    w = W.Workload(700 + seed, "monarch", B=B, L=L, Dch=Dch, H=H, d=d, dtype="bf16", fft_len=0, T=0,
                   rmin=rmin, rmax=rmax)
    return w, W.params(w)


def _oracle(oracle, w, p, q, k, v):
    qf, kf, vf = W.to_f64(q), W.to_f64(k), W.to_f64(v)
    h = oracle.filter_from_modes(p.lam, p.R, p.Dskip, w.L)
    return oracle.conv_direct(qf, kf, vf, h, H=w.H), oracle.prompt_state(kf, vf, p.lam, H=w.H)


def _run(w, p, N, tensor_cores=True):
    q, k, v = W.prefill_inputs(w)
    lam, R, D = dev_params(p)
    nbytes = ops.prefill_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d, N)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    with ops.fft_tensor_cores(tensor_cores):
        y, s = ops.prefill(q.cuda(), k.cuda(), v.cuda(), lam, R, D, N, workspace=ws)
    assert ops.prefill_error(ws, w.B, w.L, w.Dch, w.H, w.d, N) == 0
    return (q, k, v), y, s


CASES = [
    # B, L, Dch, H, d, fft_len
    (1, 2048, 16, 2, 16, 4096),      # whole half-length prompt, 64 x 64 x 1
    (2, 1000, 16, 1, 8, 4096),       # ragged prompt, two sequences
    (1, 4096, 16, 2, 16, 8192),      # 64 x 64 x 2 (the mid workload's length)
    (2, 3001, 24, 3, 16, 8192),      # ragged, three channel groups per sequence
    (1, 8192, 8, 2, 16, 16384),      # 64 x 64 x 4, two channel groups of 4
    (1, 5000, 12, 3, 4, 16384),      # ragged, heads of 4 channels
    (1, 1, 8, 1, 1, 4096),           # a single token, d = 1
    (1, 17, 8, 4, 64, 8192),         # d at the maximum, heads of 2 channels
    (3, 700, 16, 8, 20, 4096),       # d = 20 (two state segments per mode), 8 heads
    (1, 129, 8, 2, 2, 4096),         # a prompt just past two token rows of 64
]


@pytest.mark.parametrize("B,L,Dch,H,d,N", CASES)
def test_tensor_core_prefill_matches_oracle(oracle, record_property, B, L, Dch, H, d, N):
    w, p = _case(L + Dch + d + N // 4096, B, L, Dch, H, d)
    (q, k, v), y, s = _run(w, p, N)
    y_ref, s_ref = _oracle(oracle, w, p, q, k, v)
    ey = rel_err(y.cpu().double().numpy(), y_ref)
    es = rel_err(state_c128(s), s_ref)
    record_property("y_err", ey)
    record_property("state_err", es)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)
    assert ey <= Y_MARGIN and es <= S_MARGIN, (ey, es)


def test_long_memory_poles_use_the_bf16_part_of_the_state(oracle, record_property):
    """|lambda| up to 0.999: the state window spans the whole prompt, beyond the 1024 tokens
    whose u is kept in fp32; the older tokens enter from the bf16 operand."""
    w, p = _case(91, 1, 6000, 8, 2, 16, rmin=0.99, rmax=0.999)
    (q, k, v), y, s = _run(w, p, 16384)
    y_ref, s_ref = _oracle(oracle, w, p, q, k, v)
    ey = rel_err(y.cpu().double().numpy(), y_ref)
    es = rel_err(state_c128(s), s_ref)
    record_property("y_err", ey)
    record_property("state_err", es)
    assert ey <= TOL["bf16"] and es <= TOL["bf16"], (ey, es)


def test_route_is_taken_and_both_routes_agree():
    """Same inputs through both routes: different roundings (so the tensor-core route ran),
    the same operator within the bf16 bar; the states agree to fp32 rounding."""
    w, p = _case(5, 2, 4096, 32, 4, 16)
    (q, k, v), y_tc, s_tc = _run(w, p, 8192, tensor_cores=True)
    _, y_cc, s_cc = _run(w, p, 8192, tensor_cores=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert ops.prefill_uses_tensor_cores(qd, kd, vd, w.H, w.d, 8192)
    with ops.fft_tensor_cores(False):
        assert not ops.prefill_uses_tensor_cores(qd, kd, vd, w.H, w.d, 8192)
    assert not torch.equal(y_tc, y_cc)
    assert rel_err(y_tc.cpu().double().numpy(), y_cc.cpu().double().numpy()) <= Y_MARGIN
    assert rel_err(state_c128(s_tc), state_c128(s_cc)) <= 1e-5


def test_tensor_core_prefill_is_deterministic():
    w, p = _case(6, 2, 3000, 16, 2, 16)
    _, y1, s1 = _run(w, p, 8192)
    _, y2, s2 = _run(w, p, 8192)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_layouts_outside_the_route_fall_back_to_cuda_cores(oracle):
    """Dch not a multiple of 8 at FFT length 8192: the CUDA-core route, still within the bar."""
    w, p = _case(7, 1, 2000, 12, 2, 8)
    (q, k, v), y, s = _run(w, p, 8192)
    assert not ops.prefill_uses_tensor_cores(q.cuda(), k.cuda(), v.cuda(), w.H, w.d, 8192)
    y_ref, s_ref = _oracle(oracle, w, p, q, k, v)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["bf16"]
    assert rel_err(state_c128(s), s_ref) <= 1e-4


FOURSTEP = [
    # B, L, Dch, H, d, fft_len: the four-step route, inner 8192-point rows on the tensor cores
    (1, 9000, 6, 3, 4, 32768),       # ragged, heads of 2 channels
    (2, 20000, 8, 2, 16, 65536),     # two sequences, N1 = 8
    (1, 40000, 4, 1, 8, 131072),     # N1 = 16 (the long prefill's length)
]


@pytest.mark.parametrize("B,L,Dch,H,d,N", FOURSTEP)
def test_four_step_inner_rows_on_tensor_cores(oracle, record_property, B, L, Dch, H, d, N):
    w, p = _case(L % 97 + d, B, L, Dch, H, d)
    (q, k, v), y, s = _run(w, p, N)
    assert ops.prefill_uses_tensor_cores(q.cuda(), k.cuda(), v.cuda(), H, d, N)
    y_ref, s_ref = oracle.recurrent(W.to_f64(q), W.to_f64(k), W.to_f64(v), p.lam, p.R, p.Dskip, H=H)
    ey = rel_err(y.cpu().double().numpy(), y_ref)
    es = rel_err(state_c128(s), s_ref)
    record_property("y_err", ey)
    record_property("state_err", es)
    assert ey <= TOL["bf16"] and es <= 1e-4, (ey, es)
    assert ey <= Y_MARGIN, ey
    with ops.fft_tensor_cores(False):
        _, y_cc, _ = _run(w, p, N, tensor_cores=False)
    assert not torch.equal(y, y_cc)


@pytest.mark.parametrize("L", [1, 2, 3, 17, 200])
@pytest.mark.parametrize("N,Dch,H", [(4096, 8, 2), (8192, 16, 8), (16384, 4, 1), (32768, 6, 3)])
def test_tensor_core_prefill_in_bounds(oracle, L, N, Dch, H):
    """The bounds-checked build: no global access out of range, results as in the release build."""
    from distilled_ssm_decode_b200 import build
    path = build.build(debug_bounds=True)
    w, p = _case(L + N // 4096, 1 + (L % 2), L, Dch, H, 2)
    with ops.using_library(path):
        (q, k, v), y, s = _run(w, p, N)
        torch.cuda.synchronize()
        st, rec = ops.bounds_check()
    assert st == 0, f"out-of-range access recorded: file {rec[0]}, line {rec[1]}, index {rec[2]}, extent {rec[3]}"
    y_ref, s_ref = _oracle(oracle, w, p, q, k, v)
    assert rel_err(y.cpu().double().numpy(), y_ref) <= TOL["bf16"]
    assert rel_err(state_c128(s), s_ref) <= 1e-4
