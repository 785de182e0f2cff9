"""GPU parity of modal truncation (hyena_modal_truncate) against the fp64 oracle.

The kept modes are an integer decision taken in fp64 on both sides from the same fp32 parameters,
so kept indices and the copied modes must match exactly; the bound (a sum of the dropped scores in
index order) to fp64 rounding; the closed-form l2 error on the GPU against the oracle's direct
summation over the taps to 1e-9 relative.
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


def _cases():
    yield "mid", W.params(W.WORKLOADS["mid_bf16"])
    yield "long", W.params(W.WORKLOADS["long_prefill_bf16"])        # |lambda| up to 0.999
    w = W.Workload(700, "case", B=1, L=0, Dch=5, H=5, d=64, dtype="f32", fft_len=0, T=0)
    yield "d64", W.params(w)                                          # the largest mode count


@pytest.mark.parametrize("name,p", list(_cases()), ids=lambda x: x if isinstance(x, str) else "")
def test_truncation_matches_oracle(oracle, name, p):
    lam, R, _ = dev_params(p)
    d = lam.shape[1]
    for k in sorted({0, 1, 5, d // 2, d - 1, d}):
        kept, lo, ro, b, e = ops.modal_truncate(lam, R, k)
        # taps until the slowest mode has decayed below 1e-40 of its start: the tail is far below fp64
        J = int(np.ceil(np.log(1e-40) / np.log(np.abs(p.lam).max()))) + 1
        kr, lor, ror, br, e1r, e2r = oracle.modal_truncate(p.lam, p.R, k, J=J)
        assert np.array_equal(kept.cpu().numpy(), kr), k
        lo_c = lo.cpu().double().numpy(); ro_c = ro.cpu().double().numpy()
        assert np.array_equal(lo_c[..., 0] + 1j * lo_c[..., 1], lor), k
        assert np.array_equal(ro_c[..., 0] + 1j * ro_c[..., 1], ror), k
        np.testing.assert_allclose(b.cpu().numpy(), br, rtol=1e-14, atol=0)
        np.testing.assert_allclose(e.cpu().numpy(), e2r, rtol=1e-9, atol=1e-300)
        assert np.all(e1r <= br * (1 + 1e-12))


def test_truncation_ties_and_zero_pole():
    """Equal scores keep the lower index; lambda = 0 modes score |R|."""
    lam = torch.tensor([[[0.5, 0.0], [0.5, 0.0], [0.0, 0.0]]], device="cuda")
    R = torch.tensor([[[1.0, 0.0], [-1.0, 0.0], [2.0, 0.0]]], device="cuda")
    kept, _, _, b, e = ops.modal_truncate(lam, R, 1)
    assert kept.cpu().tolist() == [[0]]                 # scores 2, 2, 2: index 0 wins
    assert b.item() == pytest.approx(4.0, rel=1e-15)
    kept, _, _, b, _ = ops.modal_truncate(lam, R, 2)
    assert kept.cpu().tolist() == [[0, 1]]
