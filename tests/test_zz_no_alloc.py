"""The scratch-free prefill (hyena_prefill_noalloc) against the regular one.

hyena_prefill_noalloc is for callers that cannot allocate or pass device scratch
where they call us -- a plugin or FFI layer that only sees the tensors it was
given, a latency-critical loop that must not risk the device synchronisation of
cudaMalloc/cudaFree, or a memory budget fixed at start-up.  It keeps its scratch
in a fixed array inside the library.  This test calls both entry points through
the C ABI on the same inputs, twice in a row with different filter parameters
(the shared array keeps the first call's filter and spectra, which must not
leak into the second), and requires bit-identical results: both run the same
kernels on the same data.  It
also checks that a problem larger than the array is refused with a clear status
instead of being run.

The file is named to be collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from distilled_ssm_decode_b200 import ops
from distilled_ssm_decode_b200 import workloads as W

pytestmark = pytest.mark.gpu

ERR_CAPACITY = -7


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(q, k, v, lam, R, D, fft_len, y, state):
    B, L, Dch = q.shape
    H, d = lam.shape[0], lam.shape[1]
    st = ops.lib().hyena_prefill_noalloc(_p(q), _p(k), _p(v), ops.HYENA_BF16, B, L, Dch, H, d, fft_len,
                                         _p(lam), _p(R), _p(D), _p(y), _p(state),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _rel(a, b):
    a = a.detach().cpu().double().numpy()
    b = b.detach().cpu().double().numpy()
    return float(np.abs(a - b).max() / np.abs(b).max())


def test_noalloc_prefill_matches_regular_entry_point_twice():
    assert torch.cuda.is_available(), "GPU test"
    from distilled_ssm_decode_b200 import build
    build.build()
    w = W.WORKLOADS["mid_bf16"]
    for call in range(2):
        # each call has its own filter parameters (and inputs): the shared array holds the previous
        # call's filter and spectra, so if a call did not rewrite them its y would differ
        p = W.params(w, layer=call)
        lam, R, D = p.lam_f32().cuda(), p.R_f32().cuda(), p.Dskip_f32().cuda()
        need = ops.prefill_workspace_bytes(w.B, w.L, w.Dch, w.H, w.d, w.fft_len)
        assert 0 < need <= ops.lib().hyena_prefill_noalloc_capacity()
        q, k, v = (t.cuda() for t in W.prefill_inputs(w, layer=call, B=2, L=w.L, Dch=w.Dch))
        y_ref, s_ref = ops.prefill(q, k, v, lam, R, D, w.fft_len)
        y = torch.full_like(q, float("nan"))
        s = torch.full_like(s_ref, float("nan"))
        assert _noalloc(q, k, v, lam, R, D, w.fft_len, y, s) == 0
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the results are bit-identical
        assert torch.equal(y, y_ref), _rel(y, y_ref)
        assert torch.equal(s, s_ref), _rel(s, s_ref)


def test_noalloc_prefill_refuses_problems_beyond_its_scratch():
    w = W.WORKLOADS["long_prefill_bf16"]          # a 131072-point transform needs ~400 MB
    p = W.params(w)
    lam, R, D = p.lam_f32().cuda(), p.R_f32().cuda(), p.Dskip_f32().cuda()
    x = torch.zeros((1, w.L, w.Dch), dtype=torch.bfloat16, device="cuda")
    s = torch.zeros((1, w.d, w.Dch, 2), device="cuda")
    assert _noalloc(x, x, x, lam, R, D, w.fft_len, x, s) == ERR_CAPACITY
    assert "scratch" in ops.status_string(ERR_CAPACITY)
