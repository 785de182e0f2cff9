"""C-ABI library checks that need no GPU.

The library must load, export every function that include/hyena.h declares,
and reject invalid arguments on the host (before any CUDA call) with the
documented status codes.  Every call below fails validation, so nothing is
enqueued and no CUDA context is created.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyena.h")

OK, ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_WS, ERR_UNSUP, ERR_CUDA = 0, -1, -2, -3, -4, -5, -6


@pytest.fixture(scope="module")
def lib():
    from distilled_ssm_decode_b200 import build, ops
    build.build()
    return ops.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hyena_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("hyena_filter_from_modes", "hyena_prefill", "hyena_decode_step",
                     "hyena_prefill_workspace_bytes", "hyena_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from distilled_ssm_decode_b200 import ops
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (hyena_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_binding_signatures_cover_every_declared_symbol():
    from distilled_ssm_decode_b200 import ops
    assert set(declared_functions()) <= set(ops.SIGNATURES)


def test_status_strings(lib):
    for s in (OK, ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_WS, ERR_UNSUP, ERR_CUDA, 12345):
        assert lib.hyena_status_string(s)
    assert lib.hyena_abi_version() >> 16 == 1


FAKE = 1 << 40   # an aligned, never-dereferenced address: every call below fails validation first


def _p(x=FAKE):
    return ctypes.c_void_p(x)


def prefill(lib, dtype=1, B=2, L=16, Dch=8, H=2, d=4, fft_len=32, ws=1 << 30, ptr=FAKE, wsptr=FAKE):
    return lib.hyena_prefill(_p(ptr), _p(ptr), _p(ptr), dtype, B, L, Dch, H, d, fft_len, _p(ptr), _p(ptr),
                             _p(ptr), _p(ptr), _p(ptr), _p(wsptr), ws, None)


def test_prefill_validation(lib):
    assert prefill(lib, dtype=7) == ERR_ARG
    assert prefill(lib, Dch=9, H=2) == ERR_SHAPE          # Dch % H
    assert prefill(lib, H=0) == ERR_SHAPE
    assert prefill(lib, d=0) == ERR_SHAPE
    assert prefill(lib, d=65) == ERR_SHAPE
    assert prefill(lib, fft_len=24) == ERR_SHAPE          # not a power of two
    assert prefill(lib, L=17, fft_len=32) == ERR_SHAPE    # < 2L-1
    assert prefill(lib, B=-1) == ERR_SHAPE
    assert prefill(lib, L=70000, fft_len=1 << 18) == ERR_UNSUP
    assert prefill(lib, ws=0) == ERR_WS
    assert prefill(lib, wsptr=FAKE + 8) == ERR_ALIGN       # workspace must be 256-byte aligned
    assert prefill(lib, ptr=FAKE + 2) == ERR_ALIGN         # bf16 pairs need 4-byte alignment
    assert prefill(lib, ptr=0) == ERR_ARG
    # empty problems are valid and enqueue nothing
    assert prefill(lib, B=0) == OK
    assert prefill(lib, Dch=0) == OK


def test_workspace_queries(lib):
    assert lib.hyena_prefill_workspace_bytes(8, 4096, 1024, 8, 16, 8192) > 0
    assert lib.hyena_prefill_workspace_bytes(8, 4096, 1024, 8, 16, 4096) == 0   # fft_len < 2L-1
    four = lib.hyena_prefill_workspace_bytes(1, 65536, 768, 12, 16, 131072)
    assert four >= 384 * 131072 * 8          # four-step planes for 384 channel pairs
    assert lib.hyena_prompt_state_workspace_bytes(1, 65536, 768, 16) > 0
    assert lib.hyena_filter_spectrum_workspace_bytes(4, 100, 256) >= 4 * 256 * 8


def test_decode_validation(lib):
    def call(dtype=1, B=4, Dch=8, H=2, d=4, ptr=FAKE, sptr=FAKE):
        return lib.hyena_decode_step(_p(ptr), _p(ptr), _p(ptr), dtype, B, Dch, H, d, _p(ptr), _p(ptr),
                                     _p(ptr), _p(sptr), _p(ptr), None)
    assert call(dtype=3) == ERR_ARG
    assert call(Dch=7, H=2) == ERR_SHAPE
    assert call(d=0) == ERR_SHAPE
    assert call(B=-2) == ERR_SHAPE
    assert call(sptr=FAKE + 4) == ERR_ALIGN
    assert call(ptr=0) == ERR_ARG
    assert call(B=0) == OK


def test_filter_and_state_validation(lib):
    assert lib.hyena_filter_from_modes(_p(), _p(), _p(), 2, 0, 10, _p(), None) == ERR_SHAPE
    assert lib.hyena_filter_from_modes(_p(), _p(), _p(), 2, 4, -1, _p(), None) == ERR_SHAPE
    assert lib.hyena_filter_from_modes(_p(0), _p(), _p(), 2, 4, 10, _p(), None) == ERR_ARG
    assert lib.hyena_filter_from_modes(_p(), _p(), _p(), 0, 4, 10, _p(), None) == OK
    assert lib.hyena_filter_spectrum(_p(), 2, 10, 100, _p(), _p(), 1 << 20, None) == ERR_SHAPE
    assert lib.hyena_filter_spectrum(_p(), 2, 10, 32, _p(), _p(), 1 << 20, None) == ERR_UNSUP
    assert lib.hyena_filter_spectrum(_p(), 2, 10, 64, _p(), _p(), 0, None) == ERR_WS
    assert lib.hyena_prompt_state(_p(), _p(), 1, 2, 10, 8, 3, 4, _p(), _p(), _p(), 1 << 20, None) == ERR_SHAPE
    assert lib.hyena_prompt_state(_p(), _p(), 1, 2, 10, 8, 2, 4, _p(), _p(), _p(), 0, None) == ERR_WS


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    """The Python binding has no fallback: a missing library is an error, not a CPU path."""
    from distilled_ssm_decode_b200 import ops
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        ops.lib()


def test_decode_layers_validation(lib):
    arr = ctypes.c_void_p * 2
    good = arr(FAKE, FAKE)
    mis = arr(FAKE + 8, FAKE)          # state pointer not 16-byte aligned

    def call(layers=2, dtype=1, B=2, Dch=8, H=2, d=4, st=good, q=good):
        return lib.hyena_decode_step_layers(layers, q, good, good, dtype, B, Dch, H, d, good, good, good,
                                            st, good, None)
    assert call(dtype=7) == ERR_ARG
    assert call(layers=-1) == ERR_SHAPE
    assert call(layers=65) == ERR_UNSUP
    assert call(Dch=9, H=3) == ERR_UNSUP       # odd channel count: no channel pairs
    assert call(Dch=6, H=2) == ERR_UNSUP       # odd channels per head
    assert call(d=0) == ERR_SHAPE
    assert call(st=mis) == ERR_ALIGN
    assert call(q=arr(FAKE + 2, FAKE)) == ERR_ALIGN
    assert call(layers=0) == OK                # nothing to do, nothing enqueued
    assert call(B=0) == OK
    assert lib.hyena_decode_step_layers(2, None, good, good, 1, 2, 8, 2, 4, good, good, good, good, good,
                                        None) == ERR_ARG


def test_fir_validation(lib):
    def step(dtype=1, B=2, Dch=8, H=2, t=3, t_max=8, ptr=FAKE):
        return lib.hyena_fir_decode_step(_p(ptr), _p(FAKE), _p(FAKE), dtype, B, Dch, H, t, t_max, _p(FAKE),
                                         _p(FAKE), _p(FAKE), None)
    assert step(dtype=7) == ERR_ARG
    assert step(t=8) == ERR_SHAPE              # t must be < t_max
    assert step(t=-1) == ERR_SHAPE
    assert step(Dch=9, H=2) == ERR_SHAPE
    assert step(B=70000) == ERR_UNSUP
    assert step(ptr=FAKE + 1) == ERR_ALIGN
    assert step(B=0) == OK
    assert lib.hyena_fir_cache_prompt(_p(), _p(), 1, 2, 9, 8, 8, _p(), None) == ERR_SHAPE   # t_max < L
    assert lib.hyena_fir_cache_prompt(_p(), _p(), 1, 2, 0, 8, 8, _p(), None) == OK          # empty prompt
    assert lib.hyena_fir_cache_prompt(_p(FAKE + 1), _p(), 1, 2, 4, 8, 8, _p(), None) == ERR_ALIGN


def test_modal_truncate_validation(lib):
    def call(H=2, d=4, k=2, ptr=FAKE, kept=FAKE):
        return lib.hyena_modal_truncate(_p(ptr), _p(FAKE), H, d, k, _p(kept), _p(FAKE), _p(FAKE), _p(FAKE),
                                        _p(FAKE), None)
    assert call(k=5) == ERR_SHAPE           # k > d
    assert call(k=-1) == ERR_SHAPE
    assert call(d=65, k=2) == ERR_SHAPE
    assert call(H=-1) == ERR_SHAPE
    assert call(ptr=FAKE + 4) == ERR_ALIGN
    assert call(kept=FAKE + 2) == ERR_ALIGN
    assert call(H=0) == OK
    assert lib.hyena_modal_truncate(_p(), _p(), 2, 4, 2, None, _p(), _p(), _p(), _p(), None) == ERR_ARG


def test_bounds_checked_build_exports_every_declared_symbol():
    """The bounds-checked variant (libhyena_b200_dbg.so, -DHYENA_DEBUG_BOUNDS) has the same ABI."""
    from distilled_ssm_decode_b200 import build
    path = build.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (hyena_\w+)", out))
    assert not [n for n in declared_functions() if n not in exported]


def test_release_build_reports_no_bounds_checks(lib):
    """hyena_debug_bounds_check answers from the host in the release build (no CUDA call)."""
    rec = (ctypes.c_longlong * 4)(7, 7, 7, 7)
    assert lib.hyena_debug_bounds_check(ctypes.cast(rec, ctypes.c_void_p)) == ERR_UNSUP
    assert tuple(rec) == (0, 0, 0, 0)
    assert lib.hyena_debug_bounds_check(None) == ERR_ARG


def test_fault_injection_hook_validates_its_arguments(lib):
    assert lib.hyena_test_chunked_inject(-2, 0.0) == ERR_ARG
    assert lib.hyena_test_chunked_inject(0, -1.0) == ERR_ARG
    assert lib.hyena_test_chunked_inject(0, 61.0) == ERR_ARG
    assert lib.hyena_test_chunked_inject(-1, 0.0) == OK


def test_fft_route_hook_and_error_offset(lib):
    assert lib.hyena_test_fft_tensor_cores(2) == ERR_ARG
    assert lib.hyena_test_fft_tensor_cores(-1) == ERR_ARG
    assert lib.hyena_test_fft_tensor_cores(0) == OK
    assert lib.hyena_test_fft_tensor_cores(1) == OK
    ws = lib.hyena_prefill_workspace_bytes(8, 4096, 1024, 8, 16, 8192)
    off = lib.hyena_prefill_error_offset(8, 4096, 1024, 8, 16, 8192)
    assert 0 < off and off + 4 <= ws and off % 4 == 0
    assert lib.hyena_prefill_error_offset(8, 4096, 1024, 8, 16, 4096) == 0    # fft_len < 2L-1


def test_route_query_follows_the_documented_rule(lib):
    BF16, F32 = 1, 0
    a = ctypes.c_void_p(1 << 20)                       # 16-byte aligned (inspected only)
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 8, 4096, 1024, 8, 16, 8192, a, a, a, a) == 1
    assert lib.hyena_prefill_uses_tensor_cores(F32, 8, 4096, 1024, 8, 16, 8192, a, a, a, a) == 0
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 8, 4096, 1020, 4, 16, 8192, a, a, a, a) == 0   # Dch % 8
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 1, 9000, 16, 2, 16, 32768, a, a, a, a) == 1    # four-step inner
    assert lib.hyena_prefill_uses_tensor_cores(F32, 1, 9000, 16, 2, 16, 32768, a, a, a, a) == 0
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 1, 900, 16, 2, 16, 2048, a, a, a, a) == 0      # too short
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 8, 4096, 1024, 8, 16, 8192, a, odd, a, a) == 0
    assert lib.hyena_prefill_uses_tensor_cores(BF16, 8, 4096, 1024, 8, 16, 4096, a, a, a, a) == ERR_SHAPE
    assert lib.hyena_prefill_uses_tensor_cores(7, 8, 4096, 1024, 8, 16, 8192, a, a, a, a) == ERR_ARG
    assert lib.hyena_test_fft_tensor_cores(0) == OK
    try:
        assert lib.hyena_prefill_uses_tensor_cores(BF16, 8, 4096, 1024, 8, 16, 8192, a, a, a, a) == 0
    finally:
        assert lib.hyena_test_fft_tensor_cores(1) == OK


def test_prefill_chunked_layers_validation(lib):
    arr = (ctypes.c_void_p * 1)(FAKE)
    call = lambda layers, dtype=1, B=2, L=64, Dch=128, H=2, d=4, ws=1 << 30: lib.hyena_prefill_chunked_layers(
        layers, arr, arr, arr, dtype, B, L, Dch, H, d, arr, arr, arr, arr, arr, _p(), ws, None)
    assert call(-1) == ERR_SHAPE
    assert call(33) == ERR_UNSUP
    assert call(1, dtype=0) == ERR_UNSUP          # fp32 activations: FFT route only
    assert call(1, Dch=64, H=2) == ERR_UNSUP      # 32 channels per head
    assert call(1, d=17) == ERR_UNSUP
    assert call(1, ws=0) == ERR_WS
    assert call(0) == OK
    assert lib.hyena_prefill_chunked_layers_workspace_bytes(33, 2, 64, 128, 2, 4) == 0
    assert lib.hyena_prefill_chunked_layers_workspace_bytes(24, 64, 512, 2048, 16, 16) > \
        lib.hyena_prefill_chunked_workspace_bytes(64, 512, 2048, 16, 16)


def test_injected_launch_failure_is_reported_before_any_cuda_call(lib):
    """A launch failure, simulated on the host (no GPU needed): valid calls of several entry points
    report HYENA_ERR_CUDA while the hook is armed, and nothing is enqueued."""
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    calls = [
        lambda: lib.hyena_decode_step(_p(), _p(), _p(), 1, 2, 8, 2, 4, _p(), _p(), _p(), _p(), _p(), None),
        lambda: prefill(lib),
        lambda: lib.hyena_prefill_chunked(_p(), _p(), _p(), 1, 2, 64, 128, 2, 4, _p(), _p(), _p(), _p(), _p(),
                                          _p(), 1 << 30, None),
        lambda: lib.hyena_prefill_chunked_layers(2, arr, arr, arr, 1, 2, 64, 128, 2, 4, arr, arr, arr, arr, arr,
                                                 _p(), 1 << 30, None),
        lambda: lib.hyena_filter_from_modes(_p(), _p(), _p(), 2, 4, 16, _p(), None),
        lambda: lib.hyena_decode_step_layers(2, arr, arr, arr, 1, 2, 8, 2, 4, arr, arr, arr, arr, arr, None),
    ]
    assert lib.hyena_test_fail_next_launches(-1) == ERR_ARG
    assert lib.hyena_test_fail_next_launches(len(calls)) == OK
    try:
        for c in calls:
            assert c() == ERR_CUDA
    finally:
        lib.hyena_test_fail_next_launches(0)
    # validation still comes first: an invalid call is reported as such and does not use up the hook
    assert lib.hyena_test_fail_next_launches(1) == OK
    try:
        assert prefill(lib, dtype=7) == ERR_ARG
    finally:
        lib.hyena_test_fail_next_launches(0)
