"""fp64 CPU oracle for the gated modal long convolution -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library never loads
it, and it shares no code with the CUDA path.

The arithmetic lives in ``hyena_oracle.c`` (plain C, IEEE double, OpenMP over
independent channels).  This module only compiles it with gcc and marshals
numpy float64 arrays into it.  Every function follows the definitions stated in
the C file's header:

* filter     h_0 = Dskip, h_j = Re sum_n R_n lambda_n^(j-1)          (modal form)
* conv       y_t = q_t * sum_{j<=t} h_{t-j} k_j v_j                   (order-2 Hyena)
* state      s_n = sum_{j<L} lambda_n^(L-1-j) k_j v_j                 (prompt -> state)
* recurrence y_t = q_t (Dskip u_t + Re sum R s), then s <- lambda s + u (O(d) decode)
* spectrum   DFT of the zero-padded filter, bins 0..N/2
* truncation keep the k modes of largest |R|/(1-|lambda|); l1 bound and direct l1/l2 tap errors

Sources: Laughing Hyena Distillery (nubint.ai review), "Proposed method" and
"Main findings"; Hyena processes long sequences 100x faster than FlashAttention
(lequren.com), "Hyena層次結構".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhyena_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) next to its source."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_filter.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _dp]
            lib.oracle_spectrum.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            _ip, ctypes.c_int, _dp]
            lib.oracle_conv_direct.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 4 + [_dp, _dp]
            lib.oracle_prompt_state.argtypes = [_dp, _dp] + [ctypes.c_int] * 5 + [_dp, _dp]
            lib.oracle_recurrent.argtypes = ([_dp, _dp, _dp] + [ctypes.c_int] * 5 +
                                             [_dp, _dp, _dp, _dp, _dp])
            lib.oracle_modal_truncate.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, _ip, _dp, _dp, _dp, _dp, _dp]
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _cplx(a) -> np.ndarray:
    """complex array [...] -> float64 [..., 2] (re, im)."""
    a = np.asarray(a)
    if np.iscomplexobj(a):
        return _f64(np.stack([a.real, a.imag], axis=-1))
    a = _f64(a)
    assert a.shape[-1] == 2
    return a


def threads() -> int:
    return int(_load().oracle_threads())


def filter_from_modes(lam, R, Dskip, L: int) -> np.ndarray:
    """h [H][L] from poles lam [H][d], residues R [H][d] (complex) and Dskip [H]."""
    lam2, R2, D = _cplx(lam), _cplx(R), _f64(Dskip)
    H, d = lam2.shape[0], lam2.shape[1]
    h = np.zeros((H, L), dtype=np.float64)
    _load().oracle_filter(_ptr(lam2), _ptr(R2), _ptr(D), H, d, L, _ptr(h))
    return h


def spectrum(h, N: int, bins=None) -> np.ndarray:
    """DFT of each head's filter zero-padded to N: complex [H][N/2+1] (or [H][len(bins)])."""
    h = _f64(h)
    H, L = h.shape
    if bins is None:
        nb = N // 2 + 1
        bp = None
    else:
        b = np.ascontiguousarray(np.asarray(bins, dtype=np.int32))
        nb = b.size
        bp = b.ctypes.data_as(_ip)
    out = np.zeros((H, nb, 2), dtype=np.float64)
    _load().oracle_spectrum(_ptr(h), H, L, N, bp, nb, _ptr(out))
    return out[..., 0] + 1j * out[..., 1]


def conv_direct(q, k, v, h, H: int) -> np.ndarray:
    """y [B][L][Dch] by the O(L^2) causal convolution with per-head filters h [H][L]."""
    q, k, v, h = _f64(q), _f64(k), _f64(v), _f64(h)
    B, L, Dch = q.shape
    assert h.shape == (H, L) and Dch % H == 0
    y = np.zeros_like(q)
    _load().oracle_conv_direct(_ptr(q), _ptr(k), _ptr(v), B, L, Dch, H, _ptr(h), _ptr(y))
    return y


def prompt_state(k, v, lam, H: int) -> np.ndarray:
    """state complex [B][d][Dch] = sum_j lam^(L-1-j) k_j v_j."""
    k, v, lam2 = _f64(k), _f64(v), _cplx(lam)
    B, L, Dch = k.shape
    d = lam2.shape[1]
    s = np.zeros((B, d, Dch, 2), dtype=np.float64)
    _load().oracle_prompt_state(_ptr(k), _ptr(v), B, L, Dch, H, d, _ptr(lam2), _ptr(s))
    return s[..., 0] + 1j * s[..., 1]


def recurrent(q, k, v, lam, R, Dskip, H: int, state=None):
    """Run T recurrent (decode) steps over q,k,v [B][T][Dch].

    Returns (y [B][T][Dch], final state complex [B][d][Dch]).  ``state`` is the
    initial state (complex [B][d][Dch]); zero when omitted.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    lam2, R2, D = _cplx(lam), _cplx(R), _f64(Dskip)
    B, T, Dch = q.shape
    d = lam2.shape[1]
    if state is None:
        s = np.zeros((B, d, Dch, 2), dtype=np.float64)
    else:
        s = _cplx(state).copy()
        assert s.shape == (B, d, Dch, 2)
    y = np.zeros_like(q)
    _load().oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), B, T, Dch, H, d,
                             _ptr(lam2), _ptr(R2), _ptr(D), _ptr(s), _ptr(y))
    return y, s[..., 0] + 1j * s[..., 1]


def decode_step(q, k, v, lam, R, Dskip, H: int, state):
    """One decode step: q,k,v [B][Dch]; returns (y [B][Dch], new state)."""
    q, k, v = (_f64(a)[:, None, :] for a in (q, k, v))
    y, s = recurrent(q, k, v, lam, R, Dskip, H, state)
    return y[:, 0, :], s


def modal_truncate(lam, R, k: int, J: int = 200000):
    """Keep the k modes of largest |R|/(1-|lambda|) per head (ties: lower index).

    Returns (kept [H][k] int, lam_out [H][k], R_out [H][k] complex, bound [H],
    err_l1 [H], err_l2 [H]): bound = sum of the dropped scores, err_* the l1 / l2 norms of
    the dropped modes' filter over taps 1..J by direct summation."""
    lam2, R2 = _cplx(lam), _cplx(R)
    H, d = lam2.shape[0], lam2.shape[1]
    assert 0 <= k <= d <= 256
    kept = np.zeros((H, max(k, 1)), dtype=np.int32)
    lo = np.zeros((H, max(k, 1), 2)); ro = np.zeros((H, max(k, 1), 2))
    b, e1, e2 = np.zeros(H), np.zeros(H), np.zeros(H)
    _load().oracle_modal_truncate(_ptr(lam2), _ptr(R2), H, d, k, J, kept.ctypes.data_as(_ip), _ptr(lo),
                                  _ptr(ro), _ptr(b), _ptr(e1), _ptr(e2))
    kept, lo, ro = kept[:, :k], lo[:, :k], ro[:, :k]
    return kept, lo[..., 0] + 1j * lo[..., 1], ro[..., 0] + 1j * ro[..., 1], b, e1, e2

