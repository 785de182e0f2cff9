"""Python binding of libhyena_b200 (argument marshalling only).

Every function here passes device pointers, sizes and the current CUDA stream
to the C ABI declared in ``include/hyena.h``; all arithmetic runs in the
library's CUDA kernels.  There is no fallback: if the shared library is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhyena_b200.so")

HYENA_F32, HYENA_BF16 = 0, 1
_DT = {torch.float32: HYENA_F32, torch.bfloat16: HYENA_BF16}

_lock = threading.Lock()
_lib = None

_vp, _fp, _i, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "hyena_status_string": (ctypes.c_char_p, [_i]),
    "hyena_abi_version": (_i, []),
    "hyena_filter_from_modes": (_i, [_fp, _fp, _fp, _i, _i, _i, _fp, _vp]),
    "hyena_filter_spectrum_workspace_bytes": (_sz, [_i, _i, _i]),
    "hyena_filter_spectrum": (_i, [_fp, _i, _i, _i, _fp, _vp, _sz, _vp]),
    "hyena_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "hyena_prefill_error_offset": (_sz, [_i, _i, _i, _i, _i, _i]),
    "hyena_prefill_uses_tensor_cores": (_i, [_i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "hyena_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp, _fp,
                           _vp, _sz, _vp]),
    "hyena_prefill_chunked_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "hyena_prefill_chunked_error_offset": (_sz, [_i, _i, _i, _i, _i]),
    "hyena_prefill_chunked": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp, _fp,
                                   _vp, _sz, _vp]),
    "hyena_prefill_chunked_layers_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "hyena_prefill_chunked_layers_error_offset": (_sz, [_i, _i, _i, _i, _i, _i]),
    "hyena_prefill_chunked_layers": (_i, [_i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _sz, _vp]),
    "hyena_prefill_noalloc_capacity": (_sz, []),
    "hyena_prefill_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp, _fp,
                                   _vp]),
    "hyena_test_chunked_inject": (_i, [_i, ctypes.c_double]),
    "hyena_test_fail_next_launches": (_i, [_i]),
    "hyena_test_fft_tensor_cores": (_i, [_i]),
    "hyena_debug_bounds_check": (_i, [_vp]),
    "hyena_prompt_state_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "hyena_prompt_state": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _fp, _fp, _vp, _sz, _vp]),
    "hyena_decode_step": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _fp, _fp, _fp, _fp, _vp, _vp]),
    "hyena_decode_step_layers": (_i, [_i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                      _vp]),
    "hyena_fir_cache_prompt": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _fp, _vp]),
    "hyena_fir_decode_step": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _fp, _fp, _vp, _vp]),
    "hyena_modal_truncate": (_i, [_fp, _fp, _i, _i, _i, _vp, _fp, _fp, _vp, _vp, _vp]),
}


class HyenaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")
        self.status = status


def _load(path: str):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{os.path.basename(path)} not found at {path}; build it with "
            "`python -m distilled_ssm_decode_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    """The loaded ctypes library (raises if the CUDA library is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = _load(LIB_PATH)
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Route every call of this module through another build of the library (for instance the
    bounds-checked libhyena_b200_dbg.so) inside the `with` block."""
    global _lib
    other = _load(path)
    with _lock:
        prev = _lib
        _lib = other
    try:
        yield other
    finally:
        with _lock:
            _lib = prev


def bounds_check():
    """Bounds-checked build only: (status, record) of the first global access out of range since
    the last check; status 0 = none, 1 = record = (file id, source line, index, extent)."""
    rec = (ctypes.c_longlong * 4)()
    st = lib().hyena_debug_bounds_check(ctypes.cast(rec, ctypes.c_void_p))
    return st, tuple(rec)


def status_string(status: int) -> str:
    return lib().hyena_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise HyenaError(fn, status)


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _params(lam, R, Dskip):
    lam = _cuda(lam, "lam", torch.float32)
    R = _cuda(R, "R", torch.float32)
    Dskip = _cuda(Dskip, "Dskip", torch.float32)
    if lam.dim() != 3 or lam.shape[-1] != 2 or R.shape != lam.shape or Dskip.shape != lam.shape[:1]:
        raise ValueError("lam, R must be [H][d][2] float32 and Dskip [H]")
    return lam, R, Dskip


def _act_dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


# ------------------------------------------------------------------ operations
def filter_from_modes(lam, R, Dskip, L: int) -> torch.Tensor:
    """h [H][L] float32: h_0 = Dskip, h_j = Re sum_n R_n lam_n^(j-1)."""
    lam, R, Dskip = _params(lam, R, Dskip)
    H, d = lam.shape[0], lam.shape[1]
    h = torch.empty((H, L), dtype=torch.float32, device=lam.device)
    _check("hyena_filter_from_modes",
           lib().hyena_filter_from_modes(_ptr(lam), _ptr(R), _ptr(Dskip), H, d, L, _ptr(h),
                                         _stream(lam.device)))
    return h


def filter_spectrum(h, fft_len: int) -> torch.Tensor:
    """complex64 [H][fft_len/2+1]: DFT of each row of h zero-padded to fft_len."""
    h = _cuda(h, "h", torch.float32)
    H, L = h.shape
    out = torch.empty((H, fft_len // 2 + 1, 2), dtype=torch.float32, device=h.device)
    nbytes = lib().hyena_filter_spectrum_workspace_bytes(H, L, fft_len)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=h.device)
    _check("hyena_filter_spectrum",
           lib().hyena_filter_spectrum(_ptr(h), H, L, fft_len, _ptr(out), _ptr(ws), nbytes,
                                       _stream(h.device)))
    return torch.view_as_complex(out)


def prefill_workspace_bytes(B, L, Dch, H, d, fft_len) -> int:
    return int(lib().hyena_prefill_workspace_bytes(B, L, Dch, H, d, fft_len))


def prefill(q, k, v, lam, R, Dskip, fft_len: int, y=None, state=None, workspace=None):
    """FFT prefill.  q,k,v [B][L][Dch] -> (y [B][L][Dch], state float32 [B][d][Dch][2])."""
    lam, R, Dskip = _params(lam, R, Dskip)
    q, k, v = _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v")
    dt = _act_dtype(q)
    B, L, Dch = q.shape
    H, d = lam.shape[0], lam.shape[1]
    if y is None:
        y = torch.empty_like(q)
    if state is None:
        state = torch.empty((B, d, Dch, 2), dtype=torch.float32, device=q.device)
    nbytes = prefill_workspace_bytes(B, L, Dch, H, d, fft_len)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _check("hyena_prefill",
           lib().hyena_prefill(_ptr(q), _ptr(k), _ptr(v), dt, B, L, Dch, H, d, fft_len,
                               _ptr(lam), _ptr(R), _ptr(Dskip), _ptr(y), _ptr(state),
                               _ptr(workspace), workspace.numel(), _stream(q.device)))
    return y, state


def prefill_chunked_workspace_bytes(B, L, Dch, H, d) -> int:
    return int(lib().hyena_prefill_chunked_workspace_bytes(B, L, Dch, H, d))


def prefill_chunked(q, k, v, lam, R, Dskip, y=None, state=None, workspace=None):
    """Chunked tensor-core prefill.  q,k,v bf16 [B][L][Dch] -> (y, state [B][d][Dch][2]).

    Returns (y, state, workspace); the int32 at chunked_error_offset() of the
    workspace is 0 after a successful run."""
    lam, R, Dskip = _params(lam, R, Dskip)
    q, k, v = _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v")
    dt = _act_dtype(q)
    B, L, Dch = q.shape
    H, d = lam.shape[0], lam.shape[1]
    if y is None:
        y = torch.empty_like(q)
    if state is None:
        state = torch.empty((B, d, Dch, 2), dtype=torch.float32, device=q.device)
    nbytes = prefill_chunked_workspace_bytes(B, L, Dch, H, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _check("hyena_prefill_chunked",
           lib().hyena_prefill_chunked(_ptr(q), _ptr(k), _ptr(v), dt, B, L, Dch, H, d, _ptr(lam),
                                       _ptr(R), _ptr(Dskip), _ptr(y), _ptr(state), _ptr(workspace),
                                       workspace.numel(), _stream(q.device)))
    return y, state, workspace


class PrefillLayerSet:
    """Host pointer arrays of a fixed set of layers for prefill_chunked_layers (built once, so that
    a call costs one library call): per layer q, k, v, y [B][L][Dch] bf16, state [B][d][Dch][2]
    float32 and the modal parameters."""

    def __init__(self, qs, ks, vs, ys, states, lams, Rs, Dskips):
        n = len(qs)
        if not all(len(x) == n for x in (ks, vs, ys, states, lams, Rs, Dskips)):
            raise ValueError("one tensor of each kind per layer")
        q0 = _cuda(qs[0], "q")
        self.dt = _act_dtype(q0)
        self.B, self.L, self.Dch = q0.shape
        ps = [_params(l, r, dk) for l, r, dk in zip(lams, Rs, Dskips)]
        self.H, self.d = ps[0][0].shape[0], ps[0][0].shape[1]
        for name, ts in (("q", qs), ("k", ks), ("v", vs), ("y", ys)):
            for t in ts:
                _cuda(t, name, q0.dtype)
                if tuple(t.shape) != (self.B, self.L, self.Dch):
                    raise ValueError(f"{name}: every layer's tensor must be [B][L][Dch]")
        for st in states:
            _cuda(st, "state", torch.float32)
        if any(p[0].shape != ps[0][0].shape for p in ps):
            raise ValueError("all layers need the same H and d")
        self.n = n
        self._keep = (list(qs), list(ks), list(vs), list(ys), list(states), ps)
        arr = ctypes.c_void_p * max(n, 1)
        self.q, self.k, self.v, self.y, self.state = (arr(*[t.data_ptr() for t in ts]) for ts in (qs, ks, vs, ys, states))
        self.lam = arr(*[p[0].data_ptr() for p in ps])
        self.R = arr(*[p[1].data_ptr() for p in ps])
        self.Dskip = arr(*[p[2].data_ptr() for p in ps])
        self.device = q0.device

    def workspace_bytes(self) -> int:
        return int(lib().hyena_prefill_chunked_layers_workspace_bytes(self.n, self.B, self.L, self.Dch, self.H, self.d))

    def error(self, workspace) -> int:
        """The kernel's error word (synchronises): 0 when every bounded wait succeeded."""
        off = int(lib().hyena_prefill_chunked_layers_error_offset(self.n, self.B, self.L, self.Dch, self.H, self.d))
        return int(workspace[off:off + 4].view(torch.int32).item())


def prefill_chunked_layers(layers: PrefillLayerSet, workspace=None):
    """Chunked prefill of every layer of the set in one launch (writes each layer's y and state).
    Returns the workspace."""
    nbytes = layers.workspace_bytes()
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=layers.device)
    _check("hyena_prefill_chunked_layers",
           lib().hyena_prefill_chunked_layers(layers.n, layers.q, layers.k, layers.v, layers.dt, layers.B, layers.L,
                                              layers.Dch, layers.H, layers.d, layers.lam, layers.R, layers.Dskip,
                                              layers.y, layers.state, _ptr(workspace), workspace.numel(),
                                              _stream(layers.device)))
    return workspace


def chunked_error(workspace, B, L, Dch, H, d) -> int:
    """The kernel's error word (synchronises): 0 when every bounded wait succeeded."""
    off = int(lib().hyena_prefill_chunked_error_offset(B, L, Dch, H, d))
    return int(workspace[off:off + 4].view(torch.int32).item())


def prefill_uses_tensor_cores(q, k, v, H: int, d: int, fft_len: int, y=None) -> bool:
    """Whether prefill(q, k, v, ...) with these tensors runs its transforms on the tensor cores."""
    B, L, Dch = q.shape
    st = lib().hyena_prefill_uses_tensor_cores(_act_dtype(q), B, L, Dch, H, d, fft_len, _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(q if y is None else y))
    if st < 0:
        _check("hyena_prefill_uses_tensor_cores", st)
    return st == 1


def prefill_error(workspace, B, L, Dch, H, d, fft_len) -> int:
    """Error word of the FFT prefill's tensor-core route (synchronises): 0 when its bounded
    waits all succeeded (and always 0 after a call that took the CUDA-core route)."""
    off = int(lib().hyena_prefill_error_offset(B, L, Dch, H, d, fft_len))
    return int(workspace[off:off + 4].view(torch.int32).item())


@contextlib.contextmanager
def fft_tensor_cores(enable: bool):
    """Test hook: inside the block every FFT prefill call runs its transforms on the tensor
    cores where that route applies (enable=True, the default outside) or on the CUDA cores
    only (enable=False)."""
    _check("hyena_test_fft_tensor_cores", lib().hyena_test_fft_tensor_cores(1 if enable else 0))
    try:
        yield
    finally:
        _check("hyena_test_fft_tensor_cores", lib().hyena_test_fft_tensor_cores(1))


def test_chunked_inject(suppress_item: int = -1, lookback_limit_s: float = 0.0):
    """Test hook: fault injection for the chunked prefill's bounded waits (see hyena.h);
    (-1, 0) restores normal operation."""
    _check("hyena_test_chunked_inject", lib().hyena_test_chunked_inject(int(suppress_item), float(lookback_limit_s)))


def prompt_state(k, v, lam, H: int, state=None):
    """state float32 [B][d][Dch][2] = sum_j lam^(L-1-j) k_j v_j (standalone reduction)."""
    lam = _cuda(lam, "lam", torch.float32)
    k, v = _cuda(k, "k"), _cuda(v, "v")
    dt = _act_dtype(k)
    B, L, Dch = k.shape
    d = lam.shape[1]
    if state is None:
        state = torch.empty((B, d, Dch, 2), dtype=torch.float32, device=k.device)
    nbytes = int(lib().hyena_prompt_state_workspace_bytes(B, L, Dch, d))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=k.device)
    _check("hyena_prompt_state",
           lib().hyena_prompt_state(_ptr(k), _ptr(v), dt, B, L, Dch, H, d, _ptr(lam), _ptr(state),
                                    _ptr(ws), ws.numel(), _stream(k.device)))
    return state


def decode_step(q, k, v, lam, R, Dskip, state, y=None):
    """One decode step: q,k,v [B][Dch]; state [B][d][Dch][2] updated in place; returns y."""
    lam, R, Dskip = _params(lam, R, Dskip)
    q, k, v = _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v")
    state = _cuda(state, "state", torch.float32)
    dt = _act_dtype(q)
    B, Dch = q.shape
    H, d = lam.shape[0], lam.shape[1]
    if y is None:
        y = torch.empty_like(q)
    _check("hyena_decode_step",
           lib().hyena_decode_step(_ptr(q), _ptr(k), _ptr(v), dt, B, Dch, H, d, _ptr(lam), _ptr(R),
                                   _ptr(Dskip), _ptr(state), _ptr(y), _stream(q.device)))
    return y


class LayerSet:
    """Host pointer arrays of a fixed set of layers for decode_step_layers (built once, reused
    every step so that a step costs one library call)."""

    def __init__(self, lams, Rs, Dskips, states):
        n = len(lams)
        if not (len(Rs) == len(Dskips) == len(states) == n):
            raise ValueError("one lam, R, Dskip and state per layer")
        ps = [_params(l, r, dk) for l, r, dk in zip(lams, Rs, Dskips)]
        self.H, self.d = ps[0][0].shape[0], ps[0][0].shape[1]
        if any(p[0].shape != ps[0][0].shape for p in ps):
            raise ValueError("all layers need the same H and d")
        self.states = [_cuda(s, "state", torch.float32) for s in states]
        self.n = n
        arr = ctypes.c_void_p * max(n, 1)
        self._keep = ps
        self.lam = arr(*[p[0].data_ptr() for p in ps])
        self.R = arr(*[p[1].data_ptr() for p in ps])
        self.Dskip = arr(*[p[2].data_ptr() for p in ps])
        self.state = arr(*[s.data_ptr() for s in self.states])


def decode_step_layers(layers: LayerSet, qs, ks, vs, ys):
    """One decode step of every layer in one launch: qs[i], ks[i], vs[i], ys[i] [B][Dch] for
    layer i; each layer's state is updated in place.  qs..ys are sequences of tensors, or
    [layers][B][Dch] tensors."""
    n = layers.n
    arr = ctypes.c_void_p * max(n, 1)
    q0 = _cuda(qs[0], "q")
    dt = _act_dtype(q0)
    B, Dch = q0.shape
    for name, ts in (("q", qs), ("k", ks), ("v", vs), ("y", ys)):
        if len(ts) != n:
            raise ValueError(f"{name}: one tensor per layer")
        for t in ts:
            _cuda(t, name, q0.dtype)
            if tuple(t.shape) != (B, Dch):
                raise ValueError(f"{name}: every layer's tensor must be [B][Dch]")
    pq, pk, pv, py = (arr(*[t.data_ptr() for t in ts]) for ts in (qs, ks, vs, ys))
    _check("hyena_decode_step_layers",
           lib().hyena_decode_step_layers(n, pq, pk, pv, dt, B, Dch, layers.H, layers.d, layers.lam,
                                          layers.R, layers.Dskip, layers.state, py,
                                          _stream(q0.device)))
    return ys


def fir_cache_prompt(k, v, t_max: int, u_cache=None):
    """History of a prompt for the undistilled baseline: u_cache float32 [B][t_max][Dch] with
    rows j < L set to k_j v_j (the rest left as they are)."""
    k, v = _cuda(k, "k"), _cuda(v, "v")
    dt = _act_dtype(k)
    B, L, Dch = k.shape
    if u_cache is None:
        u_cache = torch.zeros((B, t_max, Dch), dtype=torch.float32, device=k.device)
    _cuda(u_cache, "u_cache", torch.float32)
    _check("hyena_fir_cache_prompt",
           lib().hyena_fir_cache_prompt(_ptr(k), _ptr(v), dt, B, L, Dch, t_max, _ptr(u_cache),
                                        _stream(k.device)))
    return u_cache


def fir_decode_step(q, k, v, h, u_cache, t: int, y=None):
    """Undistilled decode of token t: y = q (sum_{j<=t} h_{t-j} u_j), history in u_cache
    [B][t_max][Dch] (row t is written); h [H][t_max] float32 taps."""
    q, k, v = _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v")
    h = _cuda(h, "h", torch.float32)
    u_cache = _cuda(u_cache, "u_cache", torch.float32)
    dt = _act_dtype(q)
    B, Dch = q.shape
    H, t_max = h.shape
    if u_cache.shape != (B, t_max, Dch):
        raise ValueError("u_cache must be [B][t_max][Dch] with t_max = h.shape[1]")
    if y is None:
        y = torch.empty_like(q)
    _check("hyena_fir_decode_step",
           lib().hyena_fir_decode_step(_ptr(q), _ptr(k), _ptr(v), dt, B, Dch, H, t, t_max, _ptr(h),
                                       _ptr(u_cache), _ptr(y), _stream(q.device)))
    return y


def modal_truncate(lam, R, k: int):
    """Keep the k modes of largest |R|/(1-|lambda|) per head.  Returns (kept int32 [H][k],
    lam_out, R_out float32 [H][k][2], bound float64 [H], err_l2 float64 [H])."""
    lam = _cuda(lam, "lam", torch.float32)
    R = _cuda(R, "R", torch.float32)
    H, d = lam.shape[0], lam.shape[1]
    dev = lam.device
    kept = torch.empty((H, k), dtype=torch.int32, device=dev)
    lo = torch.empty((H, k, 2), dtype=torch.float32, device=dev)
    ro = torch.empty((H, k, 2), dtype=torch.float32, device=dev)
    bound = torch.empty(H, dtype=torch.float64, device=dev)
    err = torch.empty(H, dtype=torch.float64, device=dev)
    nul = lambda t: _ptr(t) if k > 0 else None
    _check("hyena_modal_truncate",
           lib().hyena_modal_truncate(_ptr(lam), _ptr(R), H, d, k, nul(kept), nul(lo), nul(ro), _ptr(bound),
                                      _ptr(err), _stream(dev)))
    return kept, lo, ro, bound, err

