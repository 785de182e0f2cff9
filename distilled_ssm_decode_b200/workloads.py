"""Seeded synthetic inputs for the gated modal long convolution.

This module only draws random numbers and rounds them to the activation dtype;
it holds none of the operator's arithmetic.  Both the CUDA path (tests, bench,
smoke) and the fp64 oracle receive the arrays drawn here, so the two sides see
bit-identical inputs.

Seeding: numpy ``PCG64`` with ``seed = 1000*workload + 17*layer + tensor_id``;
per-token decode inputs use ``SeedSequence(seed, spawn_key=(step,))`` so any
step can be drawn on its own.  Values are drawn in float64, rounded to float32
(round-to-nearest-even) and, for bf16 workloads, from float32 to bf16 (again
round-to-nearest-even; this double rounding is deterministic, which is all that
matters since both sides get the rounded arrays).

Distributions (the synthetic recipe of the five operator workloads):
  |lambda| ~ U[rmin, rmax], arg lambda ~ U[0, pi]          (poles, per head)
  R ~ CN(0, 1/d): Re, Im iid N(0, 1/(2d))                  (residues, per head)
  Dskip ~ N(0, 1)                                           (feed-through, per head)
  q, k, v ~ N(0, 1), shape [B][L][Dch]                      (activations)
  decode-only workloads: initial state Re, Im iid N(0, 1)
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

# tensor ids inside one (workload, layer) seed block
T_LAM_ABS, T_LAM_ARG, T_R, T_DSKIP, T_Q, T_K, T_V, T_STATE0, T_DQ, T_DK, T_DV = range(11)


@dataclass(frozen=True)
class Workload:
    """One synthetic operator workload (sizes named as in the operator statement)."""
    wid: int                  # seed block id (1..5)
    name: str
    B: int
    L: int                    # prompt length (0: decode only)
    Dch: int                  # channels
    H: int                    # heads (weight-tied filter per head)
    d: int                    # complex poles per head
    dtype: str                # "f32" or "bf16" activations; state is always complex fp32
    fft_len: int              # FFT length of the prefill (0: no prefill)
    T: int                    # decode steps after the prompt
    layers: int = 1           # independent operator layers
    rmin: float = 0.5
    rmax: float = 0.95
    batches: tuple = field(default_factory=tuple)   # batch sweep (decode-only workload)
    random_state0: bool = False

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def act_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload(1, "tiny_f32", B=1, L=256, Dch=64, H=4, d=8, dtype="f32",
                         fft_len=512, T=32),
    "mid_bf16": Workload(2, "mid_bf16", B=8, L=4096, Dch=1024, H=8, d=16, dtype="bf16",
                         fft_len=8192, T=256),
    "gen1p3b_bf16": Workload(3, "gen1p3b_bf16", B=64, L=512, Dch=2048, H=16, d=16,
                             dtype="bf16", fft_len=1024, T=512, layers=24),
    "long_prefill_bf16": Workload(4, "long_prefill_bf16", B=1, L=65536, Dch=768, H=12,
                                  d=16, dtype="bf16", fft_len=131072, T=0,
                                  rmin=0.9, rmax=0.999),
    "decode_sweep_bf16": Workload(5, "decode_sweep_bf16", B=1024, L=0, Dch=4096, H=32,
                                  d=16, dtype="bf16", fft_len=0, T=1024,
                                  batches=(1, 16, 64, 256, 1024), random_state0=True),
}


def _seed(w: Workload, layer: int, tensor_id: int) -> int:
    return 1000 * w.wid + 17 * layer + tensor_id


def _rng(w: Workload, layer: int, tensor_id: int, step: Optional[int] = None):
    s = _seed(w, layer, tensor_id)
    if step is None:
        return np.random.Generator(np.random.PCG64(s))
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(s, spawn_key=(step,))))


def _round_act(x64: np.ndarray, w: Workload) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x64.astype(np.float32)))
    return t if w.dtype == "f32" else t.to(torch.bfloat16)


@dataclass
class Params:
    """Per-head modal parameters, already rounded to the library's fp32 storage."""
    lam: np.ndarray       # complex128 [H][d] (values exactly representable in complex64)
    R: np.ndarray         # complex128 [H][d]
    Dskip: np.ndarray     # float64 [H]

    def lam_f32(self) -> torch.Tensor:
        """[H][d][2] float32 (re, im interleaved), the library's layout."""
        return torch.from_numpy(np.stack([self.lam.real, self.lam.imag], -1).astype(np.float32))

    def R_f32(self) -> torch.Tensor:
        return torch.from_numpy(np.stack([self.R.real, self.R.imag], -1).astype(np.float32))

    def Dskip_f32(self) -> torch.Tensor:
        return torch.from_numpy(self.Dskip.astype(np.float32))


def params(w: Workload, layer: int = 0, H: Optional[int] = None, d: Optional[int] = None) -> Params:
    H = w.H if H is None else H
    d = w.d if d is None else d
    mag = _rng(w, layer, T_LAM_ABS).uniform(w.rmin, w.rmax, size=(H, d))
    arg = _rng(w, layer, T_LAM_ARG).uniform(0.0, np.pi, size=(H, d))
    lam = (mag * np.cos(arg) + 1j * (mag * np.sin(arg))).astype(np.complex64)
    rr = _rng(w, layer, T_R).normal(0.0, np.sqrt(1.0 / (2 * d)), size=(H, d, 2))
    R = (rr[..., 0] + 1j * rr[..., 1]).astype(np.complex64)
    Dskip = _rng(w, layer, T_DSKIP).normal(0.0, 1.0, size=(H,)).astype(np.float32)
    return Params(lam.astype(np.complex128), R.astype(np.complex128), Dskip.astype(np.float64))


def prefill_inputs(w: Workload, layer: int = 0, B: Optional[int] = None,
                   L: Optional[int] = None, Dch: Optional[int] = None):
    """q, k, v as CPU tensors [B][L][Dch] in the workload's activation dtype."""
    B = w.B if B is None else B
    L = w.L if L is None else L
    Dch = w.Dch if Dch is None else Dch
    out = []
    for tid in (T_Q, T_K, T_V):
        x = _rng(w, layer, tid).standard_normal(size=(B, L, Dch))
        out.append(_round_act(x, w))
    return tuple(out)


def decode_inputs(w: Workload, step: int, layer: int = 0, B: Optional[int] = None,
                  Dch: Optional[int] = None):
    """q, k, v for one decode step as CPU tensors [B][Dch]."""
    B = w.B if B is None else B
    Dch = w.Dch if Dch is None else Dch
    out = []
    for tid in (T_DQ, T_DK, T_DV):
        x = _rng(w, layer, tid, step).standard_normal(size=(B, Dch))
        out.append(_round_act(x, w))
    return tuple(out)


def initial_state(w: Workload, B: Optional[int] = None, Dch: Optional[int] = None,
                  layer: int = 0) -> torch.Tensor:
    """Random N(0,1) complex state [B][d][Dch] as complex64 (decode-only workload)."""
    B = w.B if B is None else B
    Dch = w.Dch if Dch is None else Dch
    x = _rng(w, layer, T_STATE0).standard_normal(size=(B, w.d, Dch, 2)).astype(np.float32)
    return torch.view_as_complex(torch.from_numpy(np.ascontiguousarray(x)))


def decode_pool_device(w: Workload, pool: int, B: Optional[int] = None, device="cuda",
                       layer: int = 0):
    """`pool` distinct decode-step inputs (q, k, v), each [pool][B][Dch], drawn N(0, 1) on
    the device by torch's seeded generator.  For benchmarking large batches, where drawing
    every step on the host would take minutes; parity tests use decode_inputs()."""
    B = w.B if B is None else B
    g = torch.Generator(device=device)
    out = []
    for tid in (T_DQ, T_DK, T_DV):
        g.manual_seed(_seed(w, layer, tid))
        x = torch.randn((pool, B, w.Dch), generator=g, device=device, dtype=torch.float32)
        out.append(x.to(w.torch_dtype))
    return tuple(out)


def prefill_inputs_device(w: Workload, layer: int = 0, device="cuda"):
    """q, k, v [B][L][Dch] drawn N(0, 1) on the device by torch's seeded generator (for
    benchmarking many layers, whose host-drawn inputs would take minutes); parity tests use
    prefill_inputs()."""
    g = torch.Generator(device=device)
    out = []
    for tid in (T_Q, T_K, T_V):
        g.manual_seed(_seed(w, layer, tid))
        x = torch.randn((w.B, w.L, w.Dch), generator=g, device=device, dtype=torch.float32)
        out.append(x.to(w.torch_dtype))
    return tuple(out)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a CPU tensor (fp32 / bf16 / complex64) to numpy float64/complex128."""
    if t.is_complex():
        return t.to(torch.complex128).numpy()
    return t.to(torch.float64).numpy()
