"""Helpers for GPU-vs-oracle parity tests (marshalling only, no operator arithmetic).

Tolerances: max |gpu - oracle| <= tol * max |oracle| per output tensor, with
tol = 1e-4 for fp32 activations and 2e-2 for bf16 activations (state always
complex fp32).
"""
import numpy as np
import torch

from distilled_ssm_decode_b200 import workloads as W

TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev_params(p: W.Params, device="cuda"):
    return p.lam_f32().to(device), p.R_f32().to(device), p.Dskip_f32().to(device)


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    scale = np.abs(ref).max()
    err = np.abs(gpu - ref).max()
    return float(err / scale) if scale > 0 else float(err)


def state_c128(state: torch.Tensor) -> np.ndarray:
    """[B][d][Dch][2] float32 tensor (any device) -> complex128 numpy."""
    s = state.detach().cpu().to(torch.float64).numpy()
    return s[..., 0] + 1j * s[..., 1]


def column_params(p: W.Params, H: int, Dch: int, cols):
    """Per-column parameter stack so that column i uses head(cols[i])."""
    ch = Dch // H
    heads = [c // ch for c in cols]
    return p.lam[heads], p.R[heads], p.Dskip[heads]


def sample_columns(rng, B, Dch, n):
    bs = rng.integers(0, B, size=n)
    cs = rng.integers(0, Dch, size=n)
    return list(zip(bs.tolist(), cs.tolist()))


def gather_columns(t: torch.Tensor, bc) -> np.ndarray:
    """[B][L][Dch] CPU tensor -> float64 [1][L][len(bc)] with the listed (b, c) columns."""
    bs = torch.tensor([b for b, _ in bc])
    cs = torch.tensor([c for _, c in bc])
    return W.to_f64(t[bs, :, cs].transpose(0, 1).contiguous())[None]
