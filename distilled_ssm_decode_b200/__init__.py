"""B200-native gated modal long convolution (Hyena / Laughing-Hyena operator).

y = q * (h (*) (k * v)) with one weight-tied modal-SSM filter per head, in two
modes: prefill over a prompt (long convolution + gating + prompt->state
reduction) and O(1)-per-token recurrent decode.  All arithmetic runs in the
CUDA kernels of ``libhyena_b200.so`` behind a C ABI (``include/hyena.h``);
``ops`` only marshals torch tensors into that ABI.
"""
from . import workloads  # noqa: F401  (seeded synthetic inputs; no operator arithmetic)

__all__ = ["workloads", "ops"]


def __getattr__(name):
    if name in ("ops", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
