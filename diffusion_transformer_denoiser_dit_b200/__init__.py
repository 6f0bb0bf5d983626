"""B200-native (sm_100a) DiT denoiser forward: a C-ABI CUDA library plus a thin binding.

Everything the forward computes runs in libdit_b200.so; this package only marshals
arguments (see binding.py).  Build the library with
``python -m diffusion_transformer_denoiser_dit_b200.build``.
"""
from .binding import DiT, DitError, linear_bf16, load  # noqa: F401

__all__ = ["DiT", "DitError", "linear_bf16", "load"]
