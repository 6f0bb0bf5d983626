"""CPU oracle for the sampler update around the denoiser — TEST INFRASTRUCTURE ONLY.

Plain float64 numpy restatement of one sampling step and of the step loop.  Only the
tests, the package's smoke check and the benchmark's CPU-baseline leg may import it;
the product path (the CUDA library) never does, and the two share no code.

Sources (cited by page title and section):
  [Sora-DiT]  "Sora / DiT", cv-learn.com — "방법 및 아키텍처", training-objective bullet:
              the DDPM forward process x_t = sqrt(abar_t) x_0 + sqrt(1 - abar_t) eps and
              the decoder's noise-and-covariance output (2C channels).
  [Goku]      "GOKU : Flow Based Video Generative Foundation Models", §2.3 (rectified
              flow): x_t = t x_1 + (1 - t) x_0, the network predicts the velocity that
              moves x_t toward x_1.

Readings taken where the pages are silent:
  * the epsilon step is the deterministic one implied by the forward process: the
    clean latent implied by the predicted noise is carried to the next noise level
    with the same noise (no fresh noise is drawn);
  * the noise levels abar and the rectified-flow times are the caller's (the pages
    give no schedule);
  * a learned-covariance head writes [eps | Sigma]: the step reads the first C
    channels of the C_out = 2C output;
  * the rectified-flow step is one explicit Euler step of dx/dt = v.
"""
from __future__ import annotations

from typing import Callable, Sequence

import numpy as np

F64 = np.float64
DDIM, EULER = 0, 1


def ddim_step(x_t, eps, abar_t: float, abar_next: float):
    """One deterministic step of the DDPM forward process ([Sora-DiT] training
    objective): x_0 = (x_t - sqrt(1 - abar_t) eps) / sqrt(abar_t) is the clean latent the
    predicted noise implies, and the result is that x_0 at level abar_next with the same
    noise, sqrt(abar_next) x_0 + sqrt(1 - abar_next) eps."""
    x_t = np.asarray(x_t, dtype=F64)
    eps = np.asarray(eps, dtype=F64)
    x0 = (x_t - np.sqrt(1.0 - abar_t) * eps) / np.sqrt(abar_t)
    return np.sqrt(abar_next) * x0 + np.sqrt(1.0 - abar_next) * eps


def euler_step(x, v, t: float, t_next: float):
    """One Euler step along the rectified-flow path ([Goku] §2.3): x + (t_next - t) v."""
    return np.asarray(x, dtype=F64) + (t_next - t) * np.asarray(v, dtype=F64)


def prediction(model_out, C: int):
    """The channels the step uses: the first C of the denoiser output (eps of an
    [eps | Sigma] head, or the whole velocity when C_out = C)."""
    return np.asarray(model_out, dtype=F64)[:, :C]


def step(kind: int, x, model_out, a: float, b: float):
    """x after one step of `kind` (DDIM: a, b = abar now / next; EULER: a, b = t now / next)."""
    C = np.asarray(x).shape[1]
    pred = prediction(model_out, C)
    if kind == DDIM:
        return ddim_step(x, pred, a, b)
    if kind == EULER:
        return euler_step(x, pred, a, b)
    raise ValueError("unknown sampler kind")


def sample(kind: int, model: Callable, x, model_t: Sequence[float], levels: Sequence[float]):
    """`len(model_t)` steps: at step i the denoiser sees timestep model_t[i] (the same
    for every sample), and the state moves from levels[i] to levels[i + 1]."""
    assert len(levels) == len(model_t) + 1
    x = np.asarray(x, dtype=F64)
    for i, ti in enumerate(model_t):
        x = step(kind, x, model(x, float(ti)), float(levels[i]), float(levels[i + 1]))
    return x
