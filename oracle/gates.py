"""fp64 gate front-ends of the KDA family, for the oracle.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): nothing in the product path
imports it, and it shares no code with the CUDA library.

Each function turns what a caller of the fused or scalar-gate entry points passes into
the inputs of the plain recurrence (:func:`oracle.recurrent`): a per-channel
``log_alpha [T, H, dk]``, a write strength ``beta [T, H]`` and, when asked, unit-length
keys and queries.  All arithmetic is fp64 on the exact values the GPU receives.

* Fused per-channel decay ("Ten questions" Q9): the gate line of the open KDA
  implementation that the page reads out, g = -exp(A_log) * softplus(f + dt_bias) with
  softplus(x) = ln(1 + e^x), and alpha = e^g.  softplus is positive, so g is negative and
  alpha lies in (0, 1) whatever the network outputs.  The page fixes no shapes; here f is
  per (token, head, channel) and A_log, dt_bias per (head, channel) -- a per-head A_log
  is the special case of equal channels.
* Write strength from a logit ("Ten questions" Q9: KDA takes beta from a sigmoid;
  "22,580" §5.2 layer code): beta = 1 / (1 + e^-b).
* Key / query normalisation ("22,580" §5.2 layer code: q and k are scaled to unit length
  before the recurrence): x / max(||x||_2, eps) per (token, head), eps = 1e-12.
* Scalar gate (Gated DeltaNet, "22,580" §08): one alpha per (token, head) for every
  channel; alpha = 1 everywhere is DeltaNet ("22,580" §5-§6).  The recurrence is the same
  with the scalar repeated over the d_k channels.
"""
from __future__ import annotations

import numpy as np

NORM_EPS = 1e-12


def widen(x, dtype: str | None = None) -> np.ndarray:
    """The exact value of a stored array in fp64: uint16 arrays are raw bf16 bits."""
    a = np.asarray(x)
    if a.dtype == np.uint16 or dtype == "bf16":
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def softplus(x) -> np.ndarray:
    """ln(1 + e^x) in fp64 without overflow: max(x, 0) + ln(1 + e^-|x|)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x) -> np.ndarray:
    """1 / (1 + e^-x) in fp64, evaluated on the side that does not overflow."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def fused_log_alpha(f, A_log, dt_bias) -> np.ndarray:
    """log alpha = g = -exp(A_log) * softplus(f + dt_bias) ("Ten questions" Q9).

    f: [T, H, dk] (uint16 = bf16 bits, or float); A_log, dt_bias: [H, dk].  Returns fp64
    [T, H, dk]."""
    fx = widen(f)
    A = np.asarray(A_log, dtype=np.float64)
    b = np.asarray(dt_bias, dtype=np.float64)
    return -np.exp(A)[None] * softplus(fx + b[None])


def l2_normalize(x) -> np.ndarray:
    """x / max(||x||_2, eps) along the last axis, fp64 ("22,580" §5.2, F.normalize)."""
    xx = widen(x)
    n = np.sqrt(np.sum(xx * xx, axis=-1, keepdims=True))
    return xx / np.maximum(n, NORM_EPS)


def broadcast_scalar(log_alpha_th, dk: int) -> np.ndarray:
    """A scalar gate [T, H] (or None: no decay, DeltaNet) as the per-channel log alpha
    [T, H, dk] of the KDA recurrence, fp64."""
    la = np.asarray(log_alpha_th, dtype=np.float64)
    return np.repeat(la[..., None], dk, axis=-1)
