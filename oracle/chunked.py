"""Independent fp64 chunked form of the KDA recurrence (numpy).

TEST INFRASTRUCTURE ONLY: used to pin "chunked == recurrent" for the oracle.

The chunked algorithm is the WY/UT reparameterisation of the delta rule of
"22,580" §6.3 (chunk the sequence into blocks of C tokens; inside a chunk,
solve the C x C unit-lower-triangular system for all corrections at once;
between chunks carry the state), extended with the per-channel cumulative
decay of the gated variants ("22,580" §08 / §9.1; aidehub "Gated DeltaNet":
a value written at step i and read at step r has been scaled by the decays of
the steps after i up to r).  Per chunk, with g the inclusive cumulative sum of
log_alpha inside the chunk (per channel) and s the query scale:

  D[r,i,c] = exp(g[r,c] - g[i,c])                  (i <= r)
  A[r,i]   = beta_r sum_c k[r,c] k[i,c] D[r,i,c]     (i <  r; strictly lower)
  T        = (I + A)^{-1}                            (explicit fp64 inverse)
  W        = T (beta * (k * e^g)),  U = T (beta * v)
  u        = U - W S
  P[r,i]   = s sum_c q[r,c] k[i,c] D[r,i,c]          (i <= r)
  o        = (s q * e^g) S + P u
  S       <- Diag(e^{g_last}) S + (k * e^{g_last - g})^T u

Requires finite log_alpha (alpha > 0).
"""
from __future__ import annotations

import numpy as np


def chunk_terms(k, v, log_alpha, beta, q, scale):
    """The per-chunk matrices for one chunk (fp64).  Returns a dict."""
    n = k.shape[0]
    g = np.cumsum(log_alpha, axis=0)
    lower = np.tril(np.ones((n, n), dtype=bool))
    diff = g[:, None, :] - g[None, :, :]
    D = np.where(lower[:, :, None], np.exp(np.where(lower[:, :, None], diff, 0.0)), 0.0)
    A = np.tril(beta[:, None] * np.einsum("rc,ic,ric->ri", k, k, D), -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    eg = np.exp(g)
    W = Tm @ (beta[:, None] * (k * eg))
    U = Tm @ (beta[:, None] * v)
    P = np.tril(scale * np.einsum("rc,ic,ric->ri", q, k, D))
    return dict(g=g, A=A, T=Tm, W=W, U=U, P=P, Qt=scale * q * eg,
                Kc=k * np.exp(g[-1][None, :] - g), decay=np.exp(g[-1]))


def chunked_single(q, k, v, log_alpha, beta, S0, C, scale=None):
    """One (sequence, head): q, k, log_alpha [T, dk]; v [T, dv]; beta [T];
    S0 [dk, dv] or None.  Returns (o [T, dv], S_final [dk, dv]) in fp64."""
    q, k, v, log_alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    T, dk = q.shape
    dv = v.shape[1]
    if scale is None:
        scale = dk ** -0.5
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        m = chunk_terms(k[sl], v[sl], log_alpha[sl], beta[sl], q[sl], scale)
        u = m["U"] - m["W"] @ S
        o[sl] = m["Qt"] @ S + m["P"] @ u
        S = m["decay"][:, None] * S + m["Kc"].T @ u
    return o, S
