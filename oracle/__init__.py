"""fp64 CPU oracle for Kimi Delta Attention (KDA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library.

Routines:

* :func:`recurrent` -- the plain token-by-token definition in C (fp64,
  pthreads over (sequence, head) pairs), ``kda_oracle.c``;
* :func:`backward` -- its gradients by reverse mode, token by token in C (fp64),
  ``kda_oracle_bwd.c``; pinned by finite differences on :func:`recurrent`;
* :func:`oracle.chunked.chunked_single` -- the chunked WY/UT form in numpy fp64
  (explicit inverse of ``I + A``), used only to pin "chunked == recurrent";
* :mod:`oracle.gates` -- the gate front-ends of the fused and scalar gate forms.

Inputs may be float64, float32 or uint16 (raw bf16 bits); the C code widens
every value exactly to fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "kda_oracle.c"), os.path.join(_HERE, "kda_oracle_bwd.c")]
_SO = os.path.join(_HERE, "_kda_oracle.so")
_lib = None

# Element type codes understood by kda_oracle.c.
_DT = {np.dtype(np.float64): 0, np.dtype(np.float32): 1, np.dtype(np.uint16): 2}


def build(force: bool = False) -> str:
    """Compile the C oracle (strict IEEE fp64: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(map(os.path.getmtime, _SRCS)):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-pthread", *_SRCS, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        f = lib.kda_oracle_recurrent
        P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        f.argtypes = [P, I, P, I, P, I, P, I, P, I, P, I, P, L, L, L, L, D, P, L, P, P, I]
        f.restype = ctypes.c_int
        b = lib.kda_oracle_backward
        b.argtypes = [P, I] * 8 + [P, L, L, L, L, D, P, L, P, P, P, P, P, P, I]
        b.restype = ctypes.c_int
        _lib = lib
    return _lib


def _arr(x):
    a = np.ascontiguousarray(x)
    if a.dtype not in _DT:
        a = np.ascontiguousarray(a, dtype=np.float64)
    return a, _DT[a.dtype]


def recurrent(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, scale=None,
              tasks=None, nthreads=None):
    """Run the fp64 recurrence.

    q, k, log_alpha: [T_total, H, dk]; v: [T_total, H, dv]; beta: [T_total, H];
    S0: [N, H, dk, dv] or None (zero state); cu_seqlens: N + 1 offsets, or None
    for a single sequence of T_total tokens.  ``scale`` defaults to dk**-0.5.
    ``tasks``: iterable of (n, h) pairs (default: every pair).

    Returns ``(outs, states)``: lists in task order of o [T_n, dv] and
    S_final [dk, dv] (fp64).
    """
    lib = _load()
    qa, qd = _arr(q)
    ka, kd = _arr(k)
    va, vd = _arr(v)
    la, lad = _arr(log_alpha)
    ba, bd = _arr(beta)
    T_total, H, dk = qa.shape
    dv = va.shape[2]
    if ka.shape != qa.shape or la.shape != qa.shape or va.shape[:2] != (T_total, H) \
            or ba.shape != (T_total, H):
        raise ValueError("inconsistent shapes")
    cu = np.array([0, T_total] if cu_seqlens is None else cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    if N < 1 or cu[0] != 0 or cu[-1] != T_total or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T_total")
    if S0 is not None:
        sa, sd = _arr(S0)
        if sa.shape != (N, H, dk, dv):
            raise ValueError("S0 shape")
    else:
        sa, sd = None, 0
    if tasks is None:
        tasks = [(n, h) for n in range(N) for h in range(H)]
    tk = np.ascontiguousarray(np.array(list(tasks), dtype=np.int64).reshape(-1, 2))
    lens = cu[tk[:, 0] + 1] - cu[tk[:, 0]]
    out = np.zeros(int((lens * dv).sum()), dtype=np.float64)
    st = np.zeros(len(tk) * dk * dv, dtype=np.float64)
    if scale is None:
        scale = float(dk) ** -0.5
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = lib.kda_oracle_recurrent(
        qa.ctypes.data, qd, ka.ctypes.data, kd, va.ctypes.data, vd, la.ctypes.data, lad,
        ba.ctypes.data, bd, None if sa is None else sa.ctypes.data, sd, cu.ctypes.data, N,
        H, dk, dv, float(scale), tk.ctypes.data, len(tk), out.ctypes.data, st.ctypes.data,
        int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_recurrent rejected its arguments (rc={rc})")
    outs, states, off = [], [], 0
    for j, L in enumerate(lens):
        outs.append(out[off:off + L * dv].reshape(L, dv))
        off += L * dv
        states.append(st[j * dk * dv:(j + 1) * dk * dv].reshape(dk, dv))
    return outs, states


def recurrent_full(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, scale=None,
                   nthreads=None):
    """All pairs; returns o [T_total, H, dv] and S_final [N, H, dk, dv] (fp64)."""
    T_total, H, dk = np.shape(q)
    dv = np.shape(v)[2]
    cu = np.array([0, T_total] if cu_seqlens is None else cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    tasks = [(n, h) for n in range(N) for h in range(H)]
    outs, states = recurrent(q, k, v, log_alpha, beta, S0, cu, scale=scale, tasks=tasks,
                             nthreads=nthreads)
    o = np.zeros((T_total, H, dv))
    S = np.zeros((N, H, dk, dv))
    for (n, h), on, sn in zip(tasks, outs, states):
        o[cu[n]:cu[n + 1], h] = on
        S[n, h] = sn
    return o, S


def backward(q, k, v, log_alpha, beta, S0, cu_seqlens, dO, dS_final=None, *, scale=None,
             tasks=None, nthreads=None):
    """Gradients of L = sum(dO * o) + sum(dS_final * S_final) with respect to every input,
    by reverse mode through the fp64 recurrence.

    Shapes as :func:`recurrent`, plus dO [T_total, H, dv] and dS_final [N, H, dk, dv] (or
    None).  Returns a dict of fp64 arrays in full layout: dq, dk, dlog_alpha [T_total, H, dk],
    dv [T_total, H, dv], dbeta [T_total, H], dS0 [N, H, dk, dv] (rows of pairs outside
    ``tasks`` are zero)."""
    lib = _load()
    qa, qd = _arr(q)
    ka, kd = _arr(k)
    va, vd = _arr(v)
    la, lad = _arr(log_alpha)
    ba, bd = _arr(beta)
    oa, od = _arr(dO)
    T_total, H, dk = qa.shape
    dv = va.shape[2]
    cu = np.array([0, T_total] if cu_seqlens is None else cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    if ka.shape != qa.shape or la.shape != qa.shape or va.shape[:2] != (T_total, H) \
            or ba.shape != (T_total, H) or oa.shape != va.shape:
        raise ValueError("inconsistent shapes")
    if N < 1 or cu[0] != 0 or cu[-1] != T_total or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T_total")
    sa, sd = _arr(S0) if S0 is not None else (None, 0)
    fa, fd = _arr(dS_final) if dS_final is not None else (None, 0)
    for x in (sa, fa):
        if x is not None and x.shape != (N, H, dk, dv):
            raise ValueError("state shape")
    if tasks is None:
        tasks = [(n, h) for n in range(N) for h in range(H)]
    tk = np.ascontiguousarray(np.array(list(tasks), dtype=np.int64).reshape(-1, 2))
    out = {"dq": np.zeros((T_total, H, dk)), "dk": np.zeros((T_total, H, dk)),
           "dv": np.zeros((T_total, H, dv)), "dlog_alpha": np.zeros((T_total, H, dk)),
           "dbeta": np.zeros((T_total, H)), "dS0": np.zeros((N, H, dk, dv))}
    if scale is None:
        scale = float(dk) ** -0.5
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = lib.kda_oracle_backward(
        qa.ctypes.data, qd, ka.ctypes.data, kd, va.ctypes.data, vd, la.ctypes.data, lad,
        ba.ctypes.data, bd, None if sa is None else sa.ctypes.data, sd, oa.ctypes.data, od,
        None if fa is None else fa.ctypes.data, fd, cu.ctypes.data, N, H, dk, dv, float(scale),
        tk.ctypes.data, len(tk), out["dq"].ctypes.data, out["dk"].ctypes.data,
        out["dv"].ctypes.data, out["dlog_alpha"].ctypes.data, out["dbeta"].ctypes.data,
        out["dS0"].ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_backward rejected its arguments (rc={rc})")
    return out
