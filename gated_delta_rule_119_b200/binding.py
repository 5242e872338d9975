"""Thin Python binding of libkda.so (ctypes).

Argument marshalling only: every step of KDA runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing, :func:`load_library` raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

KDA_F32, KDA_BF16 = 0, 1
# gate forms and flags of the _ex entry points (kda_gate_kind, kda_gate_flags)
GATE_CHANNEL, GATE_SCALAR, GATE_NONE, GATE_FUSED = 0, 1, 2, 3
NORM_Q, NORM_K, BETA_LOGIT = 1, 2, 4
STATUS = {0: "KDA_OK", -1: "KDA_ERR_NULL", -2: "KDA_ERR_DIM", -3: "KDA_ERR_CHUNK",
          -4: "KDA_ERR_ALIGN", -5: "KDA_ERR_DTYPE", -6: "KDA_ERR_ALIAS", -7: "KDA_ERR_CUDA",
          -8: "KDA_ERR_TIMEOUT", -9: "KDA_ERR_SCRATCH", -10: "KDA_ERR_GATE", -11: "KDA_ERR_INDEX"}
EXPORTS = ("kda_chunk_bwd", "kda_chunk_fwd", "kda_chunk_fwd_ex", "kda_chunk_fwd_noalloc", "kda_decode_ex",
           "kda_decode_step", "kda_device_status", "kda_selftest_wait_timeout",
           "kda_status_string")
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024   # KDA_NOALLOC_SCRATCH_BYTES

_lib = None


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kda_status_string(status)}")


def load_library(path: str | None = None):
    """Load libkda.so (built in-tree by ``gated_delta_rule_119_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libkda.so not found at {p}: build it with "
                           "`python -m gated_delta_rule_119_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    V, F, I32 = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [V, V, V, F, F, F, V, V, F] + [I32] * 7 + [V]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [V, V, V, F, F, F, V, V, F] + [I32] * 7 + [V]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [V, V, V, F, F, F, V] + [I32] * 5 + [V]
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_chunk_fwd_ex.argtypes = [V, V, V, I32, V, F, F, I32, F, F, V, V, F] + [I32] * 7 + [V]
    lib.kda_chunk_fwd_ex.restype = ctypes.c_int
    lib.kda_decode_ex.argtypes = [V, V, V, I32, V, F, F, I32, F, F, V, V] + [I32] * 7 + [V]
    lib.kda_decode_ex.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [V, V, V, I32, V, F, F, V, V, F, V, V, V, F, F, F] + [I32] * 7 + [V]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_selftest_wait_timeout.argtypes = [I32, V]
    lib.kda_selftest_wait_timeout.restype = ctypes.c_int
    lib.kda_device_status.argtypes = []
    lib.kda_device_status.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


def kda_device_status() -> int:
    """Synchronise the device; KDA_ERR_TIMEOUT (-8) if a kernel gave up a bounded
    wait since the previous call, else 0.  Clears the record."""
    return load_library().kda_device_status()


def kda_selftest_wait_timeout(limit_us: int, stream: int = 0) -> int:
    """Launch the bounded-wait self-test (one thread waits on an mbarrier nothing arrives at
    for about `limit_us` microseconds, then records a timeout).  Returns the launch status."""
    return load_library().kda_selftest_wait_timeout(int(limit_us), stream or None)


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


# ----------------------------------------------------------------- raw ABI calls
def chunk_fwd_raw(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, dk, dv,
                  C, dtype, stream) -> int:
    """Call the C entry point with integer addresses (0 = NULL)."""
    return load_library().kda_chunk_fwd(q or None, k or None, v or None, log_alpha or None,
                                        beta or None, S0 or None, cu_seqlens or None,
                                        out or None, S_final or None, B, T, H, dk, dv, C,
                                        dtype, stream or None)


def chunk_fwd_noalloc_raw(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, dk,
                          dv, C, dtype, stream) -> int:
    """kda_chunk_fwd_noalloc with integer addresses (0 = NULL)."""
    return load_library().kda_chunk_fwd_noalloc(q or None, k or None, v or None,
                                                log_alpha or None, beta or None, S0 or None,
                                                cu_seqlens or None, out or None, S_final or None,
                                                B, T, H, dk, dv, C, dtype, stream or None)


def chunk_fwd_ex_raw(q, k, v, gate_kind, gate, A_log, dt_bias, flags, beta, S0, cu_seqlens,
                     out, S_final, B, T, H, dk, dv, C, dtype, stream) -> int:
    """kda_chunk_fwd_ex with integer addresses (0 = NULL)."""
    return load_library().kda_chunk_fwd_ex(q or None, k or None, v or None, gate_kind, gate or None,
                                           A_log or None, dt_bias or None, flags, beta or None,
                                           S0 or None, cu_seqlens or None, out or None,
                                           S_final or None, B, T, H, dk, dv, C, dtype,
                                           stream or None)


def chunk_bwd_raw(q, k, v, gate_kind, gate, beta, S0, cu_seqlens, dO, dS_final, dq, dk, dv,
                  dgate, dbeta, dS0, B, T, H, dk_, dv_, C, dtype, stream) -> int:
    """kda_chunk_bwd with integer addresses (0 = NULL)."""
    return load_library().kda_chunk_bwd(q or None, k or None, v or None, gate_kind, gate or None,
                                        beta or None, S0 or None, cu_seqlens or None, dO or None,
                                        dS_final or None, dq or None, dk or None, dv or None,
                                        dgate or None, dbeta or None, dS0 or None, B, T, H, dk_,
                                        dv_, C, dtype, stream or None)


def decode_ex_raw(q, k, v, gate_kind, gate, A_log, dt_bias, flags, beta, state_pool, state_idx,
                  out, N, L, H, dk, dv, P, dtype, stream) -> int:
    """kda_decode_ex with integer addresses (0 = NULL)."""
    return load_library().kda_decode_ex(q or None, k or None, v or None, gate_kind, gate or None,
                                        A_log or None, dt_bias or None, flags, beta or None,
                                        state_pool or None, state_idx or None, out or None, N, L,
                                        H, dk, dv, P, dtype, stream or None)


def decode_step_raw(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dtype,
                    stream) -> int:
    return load_library().kda_decode_step(q or None, k or None, v or None, log_alpha or None,
                                          beta or None, S_inout or None, out or None, N, H, dk,
                                          dv, dtype, stream or None)


# ------------------------------------------------------------ torch-facing calls
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return 0 if t is None else t.data_ptr()


def _check(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def kda_chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, out=None, S_final=None,
                  *, C: int = 64, output_final_state: bool = True, stream=None):
    """Chunked KDA prefill.

    Fixed-length: q, k, log_alpha [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H].
    Varlen: q, k, log_alpha [T, H, dk] ... and ``cu_seqlens`` int32 [N + 1].
    Returns ``(out, S_final)`` (S_final is None when ``output_final_state`` is
    False and no buffer was given).
    """
    torch = _torch()
    dt = _dtype_code(q)
    if cu_seqlens is None:
        B, T, H, dk = q.shape
        N = B
    else:
        T, H, dk = q.shape
        N = cu_seqlens.numel() - 1
        B = N
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, q.dtype)
    for t, n in ((log_alpha, "log_alpha"), (beta, "beta"), (S0, "S0"), (S_final, "S_final")):
        _check(t, n, torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:-1] != q.shape[:-1] \
            or tuple(beta.shape) != tuple(q.shape[:-1]):
        raise ValueError("inconsistent q/k/v/log_alpha/beta shapes")
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if S_final is None and output_final_state:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = chunk_fwd_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                       _ptr(cu_seqlens), _ptr(out), _ptr(S_final), B, T, H, dk, dv, C, dt,
                       st.cuda_stream)
    if rc != 0:
        raise KDAError(rc, "kda_chunk_fwd")
    return out, S_final


def kda_decode_step(q, k, v, log_alpha, beta, S_inout, out=None, *, stream=None):
    """One decode step for N sequences: q, k, log_alpha [N, H, dk]; v [N, H, dv];
    beta [N, H]; S_inout [N, H, dk, dv] fp32 (updated in place).  Returns out."""
    torch = _torch()
    dt = _dtype_code(q)
    N, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, q.dtype)
    for t, n in ((log_alpha, "log_alpha"), (beta, "beta"), (S_inout, "S_inout")):
        _check(t, n, torch.float32)
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = decode_step_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S_inout),
                         _ptr(out), N, H, dk, dv, dt, st.cuda_stream)
    if rc != 0:
        raise KDAError(rc, "kda_decode_step")
    return out


def _gate_kind(gate, gate_kind):
    """The gate form: explicit, or GATE_NONE when no gate tensor is given."""
    if gate_kind is None:
        return GATE_NONE if gate is None else GATE_CHANNEL
    return gate_kind


def _flags(norm_q, norm_k, beta_logits):
    return (NORM_Q if norm_q else 0) | (NORM_K if norm_k else 0) | (BETA_LOGIT if beta_logits else 0)


def kda_chunk_fwd_ex(q, k, v, gate, beta, S0=None, cu_seqlens=None, out=None, S_final=None, *,
                     gate_kind=None, A_log=None, dt_bias=None, norm_q=False, norm_k=False,
                     beta_logits=False, C: int = 64, output_final_state: bool = True,
                     stream=None):
    """Chunked prefill of the KDA family (kda_chunk_fwd_ex).

    ``gate`` by ``gate_kind``: GATE_CHANNEL log_alpha [.., H, dk] fp32 (KDA), GATE_SCALAR
    log_alpha [.., H] fp32 (Gated DeltaNet), GATE_NONE None (DeltaNet), GATE_FUSED f [.., H,
    dk] in q's dtype with ``A_log``, ``dt_bias`` [H, dk] fp32.  ``norm_q``/``norm_k`` scale q/k
    to unit length in the kernel; ``beta_logits`` takes beta as logits.  Shapes otherwise as
    :func:`kda_chunk_fwd`.  Returns ``(out, S_final)``."""
    torch = _torch()
    dt = _dtype_code(q)
    kind = _gate_kind(gate, gate_kind)
    if cu_seqlens is None:
        B, T, H, dk = q.shape
        N = B
    else:
        T, H, dk = q.shape
        N = cu_seqlens.numel() - 1
        B = N
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, q.dtype)
    for t, n in ((beta, "beta"), (S0, "S0"), (S_final, "S_final"), (A_log, "A_log"),
                 (dt_bias, "dt_bias")):
        _check(t, n, torch.float32)
    _check(gate, "gate", q.dtype if kind == GATE_FUSED else torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    want = {GATE_CHANNEL: tuple(q.shape), GATE_FUSED: tuple(q.shape), GATE_SCALAR: tuple(q.shape[:-1])}
    if kind in want and (gate is None or tuple(gate.shape) != want[kind]):
        raise ValueError(f"gate must have shape {want[kind]} for gate_kind {kind}")
    if k.shape != q.shape or v.shape[:-1] != q.shape[:-1] or tuple(beta.shape) != tuple(q.shape[:-1]):
        raise ValueError("inconsistent q/k/v/beta shapes")
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if S_final is None and output_final_state:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = chunk_fwd_ex_raw(_ptr(q), _ptr(k), _ptr(v), kind, _ptr(gate), _ptr(A_log), _ptr(dt_bias),
                          _flags(norm_q, norm_k, beta_logits), _ptr(beta), _ptr(S0),
                          _ptr(cu_seqlens), _ptr(out), _ptr(S_final), B, T, H, dk, dv, C, dt,
                          st.cuda_stream)
    if rc != 0:
        raise KDAError(rc, "kda_chunk_fwd_ex")
    return out, S_final


def kda_decode_ex(q, k, v, gate, beta, state_pool, state_idx=None, out=None, *, gate_kind=None,
                  A_log=None, dt_bias=None, norm_q=False, norm_k=False, beta_logits=False,
                  stream=None):
    """Decode L tokens for each of N sequences from an indexed state pool (kda_decode_ex).

    q, k [N, L, H, dk]; v [N, L, H, dv]; gate as in :func:`kda_chunk_fwd_ex` with the token
    axes [N, L]; beta [N, L, H]; state_pool [P, H, dk, dv] fp32 (updated in place);
    state_idx int32 [N] or None (slot n).  Returns out [N, L, H, dv]."""
    torch = _torch()
    dt = _dtype_code(q)
    kind = _gate_kind(gate, gate_kind)
    N, L, H, dk = q.shape
    dv = v.shape[-1]
    P = state_pool.shape[0]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, q.dtype)
    for t, n in ((beta, "beta"), (state_pool, "state_pool"), (A_log, "A_log"), (dt_bias, "dt_bias")):
        _check(t, n, torch.float32)
    _check(gate, "gate", q.dtype if kind == GATE_FUSED else torch.float32)
    _check(state_idx, "state_idx", torch.int32)
    if tuple(state_pool.shape[1:]) != (H, dk, dv):
        raise ValueError("state_pool must be [P, H, dk, dv]")
    if out is None:
        out = torch.empty((N, L, H, dv), dtype=q.dtype, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = decode_ex_raw(_ptr(q), _ptr(k), _ptr(v), kind, _ptr(gate), _ptr(A_log), _ptr(dt_bias),
                       _flags(norm_q, norm_k, beta_logits), _ptr(beta), _ptr(state_pool),
                       _ptr(state_idx), _ptr(out), N, L, H, dk, dv, P, dt, st.cuda_stream)
    if rc != 0:
        raise KDAError(rc, "kda_decode_ex")
    return out


def kda_chunk_bwd(q, k, v, gate, beta, dO, S0=None, cu_seqlens=None, dS_final=None, *,
                  gate_kind=None, need_dS0=True, C: int = 64, stream=None):
    """Gradients of a prefill (kda_chunk_bwd): returns a dict with dq, dk, dv (q's dtype),
    dgate (dlog_alpha [.., H, dk] for the per-channel gate, [.., H] for the scalar gate, None
    without decay), dbeta and dS0 (fp32; None unless ``need_dS0``).  Inputs as
    :func:`kda_chunk_fwd_ex` (gate forms CHANNEL, SCALAR, NONE; no flags); dO like o."""
    torch = _torch()
    dt = _dtype_code(q)
    kind = _gate_kind(gate, gate_kind)
    if cu_seqlens is None:
        B, T, H, dk = q.shape
        N = B
    else:
        T, H, dk = q.shape
        N = cu_seqlens.numel() - 1
        B = N
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dO, "dO")):
        _check(t, n, q.dtype)
    for t, n in ((beta, "beta"), (S0, "S0"), (dS_final, "dS_final")):
        _check(t, n, torch.float32)
    _check(gate, "gate", torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dgate": None if kind == GATE_NONE else torch.empty(gate.shape, dtype=torch.float32, device=q.device),
         "dbeta": torch.empty(beta.shape, dtype=torch.float32, device=q.device),
         "dS0": torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if need_dS0 else None}
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = chunk_bwd_raw(_ptr(q), _ptr(k), _ptr(v), kind, _ptr(gate), _ptr(beta), _ptr(S0),
                       _ptr(cu_seqlens), _ptr(dO), _ptr(dS_final), _ptr(g["dq"]), _ptr(g["dk"]),
                       _ptr(g["dv"]), _ptr(g["dgate"]), _ptr(g["dbeta"]), _ptr(g["dS0"]), B, T, H,
                       dk, dv, C, dt, st.cuda_stream)
    if rc != 0:
        raise KDAError(rc, "kda_chunk_bwd")
    return g
