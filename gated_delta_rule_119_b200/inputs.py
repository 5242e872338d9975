"""Seeded synthetic inputs for the KDA (Kimi Delta Attention) workloads.

This module is shared by the fp64 oracle tests and by the CUDA path.  It holds
only the recipe for the inputs (shapes, value distributions, seeds, the fp32 ->
bf16 storage cast); none of the recurrence's arithmetic lives here.  It imports
numpy only, so the oracle tests can use it on a machine without CUDA.

Recipe (one numpy ``default_rng(seed)`` stream per workload, PCG64):

* cut points (varlen only): distinct integers drawn uniformly from [1, T-1],
  sorted, so every sequence has length >= 1;
* q, v ~ N(0, 1);  k ~ N(0, 1), then L2-normalised per (token, head) in fp32
  before the cast to the storage dtype (the keys of the delta rule are unit
  vectors, "22,580" §5.1 and the KDA bra-ket blog's preamble);
* beta = sigmoid(N(0, 1)) per (token, head);
* log_alpha = -softplus(N(0, 1)) per (token, head, channel) -- the gate form
  of "Ten questions" Q9 with a standard-normal pre-activation;
* "extremes": heads [0, H/2) draw log_alpha ~ U(-1e-3, 0) (near no-forget),
  heads [H/2, H) draw U(-6, -3) (strong forget), beta ~ U(0.95, 1);
* S0 ~ N(0, 0.02) (standard deviation 0.02) when the workload carries a state.

Gate forms of the extended entry points (``make_form_inputs``): the tensors above, then
the form's own draws from a second stream of the same seed (``default_rng([*seed, 7])``):

* "scalar" (Gated DeltaNet): log_alpha [T, H] = -softplus(N(0, 1)) per (token, head);
* "none" (DeltaNet): no gate;
* "fused": f [T, H, dk] ~ N(0, 1) in the storage dtype, A_log [H, dk] ~ U(-1, 1) and
  dt_bias [H, dk] ~ N(0, 0.5) fp32 (log alpha = -exp(A_log) softplus(f + dt_bias) is formed
  by the kernel; the per-channel decay spans a wide range, some channels forgetting several
  times faster than the default gates); with ``spread="default"`` A_log = dt_bias = 0, so the
  fused gate is -softplus(N(0, 1)), the default gates' distribution; with ``raw`` the keys
  and queries stay unnormalised N(0, 1) draws (the kernel scales them) and beta is a
  standard-normal logit (the kernel applies the sigmoid).

Values are generated in fp32 (or fp64 and then rounded to fp32), then bf16
inputs are rounded to nearest-even from that fp32 value.  The bf16 tensors are
kept as their raw uint16 bit patterns so that every consumer sees the same
bytes.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Workloads, by name; the index is the seed.
WORKLOADS = {
    "tiny_f32": dict(index=0, B=1, T=128, H=2, dk=32, dv=32, dtype="f32",
                     state=False, varlen=False, gates="default"),
    "prefill": dict(index=1, B=4, T=4096, H=16, dk=128, dv=128, dtype="bf16",
                    state=False, varlen=False, gates="default"),
    "varlen": dict(index=2, B=8, T=65536, H=32, dk=128, dv=128, dtype="bf16",
                   state=True, varlen=True, gates="default"),
    "decode": dict(index=3, B=256, T=1000, H=32, dk=128, dv=128, dtype="bf16",
                   state=True, varlen=False, gates="default"),
    "extremes": dict(index=4, B=4, T=16384, H=16, dk=128, dv=128, dtype="bf16",
                     state=False, varlen=False, gates="extremes"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def to_storage(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    raise ValueError(f"unknown dtype {dtype!r}")


def storage_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """The exact value of a stored tensor, widened to fp64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


@dataclass
class KDAInputs:
    """One batch of KDA inputs in storage form (host numpy arrays).

    Token axis is packed: q, k [T_total, H, dk]; v [T_total, H, dv];
    log_alpha [T_total, H, dk] fp32; beta [T_total, H] fp32;
    S0 [N, H, dk, dv] fp32 or None; cu_seqlens int32 [N + 1] or None (then
    the batch is B sequences of T tokens each, T_total = B * T).
    """
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    beta: np.ndarray
    S0: np.ndarray | None
    cu_seqlens: np.ndarray | None
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str
    meta: dict = field(default_factory=dict)
    form: str = "channel"           # gate form: channel | scalar | none | fused
    f: np.ndarray | None = None     # fused gate pre-activation [T_total, H, dk] (storage dtype)
    A_log: np.ndarray | None = None     # [H, dk] fp32
    dt_bias: np.ndarray | None = None   # [H, dk] fp32
    flags: int = 0                  # NORM_Q | NORM_K | BETA_LOGIT of the extended entry points

    @property
    def n_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else len(self.cu_seqlens) - 1

    @property
    def total_tokens(self) -> int:
        return self.q.shape[0]

    def offsets(self) -> np.ndarray:
        """Sequence start offsets (length n_seqs + 1) on the packed token axis."""
        if self.cu_seqlens is not None:
            return self.cu_seqlens.astype(np.int64)
        return np.arange(self.B + 1, dtype=np.int64) * self.T


def _gates(rng, shape_la, shape_b, H, kind):
    if kind == "default":
        f = rng.standard_normal(shape_la, dtype=np.float32).astype(np.float64)
        log_alpha = (-np.logaddexp(0.0, f)).astype(np.float32)
        b = rng.standard_normal(shape_b, dtype=np.float32).astype(np.float64)
        beta = (1.0 / (1.0 + np.exp(-b))).astype(np.float32)
        return log_alpha, beta
    if kind == "extremes":
        u = rng.random(shape_la, dtype=np.float32)
        log_alpha = np.empty(shape_la, dtype=np.float32)
        half = H // 2
        log_alpha[:, :half] = -1e-3 * u[:, :half]                 # U(-1e-3, 0]
        log_alpha[:, half:] = -6.0 + 3.0 * u[:, half:]            # U(-6, -3)
        beta = (0.95 + 0.05 * rng.random(shape_b, dtype=np.float32)).astype(np.float32)
        return log_alpha, beta
    raise ValueError(kind)


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str, seed,
                state: bool = False, varlen: bool = False, gates: str = "default",
                cu_seqlens=None) -> KDAInputs:
    """Generate one batch.  With ``varlen`` the B sequences are packed into T
    tokens at seeded random cut points; an explicit ``cu_seqlens`` overrides."""
    rng = np.random.default_rng(seed)
    cu = None
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens, dtype=np.int32)
        T_total = int(cu[-1])
    elif varlen:
        if B > T:
            raise ValueError("varlen needs B <= T")
        cuts = np.sort(rng.choice(np.arange(1, T), size=B - 1, replace=False)) if B > 1 \
            else np.zeros(0, dtype=np.int64)
        cu = np.concatenate([[0], cuts, [T]]).astype(np.int32)
        T_total = T
    else:
        T_total = B * T
    q = rng.standard_normal((T_total, H, dk), dtype=np.float32)
    k = rng.standard_normal((T_total, H, dk), dtype=np.float32)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True).astype(np.float32)
    v = rng.standard_normal((T_total, H, dv), dtype=np.float32)
    log_alpha, beta = _gates(rng, (T_total, H, dk), (T_total, H), H, gates)
    n = B if cu is None else len(cu) - 1
    S0 = (0.02 * rng.standard_normal((n, H, dk, dv), dtype=np.float32)).astype(np.float32) \
        if state else None
    return KDAInputs(q=to_storage(q, dtype), k=to_storage(k, dtype), v=to_storage(v, dtype),
                     log_alpha=log_alpha, beta=beta, S0=S0, cu_seqlens=cu,
                     B=B if cu is None else n, T=T if cu is None else T_total,
                     H=H, dk=dk, dv=dv, dtype=dtype, meta=dict(seed=seed, gates=gates))


def make_form_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str, seed, form: str,
                     state: bool = False, varlen: bool = False, cu_seqlens=None, raw: bool = False,
                     gates: str = "default", spread: str = "wide") -> KDAInputs:
    """One batch for a gate form of the extended entry points: the tensors of
    :func:`make_inputs`, then the form's gate from a second stream of the seed (see the
    module recipe).  ``raw`` (fused form only): unnormalised q, k and beta logits, with the flags
    that ask the kernel to normalise and squash them."""
    inp = make_inputs(B, T, H, dk, dv, dtype, seed, state=state, varlen=varlen, gates=gates,
                      cu_seqlens=cu_seqlens)
    rng = np.random.default_rng([*np.atleast_1d(np.asarray(seed, dtype=np.int64)).tolist(), 7])
    Tt = inp.total_tokens
    inp.form = form
    if form == "channel":
        return inp
    if form == "scalar":
        f = rng.standard_normal((Tt, H), dtype=np.float32).astype(np.float64)
        inp.log_alpha = (-np.logaddexp(0.0, f)).astype(np.float32)
    elif form == "none":
        inp.log_alpha = None
    elif form == "fused":
        inp.log_alpha = None
        inp.f = to_storage(rng.standard_normal((Tt, H, dk), dtype=np.float32), dtype)
        inp.A_log = rng.uniform(-1.0, 1.0, size=(H, dk)).astype(np.float32)
        inp.dt_bias = (0.5 * rng.standard_normal((H, dk))).astype(np.float32)
        if spread == "default":
            inp.A_log[:] = 0.0
            inp.dt_bias[:] = 0.0
        if raw:
            inp.q = to_storage(rng.standard_normal((Tt, H, dk), dtype=np.float32), dtype)
            inp.k = to_storage(rng.standard_normal((Tt, H, dk), dtype=np.float32), dtype)
            inp.beta = rng.standard_normal((Tt, H), dtype=np.float32)
            inp.flags = 1 | 2 | 4          # NORM_Q | NORM_K | BETA_LOGIT
    else:
        raise ValueError(f"unknown gate form {form!r}")
    return inp


def make_workload(name: str, **override) -> KDAInputs:
    """The named prefill workload at full size (``decode`` is built by
    :func:`make_decode_state` / :func:`make_decode_step`)."""
    w = dict(WORKLOADS[name])
    w.update(override)
    if name == "decode":
        raise ValueError("use make_decode_state / make_decode_step for 'decode'")
    return make_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"], w["index"],
                       state=w["state"], varlen=w["varlen"], gates=w["gates"])


def make_decode_state(N: int, H: int, dk: int, dv: int, seed) -> np.ndarray:
    """Initial recurrent state for decode, S ~ N(0, 0.02), [N, H, dk, dv] fp32."""
    rng = np.random.default_rng([seed, 1 << 30])
    return (0.02 * rng.standard_normal((N, H, dk, dv), dtype=np.float32)).astype(np.float32)


def make_decode_step(N: int, H: int, dk: int, dv: int, dtype: str, seed, step: int,
                     gates: str = "default") -> KDAInputs:
    """Inputs of one decode step (one token for each of N sequences); every
    step has its own stream so any step can be regenerated on its own."""
    rng = np.random.default_rng([seed, step])
    q = rng.standard_normal((N, H, dk), dtype=np.float32)
    k = rng.standard_normal((N, H, dk), dtype=np.float32)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True).astype(np.float32)
    v = rng.standard_normal((N, H, dv), dtype=np.float32)
    log_alpha, beta = _gates(rng, (N, H, dk), (N, H), H, gates)
    return KDAInputs(q=to_storage(q, dtype), k=to_storage(k, dtype), v=to_storage(v, dtype),
                     log_alpha=log_alpha, beta=beta, S0=None, cu_seqlens=None,
                     B=N, T=1, H=H, dk=dk, dv=dv, dtype=dtype,
                     meta=dict(seed=seed, step=step, gates=gates))


def storage_to_torch(x: np.ndarray, dtype: str, device="cpu", pin: bool = False):
    """A stored array as a torch tensor of the matching dtype (bf16 bits are
    reinterpreted, not converted)."""
    import torch
    if dtype == "bf16" and x.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    if pin:
        t = t.pin_memory()
    return t.to(device) if device != "cpu" else t


def to_torch(inp: KDAInputs, device="cuda", pin: bool = False) -> dict:
    """Upload one batch: returns q, k, v, log_alpha, beta, S0, cu_seqlens tensors.
    Fixed-length prefill batches get the [B, T, H, d] view; varlen batches and
    decode steps stay packed ([T_total, H, d] and [N, H, d])."""
    import torch
    d = {}
    for name in ("q", "k", "v"):
        d[name] = storage_to_torch(getattr(inp, name), inp.dtype, device, pin)
    d["log_alpha"] = None if inp.log_alpha is None else storage_to_torch(inp.log_alpha, "f32", device, pin)
    d["beta"] = storage_to_torch(inp.beta, "f32", device, pin)
    d["f"] = None if inp.f is None else storage_to_torch(inp.f, inp.dtype, device, pin)
    d["A_log"] = None if inp.A_log is None else storage_to_torch(inp.A_log, "f32", device, pin)
    d["dt_bias"] = None if inp.dt_bias is None else storage_to_torch(inp.dt_bias, "f32", device, pin)
    d["S0"] = None if inp.S0 is None else storage_to_torch(inp.S0, "f32", device, pin)
    d["cu_seqlens"] = None if inp.cu_seqlens is None else \
        storage_to_torch(inp.cu_seqlens.astype(np.int32), "f32", device, pin)
    if inp.cu_seqlens is None and "step" not in inp.meta:
        for name in ("q", "k", "v", "log_alpha", "beta", "f"):
            t = d[name]
            if t is not None:
                d[name] = t.view(inp.B, inp.T, *t.shape[1:])
    return d
