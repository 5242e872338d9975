#!/usr/bin/env python3
"""Benchmark of the KDA hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|varlen|extremes|decode|tiny_f32]

A step is one pass of the whole hot path over one batch that is already
resident in HBM: one ``kda_chunk_fwd`` over the workload (prefill workloads),
or one ``kda_decode_step`` for all sequences (decode).  The default workload is
the chunked prefill B=4, T=4096, H=16, dk=dv=128, bf16 q/k/v, fp32 gates and
state, C=64.  Under torchrun every rank runs its own independent batch (a
different seed) on its own GPU: the path shards by (sequence, head) with no
exchange step, so there is no collective on the data path and scaling is weak.
Timing: CUDA events on the stream the kernels run on, a barrier and a device
synchronize on both sides of the timed region, the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the only reference this
project has) on a bounded sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_119_b200.inputs import (WORKLOADS, make_decode_state,  # noqa: E402
                                             make_decode_step, make_form_inputs, make_inputs,
                                             make_workload, to_torch)

METRIC = ("KDA prefill tokens/s + TFLOP/s (% roofline) at dk=dv=128; "
          "decode tokens/s, % HBM BW")
PROFILES = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = {"chunk": "gated_delta_rule_119_b200/csrc/kda_chunk_tc.cu",
                  "chunk_simt": "gated_delta_rule_119_b200/csrc/kda_chunk_simt.cuh",
                  "chunk_bwd": "gated_delta_rule_119_b200/csrc/kda_chunk_bwd.cu",
                  "decode": "gated_delta_rule_119_b200/csrc/kda_decode.cu"}


# ------------------------------------------------------------ algorithmic work
def alg_bytes_prefill(n_tok_heads: int, n_pairs: int, dk: int, dv: int, es: int,
                      s0: bool, s_final: bool) -> int:
    """Bytes the path must move: q, k, v, o in the input dtype, log_alpha and beta
    fp32, plus one read (S0) and one write (S_final) of each dk x dv fp32 state."""
    per_tok = es * (2 * dk + 2 * dv) + 4 * dk + 4
    return n_tok_heads * per_tok + n_pairs * dk * dv * 4 * (int(s0) + int(s_final))


def alg_flops_prefill(n_tok_heads: int, dk: int, dv: int, C: int = 64) -> int:
    """Three state products (6 dk dv), the two causal C x C products counted on
    their triangles (2 C (dk + dv)) and the C x C triangular solve (C^2 / 3)."""
    return n_tok_heads * (6 * dk * dv + 2 * C * (dk + dv) + C * C // 3)


def alg_bytes_decode(n_pairs: int, dk: int, dv: int, es: int, L: int = 1) -> int:
    """Per (sequence, head): the fp32 state read once and written once, and for each of the
    L tokens q, k, v, o in the input dtype, log_alpha and beta fp32."""
    return n_pairs * (2 * dk * dv * 4 + L * (es * (2 * dk + 2 * dv) + 4 * dk + 4))


def gate_bytes_per_token_head(form: str, dk: int, es: int) -> int:
    """The gate stream of one token-head: per-channel log_alpha fp32, one fp32 scalar, none,
    or the fused gate's f in the input dtype."""
    return {"channel": 4 * dk, "scalar": 4, "none": 0, "fused": es * dk}[form]


# Variants of the workloads for the extended entry points, measured in the workloads object:
# (base workload, gate form, unnormalised q/k + beta logits, decode tokens per call, indexed pool).
# The fused gate's parameters are A_log = dt_bias = 0 here, so its decay has the default gates'
# distribution and the comparison with "prefill" isolates the cost of the in-kernel front-end.
VARIANTS = {
    "prefill_fused": ("prefill", "fused", True, 1, False),
    "prefill_gdn": ("prefill", "scalar", False, 1, False),
    "prefill_bwd": ("prefill", "channel", False, 1, False),
    "decode_indexed": ("decode", "channel", False, 1, True),
    "decode_mtp4": ("decode", "channel", False, 4, True),
}
# fp32 FMA peak of the B200 from its unit counts: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def alg_flops_backward(n_tok_heads: int, dk: int, dv: int, C: int = 16) -> int:
    """The backward's state-sized products per token-head, forward recomputation included:
    r = v - (k gamma) S and the state update (4 dk dv), du's (k kappa) dS' (2 dk dv), the previous
    chunk's dS (4 dk dv), d(s q gamma), d(k gamma), d(k kappa) (6 dk dv) and d gamma_last (dk dv);
    plus the C x C products of the chunk (8 C (dk + dv))."""
    return n_tok_heads * (17 * dk * dv + 8 * C * (dk + dv))


# ----------------------------------------------------------- distributed plumbing
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch: weak scaling over independent problems."""
    return base if rank == 0 else base * 1000 + rank


def reduce_max(x: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clock sampler
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every `period` s."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.error = str(e)
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                break
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        return False

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "NVML, every 10 ms during the timed region",
                **({"error": self.error} if self.error else {})}


# --------------------------------------------------------------- profile lookup
def source_digest(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel_key: str, workload: str):
    """DRAM bytes per call recorded in a committed ncu summary (for the tensor-core
    prefill: both of its kernels, read + write), or None when there is none or the
    kernel source changed since it was taken."""
    stem = os.path.splitext(os.path.basename(KERNEL_SOURCES[kernel_key]))[0]
    path = os.path.join(PROFILES, f"{stem}__{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != source_digest(KERNEL_SOURCES[kernel_key]):
        return None
    return float(m.group(1))


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), recorded beside the oracle's core count."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- CPU baseline
PARITY_BAR = {"bf16": 2e-2, "f32": 1e-4}


def _rel(x, r) -> float:
    x, r = np.asarray(x, dtype=np.float64), np.asarray(r, dtype=np.float64)
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def sample_parity(tasks, outs, states, gpu_pair, dtype: str) -> dict:
    """Max relative error, max|x - r| / max|r|, of the GPU's o and final states against the
    oracle's results for the same (sequence, head) pairs, pooled over the pairs and for the
    worst pair on its own.  gpu_pair(n, h) -> (o [len, dv], S [dk, dv]).  A failure to read
    the GPU's result is reported in place of the numbers; it never stops the bench."""
    try:
        go, ro, gs, rs, po, ps = [], [], [], [], [], []
        for (n, h), o_ref, s_ref in zip(tasks, outs, states):
            o_gpu, s_gpu = gpu_pair(n, h)
            if np.size(o_ref):
                go.append(np.asarray(o_gpu, dtype=np.float64).ravel())
                ro.append(np.asarray(o_ref, dtype=np.float64).ravel())
                po.append(_rel(o_gpu, o_ref))
            gs.append(np.asarray(s_gpu, dtype=np.float64).ravel())
            rs.append(np.asarray(s_ref, dtype=np.float64).ravel())
            ps.append(_rel(s_gpu, s_ref))
        eo = _rel(np.concatenate(go), np.concatenate(ro))
        es = _rel(np.concatenate(gs), np.concatenate(rs))
        bar = PARITY_BAR[dtype]
        return {"o_max_rel_err": eo, "S_final_max_rel_err": es,
                "o_worst_pair_rel_err": max(po), "S_final_worst_pair_rel_err": max(ps),
                "bar": bar, "pass": bool(max(eo, es, max(po), max(ps)) <= bar),
                "pairs": len(tasks), "against": "fp64 oracle, same (sequence, head) pairs"}
    except Exception as e:  # noqa: BLE001 - reported in the line instead
        return {"error": repr(e)[:300]}


def cpu_baseline(inp, budget_s: float = 12.0, gpu_pair=None):
    """The fp64 oracle as it stands, on a bounded sample of (sequence, head)
    pairs of the same workload, all host cores.  Tokens/s = token-heads / H / s.
    With ``gpu_pair`` the GPU's results for the sampled pairs are checked against
    the oracle's (``parity``)."""
    import oracle
    cores = os.cpu_count() or 1
    cu = inp.offsets()
    lens = np.diff(cu)
    order = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H) if lens[n] > 0]
    rng = np.random.default_rng(0)
    rng.shuffle(order)
    t = time.perf_counter()
    oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu,
                     tasks=order[:1], nthreads=1)
    one = max(time.perf_counter() - t, 1e-6) / max(1, lens[order[0][0]])
    # pairs that keep every core busy for about budget_s
    per_pair = one * float(np.mean(lens))
    n_pairs = int(max(1, min(len(order), round(budget_s * cores / per_pair))))
    tasks = order[:n_pairs]
    threads = min(cores, n_pairs)
    t = time.perf_counter()
    outs, states = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu,
                                    tasks=tasks, nthreads=threads)
    dt = time.perf_counter() - t
    tok_heads = int(sum(lens[n] for n, _ in tasks))
    res = {"value": tok_heads / inp.H / dt, "unit": "tokens/s", "cores": threads, "cpu_model": cpu_model(),
           "kind": "oracle", "seconds": round(dt, 3),
           "sample": f"{n_pairs} of {inp.n_seqs * inp.H} (sequence, head) pairs, "
                     f"{tok_heads} token-heads, fp64 recurrence, {threads} threads"}
    if gpu_pair is not None:
        res["parity"] = sample_parity(tasks, outs, states, gpu_pair, inp.dtype)
    return res


def oracle_view(inp):
    """The batch as the oracle reads it for a gate form of the extended entry points: the
    oracle's own gate front-end (oracle/gates.py) applied to the bytes the GPU receives --
    per-channel log alpha, beta after the sigmoid, unit-length q and k where the flags ask."""
    import dataclasses
    from oracle import gates
    q, k, beta = inp.q, inp.k, inp.beta
    if inp.form == "scalar":
        la = gates.broadcast_scalar(inp.log_alpha, inp.dk)
    elif inp.form == "none":
        la = np.zeros(inp.q.shape)
    elif inp.form == "fused":
        la = gates.fused_log_alpha(inp.f, inp.A_log, inp.dt_bias)
    else:
        la = inp.log_alpha
    if inp.flags & 1:
        q = gates.l2_normalize(q)
    if inp.flags & 2:
        k = gates.l2_normalize(k)
    if inp.flags & 4:
        beta = gates.sigmoid(beta)
    return dataclasses.replace(inp, q=q, k=k, log_alpha=la, beta=beta)


def cpu_baseline_backward(inp, dO, dSf, holder, budget_s):
    """The fp64 reverse-mode oracle on a bounded sample of (sequence, head) pairs of a backward
    workload; parity of every gradient of the GPU's last call (holder["g"]) against it, the
    worst over the gradients and pairs."""
    import oracle
    import torch
    cores = os.cpu_count() or 1
    cu = inp.offsets()
    lens = np.diff(cu)
    order = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H) if lens[n] > 0]
    t = time.perf_counter()
    oracle.backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu, dO, dSf,
                    tasks=order[:1], nthreads=1)
    per_pair = max(time.perf_counter() - t, 1e-6)
    n_pairs = int(max(1, min(len(order), round(budget_s * cores / per_pair))))
    threads = min(cores, n_pairs)
    t = time.perf_counter()
    r = oracle.backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu, dO, dSf,
                        tasks=order[:n_pairs], nthreads=threads)
    dt = time.perf_counter() - t
    res = {"value": sum(int(lens[n]) for n, _ in order[:n_pairs]) / inp.H / dt, "unit": "tokens/s",
           "cores": threads, "cpu_model": cpu_model(), "kind": "oracle", "seconds": round(dt, 3),
           "sample": f"{n_pairs} of {inp.n_seqs * inp.H} (sequence, head) pairs, fp64 reverse mode, "
                     f"{threads} threads"}
    try:
        g = holder["g"]
        torch.cuda.synchronize()
        T, H = inp.total_tokens, inp.H
        gpu = {"dq": g["dq"].float().cpu().numpy().reshape(T, H, -1),
               "dk": g["dk"].float().cpu().numpy().reshape(T, H, -1),
               "dv": g["dv"].float().cpu().numpy().reshape(T, H, -1),
               "dlog_alpha": g["dgate"].cpu().numpy().reshape(T, H, -1),
               "dbeta": g["dbeta"].cpu().numpy().reshape(T, H), "dS0": g["dS0"].cpu().numpy()}
        worst, bar = {}, PARITY_BAR[inp.dtype]
        for name, ref in r.items():
            errs = []
            for n, h in order[:n_pairs]:
                x = gpu[name][n, h] if name == "dS0" else gpu[name][cu[n]:cu[n + 1], h]
                y = ref[n, h] if name == "dS0" else ref[cu[n]:cu[n + 1], h]
                errs.append(_rel(x, y))
            worst[name] = max(errs)
        res["parity"] = {"worst_pair_rel_err": worst, "bar": bar, "pass": bool(max(worst.values()) <= bar),
                         "pairs": n_pairs, "against": "fp64 reverse-mode oracle, same pairs"}
    except Exception as e:  # noqa: BLE001 - reported in the line instead
        res["parity"] = {"error": repr(e)[:300]}
    return res


def cpu_baseline_decode_ex(ins, S0, L, budget_s, gpu_pair):
    """The oracle over the first calls of a decode variant (L tokens per sequence per call,
    ins[j] packed sequence-major [N * L, H, .]) from each sequence's initial state S0 [N, H,
    dk, dv], on a bounded sample of (sequence, head) pairs; parity against gpu_pair."""
    import oracle
    cores = os.cpu_count() or 1
    views = [oracle_view(i) for i in ins]
    N, H = ins[0].n_seqs, ins[0].H
    calls = len(views)

    def stack(name):
        xs = [np.asarray(getattr(v, name)) for v in views]
        return np.stack([x.reshape(N, L, *x.shape[1:]) for x in xs], 1).reshape(N * calls * L, *xs[0].shape[1:])
    arrs = [stack(x) for x in ("q", "k", "v", "log_alpha", "beta")]
    cu = np.arange(N + 1) * calls * L
    order = [(n, h) for n in range(N) for h in range(H)]
    t = time.perf_counter()
    oracle.recurrent(*arrs, S0, cu, tasks=order[:1], nthreads=1)
    per_pair = max(time.perf_counter() - t, 1e-6)
    n_pairs = int(max(1, min(len(order), round(budget_s * cores / per_pair))))
    threads = min(cores, n_pairs)
    t = time.perf_counter()
    outs, states = oracle.recurrent(*arrs, S0, cu, tasks=order[:n_pairs], nthreads=threads)
    dt = time.perf_counter() - t
    res = {"value": n_pairs * calls * L / H / dt, "unit": "tokens/s", "cores": threads, "cpu_model": cpu_model(), "kind": "oracle",
           "seconds": round(dt, 3),
           "sample": f"{n_pairs} of {N * H} (sequence, head) states x {calls} calls of {L} tokens, "
                     f"fp64 recurrence, {threads} threads"}
    res["parity"] = sample_parity(order[:n_pairs], outs, states, gpu_pair, ins[0].dtype)
    return res


def cpu_baseline_decode(ins, S0, budget_s: float = 12.0, gpu_pair=None):
    """The fp64 oracle over the first steps of the decode workload from its initial state,
    on a bounded sample of (sequence, head) states; ``gpu_pair`` as in cpu_baseline, the
    GPU's o for those steps and its state after them."""
    import oracle
    cores = os.cpu_count() or 1
    N, H = ins[0].q.shape[0], ins[0].q.shape[1]
    steps = len(ins)
    stack = lambda name: np.stack([getattr(i, name) for i in ins], axis=1).reshape(
        N * steps, *getattr(ins[0], name).shape[1:])
    cu = np.arange(N + 1) * steps
    arrs = [stack(x) for x in ("q", "k", "v", "log_alpha", "beta")]
    order = [(n, h) for n in range(N) for h in range(H)]
    t = time.perf_counter()
    oracle.recurrent(*arrs, S0, cu, tasks=order[:1], nthreads=1)
    per_pair = max(time.perf_counter() - t, 1e-6)
    n_pairs = int(max(1, min(len(order), round(budget_s * cores / per_pair))))
    threads = min(cores, n_pairs)
    t = time.perf_counter()
    outs, states = oracle.recurrent(*arrs, S0, cu, tasks=order[:n_pairs], nthreads=threads)
    dt = time.perf_counter() - t
    # a decode token is one sequence's step over all H heads
    res = {"value": n_pairs * steps / H / dt, "unit": "tokens/s", "cores": threads, "cpu_model": cpu_model(),
           "kind": "oracle", "seconds": round(dt, 3),
           "sample": f"{n_pairs} of {N * H} (sequence, head) states x {steps} steps, "
                     f"fp64 recurrence, {threads} threads"}
    if gpu_pair is not None:
        res["parity"] = sample_parity(order[:n_pairs], outs, states, gpu_pair, ins[0].dtype)
    return res


# -------------------------------------------------------------------- the runs
def workload_config(name, inp_or_dims, n_gpus):
    w = WORKLOADS[name]
    cfg = {"workload": name, "B": w["B"], "T": w["T"], "H": w["H"], "dk": w["dk"],
           "dv": w["dv"], "chunk": 64, "dtype": w["dtype"], "state_in": w["state"],
           "varlen": w["varlen"], "gates": w["gates"],
           "global_batch": w["B"] * n_gpus, "seq_len": w["T"],
           "parallelism": f"dp{n_gpus}: independent batches per rank, no collective"}
    return cfg


def setup_workload(name, args, device, rank):
    """Inputs of one workload resident on the device and the step that runs it.  Returns a
    dict: step(i), units per step (tokens), algorithmic bytes and FLOPs per step, the
    kernel key, kernel launches per step, and parity(budget_s) -> the oracle's CPU baseline
    on a bounded sample with the GPU's results for the same pairs checked against it."""
    import torch
    from gated_delta_rule_119_b200 import kda_chunk_fwd, kda_decode_step
    if name in VARIANTS:
        return setup_variant(name, args, device, rank)
    w = WORKLOADS[name]
    es = 2 if w["dtype"] == "bf16" else 4
    if name == "decode":
        N, H, dk, dv = w["B"], w["H"], w["dk"], w["dv"]
        n_in = max(1, min(args.decode_inputs, args.steps + args.warmup))
        ins = [make_decode_step(N, H, dk, dv, w["dtype"], rank_seed(w["index"], rank), t)
               for t in range(n_in)]
        S0 = make_decode_state(N, H, dk, dv, rank_seed(w["index"], rank))
        dev_in = [to_torch(i, device) for i in ins]
        S = torch.from_numpy(S0).to(device)
        out = torch.empty((N, H, dv), dtype=dev_in[0]["q"].dtype, device=device)

        def step(i):
            d = dev_in[i % n_in]
            kda_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S, out)

        def parity(budget):
            n_chk = min(4, len(ins))
            try:
                pairs = decode_pairs(dev_in[:n_chk], S0, device, kda_decode_step)
            except Exception as e:  # noqa: BLE001 - reported by the parity entry instead
                def pairs(n, hh, err=repr(e)):
                    raise RuntimeError(err)
            return cpu_baseline_decode(ins[:n_chk], S0, budget, pairs)
        return dict(step=step, units=N, bytes=alg_bytes_decode(N * H, dk, dv, es),
                    flops=N * H * 7 * dk * dv, kernel_key="decode", launches=1, parity=parity,
                    hold=(dev_in, S, out))
    inp = make_workload(name) if rank == 0 else make_inputs(
        w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"], rank_seed(w["index"], rank),
        state=w["state"], varlen=w["varlen"], gates=w["gates"])
    d = to_torch(inp, device)
    out = torch.empty(d["v"].shape, dtype=d["q"].dtype, device=device)
    Sf = torch.empty((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=torch.float32, device=device)

    def step(i):
        kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                      d["cu_seqlens"], out, Sf)

    def parity(budget):
        return cpu_baseline(inp, budget, prefill_pairs(out, Sf, inp))
    tok_heads = inp.total_tokens * inp.H
    tc = w["dtype"] == "bf16" and w["dk"] == 128 and w["dv"] == 128
    return dict(step=step, units=inp.total_tokens,
                bytes=alg_bytes_prefill(tok_heads, inp.n_seqs * inp.H, inp.dk, inp.dv, es,
                                        inp.S0 is not None, True),
                flops=alg_flops_prefill(tok_heads, inp.dk, inp.dv),
                kernel_key="chunk" if tc else "chunk_simt",
                # intra-chunk kernel + scan kernel, plus the slot-offset kernel for varlen
                launches=(2 + (inp.cu_seqlens is not None)) if tc else 1,
                parity=parity, hold=(d, out, Sf))


def setup_variant(name, args, device, rank):
    """A VARIANTS entry: the base workload's shapes through kda_chunk_fwd_ex / kda_decode_ex,
    in the same dict form as setup_workload."""
    import torch
    from gated_delta_rule_119_b200 import kda_chunk_fwd_ex, kda_decode_ex
    base, form, raw, L, indexed = VARIANTS[name]
    w = WORKLOADS[base]
    es = 2 if w["dtype"] == "bf16" else 4
    kind = {"channel": 0, "scalar": 1, "none": 2, "fused": 3}[form]
    flags = dict(norm_q=raw, norm_k=raw, beta_logits=raw)
    if base == "decode":
        N, H, dk, dv = w["B"], w["H"], w["dk"], w["dv"]
        n_in = max(1, min(args.decode_inputs // L, args.steps + args.warmup))
        ins = [make_form_inputs(N, L, H, dk, dv, w["dtype"], (rank_seed(w["index"], rank), t), form,
                                raw=raw) for t in range(n_in)]
        pool0 = make_decode_state(N, H, dk, dv, rank_seed(w["index"], rank))
        perm = np.random.default_rng(11).permutation(N).astype(np.int32) if indexed else None
        dev_in = [to_torch(i, device) for i in ins]
        pool = torch.from_numpy(pool0).to(device)
        idx = torch.from_numpy(perm).to(device) if indexed else None
        out = torch.empty((N, L, H, dv), dtype=dev_in[0]["q"].dtype, device=device)

        def call(d, pool_, out_):
            gate = d["f"] if form == "fused" else d["log_alpha"]
            kda_decode_ex(d["q"], d["k"], d["v"], gate, d["beta"], pool_, idx, out_, gate_kind=kind,
                          A_log=d["A_log"], dt_bias=d["dt_bias"], **flags)

        def step(i):
            call(dev_in[i % n_in], pool, out)

        def parity(budget):
            n_chk = min(2, n_in)
            chk = torch.from_numpy(pool0).to(device)
            outs = []
            for d in dev_in[:n_chk]:
                o_ = torch.empty_like(out)
                call(d, chk, o_)
                outs.append(o_)
            torch.cuda.synchronize(device)
            slot = perm if indexed else np.arange(N)

            def gpu_pair(n, hh):
                o = torch.cat([o_[n, :, hh] for o_ in outs]).float().cpu().numpy()
                return o, chk[int(slot[n]), hh].cpu().numpy()
            return cpu_baseline_decode_ex(ins[:n_chk], pool0[slot], L, budget, gpu_pair)
        per_pair = 2 * dk * dv * 4 + L * (es * (2 * dk + 2 * dv) + gate_bytes_per_token_head(form, dk, es) + 4)
        return dict(step=step, units=N * L, bytes=N * H * per_pair + (4 * N if indexed else 0),
                    flops=N * L * H * 7 * dk * dv, kernel_key="decode", launches=1, parity=parity,
                    hold=(dev_in, pool, out))
    inp = make_form_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"], rank_seed(w["index"], rank),
                           form, state=w["state"], varlen=w["varlen"], raw=raw, gates=w["gates"],
                           spread="default")
    d = to_torch(inp, device)
    if name == "prefill_bwd":
        return setup_backward(inp, d, device)
    out = torch.empty(d["v"].shape, dtype=d["q"].dtype, device=device)
    Sf = torch.empty((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=torch.float32, device=device)
    gate = d["f"] if form == "fused" else d["log_alpha"]

    def step(i):
        kda_chunk_fwd_ex(d["q"], d["k"], d["v"], gate, d["beta"], d["S0"], d["cu_seqlens"], out, Sf,
                         gate_kind=kind, A_log=d["A_log"], dt_bias=d["dt_bias"], **flags)

    def parity(budget):
        return cpu_baseline(oracle_view(inp), budget, prefill_pairs(out, Sf, inp))
    tok_heads = inp.total_tokens * inp.H
    per_tok = es * (2 * inp.dk + 2 * inp.dv) + gate_bytes_per_token_head(form, inp.dk, es) + 4
    states = inp.n_seqs * inp.H * inp.dk * inp.dv * 4 * ((inp.S0 is not None) + 1)
    params = 2 * inp.H * inp.dk * 4 if form == "fused" else 0
    return dict(step=step, units=inp.total_tokens, bytes=tok_heads * per_tok + states + params,
                flops=alg_flops_prefill(tok_heads, inp.dk, inp.dv), kernel_key="chunk",
                launches=2 + (inp.cu_seqlens is not None), parity=parity, hold=(d, out, Sf))


def setup_backward(inp, d, device):
    """The backward pass (kda_chunk_bwd) on a prefill workload: dO and dS_final drawn from
    N(0, 1); parity of every gradient on a bounded oracle sample."""
    import torch
    from gated_delta_rule_119_b200 import kda_chunk_bwd
    rng = np.random.default_rng([int(inp.meta["seed"]) if np.ndim(inp.meta["seed"]) == 0 else 0, 99])
    dO = rng.standard_normal((inp.total_tokens, inp.H, inp.dv), dtype=np.float32)
    dO_t = torch.from_numpy(dO).to(device).to(d["q"].dtype).view(d["v"].shape)
    dO_bits = dO_t.view(-1).view(torch.int16).cpu().numpy().view(np.uint16).reshape(dO.shape) \
        if inp.dtype == "bf16" else dO
    dSf = rng.standard_normal((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=np.float32)
    dSf_t = torch.from_numpy(dSf).to(device)
    holder = {}

    def step(i):
        holder["g"] = kda_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dO_t, d["S0"],
                                    d["cu_seqlens"], dSf_t)

    def parity(budget):
        return cpu_baseline_backward(inp, dO_bits, dSf, holder, budget)
    tok_heads = inp.total_tokens * inp.H
    es = 2 if inp.dtype == "bf16" else 4
    # read q, k, v, log_alpha, beta, dO (+ dS_final, S0); write dq, dk, dv, dlog_alpha, dbeta, dS0
    per_tok = es * (3 * inp.dk + 2 * inp.dv) + es * (2 * inp.dk + inp.dv) + 2 * 4 * inp.dk + 2 * 4
    states = inp.n_seqs * inp.H * inp.dk * inp.dv * 4 * (2 + (inp.S0 is not None))
    return dict(step=step, units=inp.total_tokens, bytes=tok_heads * per_tok + states,
                flops=alg_flops_backward(tok_heads, inp.dk, inp.dv), kernel_key="chunk_bwd",
                launches=2, parity=parity, hold=(d, dO_t, dSf_t, holder), bound="alu")


def time_steps(step, steps, warmup, device, stream, min_timed_s=1.0, min_passes=5,
               max_passes=200, sampler=None):
    """W untimed warm-up steps, then passes of exactly `steps` timed steps, each pass
    bracketed by CUDA events on the launching stream with a synchronize after it; at least
    `min_passes` passes and until about `min_timed_s` of timed work.  A barrier and a device
    synchronize stand on both sides of the timed region.  Returns ms per step of each pass."""
    import torch
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    passes = []
    with (sampler if sampler is not None else _NullCtx()):
        while True:
            ev0.record(stream)
            for i in range(steps):
                step(warmup + i)
            ev1.record(stream)
            torch.cuda.synchronize(device)
            passes.append(ev0.elapsed_time(ev1) / steps)
            done_s = sum(passes) * steps / 1e3
            if len(passes) >= max_passes or (len(passes) >= min_passes and done_s >= min_timed_s):
                break
    barrier(device)
    torch.cuda.synchronize(device)
    return passes


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def launch_duration_ms(step, n, device, stream):
    """Mean duration of one call, CUDA events around each call on the launching stream.
    For the tensor-core prefill a call is its kernels back to back (intra-chunk, then
    scan); the roofline is taken over the call because the algorithmic bytes (q, k, v,
    gates in; o and states out) belong to the pair, not to either kernel alone."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        step(i)
        b.record(stream)
    torch.cuda.synchronize(device)
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def roofline_entry(wl, launch_ms, hbm, peak_kind, name):
    if wl.get("bound") == "alu":
        achieved = wl["flops"] / (launch_ms / 1e3) / 1e12
        return {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_PEAK_TFLOPS, "traffic": profiled_traffic(wl["kernel_key"], name),
                "peak_kind": "fp32 FMA peak from the unit counts (148 SMs x 128 lanes x 2 x 1.965 GHz)",
                "kernel": "kda_chunk_bwd_kernel + kda_chunk_bwd_reduce_kernel (one kda_chunk_bwd call)",
                "alg_flops_per_launch": wl["flops"], "alg_bytes_per_launch": wl["bytes"],
                "hbm_frac": wl["bytes"] / (launch_ms / 1e3) / 1e9 / hbm, "launch_ms": launch_ms}
    achieved = wl["bytes"] / (launch_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": profiled_traffic(wl["kernel_key"], name),
            "peak_kind": f"{peak_kind} (STREAM-style copy, burst)",
            "kernel": {"chunk": "kda_chunk_intra_kernel + kda_chunk_scan_kernel "
                                "(one kda_chunk_fwd call)",
                       "chunk_simt": "kda_chunk_simt_kernel",
                       "decode": "kda_decode_step_kernel (one token, per-channel gate) / "
                                 "kda_decode_single_kernel (one token, other forms) / "
                                 "kda_decode_kernel (L tokens)"}[wl["kernel_key"]],
            "alg_bytes_per_launch": wl["bytes"], "launch_ms": launch_ms}


def run_ours(args, rank, local_rank, world):
    import torch
    from gated_delta_rule_119_b200 import load_library
    load_library()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    name = args.workload
    w = WORKLOADS[name]
    hbm, bf16_tf, peak_kind = measured_peaks()
    stream = torch.cuda.current_stream(device)
    wl = setup_workload(name, args, device, rank)

    clk = ClockSampler(device.index if device.index is not None else 0)
    passes = time_steps(wl["step"], args.steps, args.warmup, device, stream,
                        min_timed_s=args.min_timed_s, sampler=clk)
    ms = reduce_max(statistics.median(passes), device)
    launch_ms = reduce_max(launch_duration_ms(wl["step"], min(args.steps, 20), device, stream),
                           device)

    # end to end through the public API with host buffers
    e2e = run_e2e(args, name, device, stream, rank)

    value = wl["units"] * world / (ms / 1e3)
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "timed_passes": {"passes": len(passes), "median_ms": statistics.median(passes),
                         "min_ms": min(passes), "max_ms": max(passes),
                         "note": f"each pass times exactly {args.steps} steps; ms_per_step is "
                                 "the median pass (max over ranks)"},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w["dtype"], "data": "synthetic (seeded numpy; see inputs.py recipe)",
        "config": {**workload_config(name, None, world),
                   "l2": "no flush: the inputs of one step exceed the 126 MB L2"
                   if wl["bytes"] > 126e6 else "inputs fit in L2; reported as is"},
        "tflops": wl["flops"] / (launch_ms / 1e3) / 1e12,
        "roofline": roofline_entry(wl, launch_ms, hbm, peak_kind, name),
        "clocks": clk.summary(),
        "e2e": e2e,
        "gpu_launches": args.steps * len(passes) * wl["launches"],
        "gpu_launches_note": "kernel launches of this library inside the timed region "
                             f"({wl['launches']} per step, {len(passes)} passes of "
                             f"{args.steps} steps)",
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = wl["parity"](args.cpu_budget)
        if "parity" in res["cpu_baseline"]:
            res["parity"] = res["cpu_baseline"].pop("parity")
    del wl
    torch.cuda.empty_cache()
    if world == 1 and args.workloads:
        res["workloads"] = {}
        for other in [x for x in args.workloads.split(",") if x and x != name]:
            res["workloads"][other] = run_other_workload(other, args, device, stream, rank,
                                                         hbm, peak_kind)
            torch.cuda.empty_cache()
    return res


def variant_config(name):
    base, form, raw, L, indexed = VARIANTS[name]
    return {**workload_config(base, None, 1), "variant": name, "gate_form": form,
            "in_kernel_norm_and_beta_logits": raw, "decode_tokens_per_call": L,
            "indexed_state_pool": indexed}


def run_other_workload(name, args, device, stream, rank, hbm, peak_kind):
    """One more workload in the same process: ms per step (median of timed passes), tokens/s,
    its roofline and parity on a bounded oracle sample.  Failures are reported, not raised."""
    try:
        wl = setup_workload(name, args, device, rank)
        steps = min(args.steps, 20)
        clk = ClockSampler(device.index if device.index is not None else 0)
        passes = time_steps(wl["step"], steps, 3, device, stream, min_timed_s=0.3, sampler=clk)
        launch_ms = launch_duration_ms(wl["step"], min(steps, 10), device, stream)
        ms = statistics.median(passes)
        entry = {"ms_per_step": ms, "min_ms": min(passes), "max_ms": max(passes),
                 "passes": len(passes), "steps_per_pass": steps,
                 "value": wl["units"] / (ms / 1e3), "unit": "tokens/s",
                 "tflops": wl["flops"] / (launch_ms / 1e3) / 1e12,
                 "roofline": roofline_entry(wl, launch_ms, hbm, peak_kind, name),
                 "clocks": clk.summary(), "gpu_launches_per_step": wl["launches"],
                 "config": variant_config(name) if name in VARIANTS else workload_config(name, None, 1)}
        if not args.no_cpu_baseline:
            cb = wl["parity"](args.workload_parity_budget)
            entry["parity"] = cb.pop("parity", None)
            entry["cpu_baseline"] = cb
        del wl
        return entry
    except Exception as e:  # noqa: BLE001 - reported in the line instead
        return {"error": repr(e)[:300]}


def prefill_pairs(out, S_final, inp):
    """gpu_pair(n, h) for a prefill call's results: o of sequence n's tokens at head h
    (the token axis packed, whatever the view of ``out``) and its final state."""
    o_flat, cu = out.view(-1, inp.H, inp.dv), inp.offsets()

    def gpu_pair(n, hh):
        o = o_flat[int(cu[n]):int(cu[n + 1]), hh].float().cpu().numpy()
        return o, S_final[n, hh].cpu().numpy()
    return gpu_pair


def decode_pairs(dev_in, S0, device, kda_decode_step):
    """The GPU's results for the decode steps the CPU baseline replays: the same step
    inputs from the initial state, on a copy of it.  Returns gpu_pair(n, h)."""
    import torch
    S_chk = torch.from_numpy(S0).to(device, copy=True)
    outs = [kda_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S_chk) for d in dev_in]
    if torch.device(device).type == "cuda":
        torch.cuda.synchronize(device)

    def gpu_pair(n, hh):
        o = torch.stack([o[n, hh] for o in outs]).float().cpu().numpy()
        return o, S_chk[n, hh].cpu().numpy()
    return gpu_pair


def e2e_groups(N: int, cu=None, max_groups: int = 4):
    """The end-to-end path's sequence groups: up to ``max_groups`` contiguous ranges of the N
    sequences, as (first, end, token slice, rebased cu_seqlens or None).  Token tensors lead with
    the sequence axis (fixed length: the slice is over sequences) or are packed (the slice is the
    group's token range and its cu_seqlens start at 0)."""
    P = min(N, max_groups)
    out = []
    for g in range(P):
        b0, b1 = N * g // P, N * (g + 1) // P
        if cu is None:
            out.append((b0, b1, slice(b0, b1), None))
        else:
            out.append((b0, b1, slice(int(cu[b0]), int(cu[b1])),
                        (np.asarray(cu[b0:b1 + 1], dtype=np.int64) - int(cu[b0])).astype(np.int32)))
    return out


def run_e2e(args, name, device, stream, rank, return_outputs=False):
    """The same metric through the public call with pinned host buffers: every step copies its
    inputs host -> device, makes the call and copies its results back, all inside the timed
    region.  The N sequences go in up to four groups on three streams (copies in, the calls,
    copies out), so a group's results travel back while the next group's inputs travel in and
    another group is computed: the host link carries both directions at once.  With
    ``return_outputs`` the host buffers of the last step's results come back too (for tests)."""
    import torch
    from gated_delta_rule_119_b200 import kda_chunk_fwd, kda_decode_step
    w = WORKLOADS[name]
    steps = max(1, min(args.steps, args.e2e_steps))
    if name == "decode":
        N, H, dk, dv = w["B"], w["H"], w["dk"], w["dv"]
        inp = make_decode_step(N, H, dk, dv, w["dtype"], rank_seed(w["index"], rank), 0)
        host = to_torch(inp, "cpu", pin=True)
        S_host = torch.from_numpy(make_decode_state(N, H, dk, dv, 5)).pin_memory()
        out_host = torch.empty((N, H, dv), dtype=host["q"].dtype).pin_memory()
        S_dev = torch.empty_like(S_host, device=device)
        S_dev.copy_(S_host)
        units, cu = N, None
    else:
        inp = make_workload(name) if rank == 0 else make_inputs(
            w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"], rank_seed(w["index"], rank),
            state=w["state"], varlen=w["varlen"], gates=w["gates"])
        host = to_torch(inp, "cpu", pin=True)
        out_host = torch.empty(host["v"].shape, dtype=host["q"].dtype).pin_memory()
        S_host = torch.empty((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=torch.float32).pin_memory()
        N, units = inp.n_seqs, inp.total_tokens
        cu = None if host["cu_seqlens"] is None else host["cu_seqlens"].numpy().astype(np.int64)
    # Decode keeps the recurrent state resident in HBM across steps (it is the model's
    # memory, not a step input): a step moves the new token's q, k, v and gates in and
    # its o out.  Prefill moves every input in and o plus the final states out.
    groups = []
    plan = e2e_groups(N, cu)
    bounds = [(b0, b1) for b0, b1, _, _ in plan]
    for b0, b1, sl, cu_g in plan:
        hin = {k: (None if host.get(k) is None else host[k][sl]) for k in ("q", "k", "v", "log_alpha", "beta")}
        hin["S0"] = None if host.get("S0") is None else host["S0"][b0:b1]
        hin["cu_seqlens"] = None if cu_g is None else torch.from_numpy(cu_g).pin_memory()
        g = {"in": hin, "dev": {k: (None if t is None else torch.empty_like(t, device=device))
                                for k, t in hin.items()},
             "out_h": out_host[sl], "out_d": torch.empty_like(out_host[sl], device=device)}
        if name != "decode":
            g["S_h"] = S_host[b0:b1]
            g["S_d"] = torch.empty_like(g["S_h"], device=device)
        groups.append(g)
    h2d = sum(t.numel() * t.element_size() for g in groups for t in g["in"].values() if t is not None)
    d2h = sum(g["out_h"].numel() * g["out_h"].element_size() + (g["S_h"].numel() * 4 if "S_h" in g else 0)
              for g in groups)
    s_in, s_c, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_i = [torch.cuda.Event() for _ in groups]   # group g's inputs are on the device
    ev_c = [torch.cuda.Event() for _ in groups]   # group g's call is done (its input buffers are free)
    ev_o = [torch.cuda.Event() for _ in groups]   # group g's results are home (its output buffers are free)

    def one():
        for gi, (g, (b0, b1)) in enumerate(zip(groups, bounds)):
            s_in.wait_event(ev_c[gi])
            with torch.cuda.stream(s_in):
                for k, t in g["in"].items():
                    if t is not None:
                        g["dev"][k].copy_(t, non_blocking=True)
            ev_i[gi].record(s_in)
            s_c.wait_event(ev_i[gi])
            s_c.wait_event(ev_o[gi])
            d = g["dev"]
            if name == "decode":
                kda_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S_dev[b0:b1], g["out_d"],
                                stream=s_c)
            else:
                kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"],
                              g["out_d"], g["S_d"], stream=s_c)
            ev_c[gi].record(s_c)
            s_out.wait_event(ev_c[gi])
            with torch.cuda.stream(s_out):
                g["out_h"].copy_(g["out_d"], non_blocking=True)
                if "S_h" in g:
                    g["S_h"].copy_(g["S_d"], non_blocking=True)
            ev_o[gi].record(s_out)

    one()
    torch.cuda.synchronize(device)
    barrier(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(s_in)
    for _ in range(steps):
        one()
    ev1.record(s_out)                             # after the last group's results are home
    torch.cuda.synchronize(device)
    ms = reduce_max(ev0.elapsed_time(ev1) / steps, device)
    world = int(os.environ.get("WORLD_SIZE", 1))
    res = {"value": units * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "steps": steps, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "path": f"pinned host -> kda_* public call -> pinned host, the sequences in {len(groups)} groups on "
                   "three streams (copies in, calls, copies out overlapping)"
                   + (" (decode state resident in HBM)" if name == "decode" else "")}
    return (res, host, out_host, S_host) if return_outputs else res


def run_reference(args, rank, world):
    """The fp64 CPU oracle on a bounded sample of the same workload."""
    name = args.workload
    w = WORKLOADS[name]
    samples = []
    for i in range(args.warmup + args.steps):
        if name == "decode":
            N, H, dk, dv = w["B"], w["H"], w["dk"], w["dv"]
            ins = [make_decode_step(N, H, dk, dv, w["dtype"], w["index"], t) for t in range(2)]
            cb = cpu_baseline_decode(ins, make_decode_state(N, H, dk, dv, w["index"]),
                                     args.ref_step_budget)
        else:
            if i == 0:
                inp = make_workload(name)
            cb = cpu_baseline(inp, args.ref_step_budget)
        if i >= args.warmup:
            samples.append(cb)
    value = statistics.median(s["value"] for s in samples)
    ms = float(np.median([s["seconds"] * 1e3 for s in samples]))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy; see inputs.py recipe)",
            "config": workload_config(name, None, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": samples[-1]["cores"], "cpu_model": cpu_model(),
                             "kind": "oracle", "sample": samples[-1]["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def profile_bwd_small():
    """Three kda_chunk_bwd calls on B=4 T=512 H=16 dk=dv=128 bf16: the prefill_bwd workload's
    CTAs (one per (sequence, head, d_v half)) with an eighth of its chunks, a case small enough
    for a full ncu capture."""
    import torch
    from gated_delta_rule_119_b200 import kda_chunk_bwd
    d = to_torch(make_inputs(4, 512, 16, 128, 128, "bf16", 3), "cuda")
    g = torch.Generator(device="cpu").manual_seed(5)
    dO = torch.randn(d["v"].shape, generator=g).to("cuda").to(d["q"].dtype)
    for _ in range(3):
        r = kda_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dO, d["S0"], d["cu_seqlens"])
    torch.cuda.synchronize()
    print("ok", float(r["dq"].float().abs().max()), flush=True)


PROFILE_CASES = {"bwd_small": profile_bwd_small}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="prefill")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--decode-inputs", type=int, default=64,
                    help="distinct per-step decode inputs held on the device (cycled)")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of host-core work for the CPU baseline sample")
    ap.add_argument("--ref-step-budget", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the timed passes of --steps steps until about this much "
                         "timed work (at least 5 passes)")
    ap.add_argument("--workloads",
                    default="decode,varlen,extremes,prefill_fused,prefill_gdn,prefill_bwd,decode_indexed,"
                            "decode_mtp4",
                    help="other workloads measured in the same process at N=1 (comma list; "
                         "empty for none)")
    ap.add_argument("--workload-parity-budget", type=float, default=3.0)
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="only run the named small case a few times (for ncu captures) and exit")
    args = ap.parse_args(argv)
    if args.profile_case:
        PROFILE_CASES[args.profile_case]()
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, local_rank, world)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
