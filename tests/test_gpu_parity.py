"""GPU parity: libkda.so (through its C ABI) against the fp64 oracle.

Error metric: max|x - r| / max|r| (l-infinity relative), for o and for the final
state, taken two ways and both held to the bar: pooled over every checked (sequence,
head) pair, and for each pair on its own (the worst pair is reported), so that a head
whose outputs are small next to the others' cannot hide a large error of its own.  Bars:
1e-4 for fp32 inputs, 2e-2 for bf16 inputs.  Inputs are the seeded synthetic ones of
``gated_delta_rule_119_b200.inputs``; the oracle reads the same bytes.
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_119_b200.inputs import (WORKLOADS, make_decode_state, make_decode_step,
                                             make_inputs, make_workload, to_torch)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(x, r):
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def kda():
    from gated_delta_rule_119_b200 import kda_chunk_fwd, kda_decode_step
    return kda_chunk_fwd, kda_decode_step


def run_chunk(inp, S_final=True):
    chunk_fwd, _ = kda()
    d = to_torch(inp)
    out, Sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                        d["cu_seqlens"], output_final_state=S_final)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().reshape(inp.total_tokens, inp.H, inp.dv)
    return o, (None if Sf is None else Sf.cpu().numpy())


def pair_errors(o, S, cu, tasks, outs, sts):
    """Pooled and worst per-pair errors of o [T_total, H, dv] and S [N, H, dk, dv] against
    the oracle's per-pair results.  Returns (pooled o, pooled S, worst o, worst S, worst o
    pair); pairs with no tokens count for S only."""
    go, ro, gs, rs, po, ps = [], [], [], [], [], []
    for (n, h), on, sn in zip(tasks, outs, sts):
        if cu[n + 1] > cu[n]:
            x = o[cu[n]:cu[n + 1], h]
            go.append(x.ravel())
            ro.append(on.ravel())
            po.append(rel_err(x, on))
        gs.append(S[n, h].ravel())
        rs.append(sn.ravel())
        ps.append(rel_err(S[n, h], sn))
    eo = rel_err(np.concatenate(go), np.concatenate(ro)) if go else 0.0
    es = rel_err(np.concatenate(gs), np.concatenate(rs))
    worst = [t for t in tasks if cu[t[0] + 1] > cu[t[0]]]
    wo = max(po) if po else 0.0
    return eo, es, wo, max(ps), (worst[int(np.argmax(po))] if po else None)


def check_against_oracle(inp, tol=None, tasks=None):
    """Runs the library on `inp` and checks o and S_final against the oracle over `tasks`
    ((sequence, head) pairs; default every pair), pooled and per pair."""
    tol = TOL[inp.dtype] if tol is None else tol
    o, S = run_chunk(inp)
    cu = inp.offsets()
    if tasks is None:
        tasks = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H)]
    outs, sts = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu,
                                 tasks=tasks)
    eo, es, wo, ws, wpair = pair_errors(o, S, cu, tasks, outs, sts)
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0, "a kernel gave up a bounded wait"
    print(f"[parity] {inp.dtype} T={inp.total_tokens} H={inp.H} dk={inp.dk} dv={inp.dv} "
          f"gates={inp.meta.get('gates')} pairs={len(tasks)}: o {eo:.3e} (worst pair {wo:.3e} "
          f"at {wpair})  S_final {es:.3e} (worst pair {ws:.3e})")
    assert eo <= tol and wo <= tol, f"o: max rel err {eo:.3e}, worst pair {wo:.3e} > {tol}"
    assert es <= tol and ws <= tol, f"S_final: max rel err {es:.3e}, worst pair {ws:.3e} > {tol}"
    return max(eo, wo), max(es, ws)


# ------------------------------------------------------------------ small cases
def test_tiny_f32_workload():
    """The fp32 workload (B=1, H=2, T=128, dk=dv=32, S0=0) in full."""
    check_against_oracle(make_workload("tiny_f32"))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 130])
@pytest.mark.parametrize("d", [32, 128])
def test_small_shapes(dtype, T, d):
    check_against_oracle(make_inputs(2, T, 3, d, d, dtype, 100 + T + d, state=T % 2 == 1))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (32, 64), (64, 64)])
def test_rectangular_heads(dtype, dk, dv):
    check_against_oracle(make_inputs(2, 150, 2, dk, dv, dtype, 7 + dk + dv, state=True))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_ragged_with_empty_sequences(dtype):
    cu = [0, 0, 1, 65, 65, 200, 263, 263]
    check_against_oracle(make_inputs(7, 0, 3, 128, 128, dtype, 211, state=True, cu_seqlens=cu))


def test_zero_tokens_returns_initial_state():
    inp = make_inputs(3, 0, 2, 64, 64, "bf16", 5, state=True, cu_seqlens=[0, 0, 0, 0])
    chunk_fwd, _ = kda()
    d = to_torch(inp)
    out, Sf = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                        d["cu_seqlens"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Sf.cpu().numpy(), inp.S0)


def test_final_state_optional_and_in_place():
    inp = make_inputs(2, 100, 2, 128, 128, "bf16", 9, state=True)
    chunk_fwd, _ = kda()
    d = to_torch(inp)
    o1, _ = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                      output_final_state=False)
    S = d["S0"].clone()
    o2, S2 = chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S, S_final=S)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S.data_ptr()
    _, ref = run_chunk(inp)
    np.testing.assert_array_equal(o1.cpu().float().numpy(), o2.cpu().float().numpy())
    np.testing.assert_array_equal(S.cpu().numpy(), ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_degenerate_gates(dtype):
    """alpha -> 0 (log_alpha = -1e4: the memory is cleared every token), beta = 0
    (nothing written), beta = 1, and no forgetting, mixed across heads."""
    inp = make_inputs(2, 140, 4, 128, 128, dtype, 17, state=True)
    inp.log_alpha[:, 0] = -1e4
    inp.beta[:, 1] = 0.0
    inp.beta[:, 2] = 1.0
    inp.log_alpha[:, 3] = 0.0
    inp.log_alpha[::7, 2] = -1e4
    check_against_oracle(inp)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_spread_past_fp32_normal_range(dtype):
    """Channels whose decay over 16 rows sums to about 90-135 (past fp32's normal range, e^-87,
    for an unscaled running product; short of the exact path's limit of 140) beside weakly
    decaying channels in the same heads: the block path's rescaled factors must keep their
    precision on every row, the last rows of each 16-row block included."""
    inp = make_inputs(2, 300, 3, 128, 128, dtype, 23, state=True)
    rng = np.random.default_rng(24)
    inp.log_alpha[:, 0, :32] = rng.uniform(-8.4, -5.6, size=(inp.total_tokens, 32)).astype(np.float32)
    inp.log_alpha[:, 1, ::4] = -7.0
    inp.log_alpha[:, 2, 64:] = rng.uniform(-6.5, -6.0, size=(inp.total_tokens, 64)).astype(np.float32)
    check_against_oracle(inp)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_extreme_gates_small(dtype):
    check_against_oracle(make_inputs(2, 300, 4, 128, 128, dtype, 19, gates="extremes",
                                     state=True))


# ---------------------------------------------------------- full-size workloads
def sampled_tasks(inp, k, seed):
    rng = np.random.default_rng(seed)
    n_seq = inp.n_seqs
    lens = np.diff(inp.offsets())
    tasks = {(int(np.argmax(lens)), int(rng.integers(inp.H)))}      # the longest sequence
    while len(tasks) < k:
        tasks.add((int(rng.integers(n_seq)), int(rng.integers(inp.H))))
    return sorted(tasks)


@pytest.mark.parametrize("name", ["prefill", "varlen", "extremes"])
def test_full_workload_all_pairs(name):
    """Each bf16 prefill workload at its full size, in the launch configuration the
    bench times; the oracle recomputes every (sequence, head) pair (64, 256 and 64 of
    them), checked pooled and pair by pair."""
    check_against_oracle(make_workload(name))


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32)])
def test_maximum_head_count(dtype, d):
    """H = 65,535, the largest head count the library accepts, over two ragged sequences of
    three tokens in all: the largest grids of both prefill paths run (every (chunk, head)
    of the intra-chunk kernel, 2 x 65,535 x 2 scan CTAs).  The oracle recomputes sampled
    (sequence, head) pairs, the last head among them; only their states are copied back."""
    H = 65535
    inp = make_inputs(2, 3, H, d, d, dtype, 1210, varlen=True)
    chunk_fwd, _ = kda()
    t = to_torch(inp)
    out, Sf = chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], None, t["cu_seqlens"],
                        output_final_state=True)
    torch.cuda.synchronize()
    tasks = sorted(set(sampled_tasks(inp, 6, 1211)) | {(0, H - 1), (1, H - 1), (1, 0)})
    cu = inp.offsets()
    o = out.float().cpu().numpy().reshape(inp.total_tokens, H, d)
    S = {(n, h): Sf[n, h].cpu().numpy() for n, h in tasks}
    del out, Sf, t
    torch.cuda.empty_cache()
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0, "a kernel gave up a bounded wait"
    outs, sts = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, cu, tasks=tasks)
    eo = rel_err(np.concatenate([o[cu[n]:cu[n + 1], h].ravel() for n, h in tasks]),
                 np.concatenate([x.ravel() for x in outs]))
    es = max(rel_err(S[task], st) for task, st in zip(tasks, sts))
    print(f"[parity] max heads {dtype} d={d}: o {eo:.3e}  S_final {es:.3e}")
    assert eo <= TOL[dtype] and es <= TOL[dtype]


# ----------------------------------------------------------------------- decode
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (32, 32), (64, 128), (128, 64)])
def test_decode_steps(dtype, dk, dv):
    _, decode = kda()
    N, H, steps = 5, 3, 6
    S0 = make_decode_state(N, H, dk, dv, 77)
    S = torch.from_numpy(S0).cuda()
    ins = [make_decode_step(N, H, dk, dv, dtype, 77, t) for t in range(steps)]
    outs = []
    for inp in ins:
        d = to_torch(inp)
        outs.append(decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S).float()
                    .cpu().numpy())
    torch.cuda.synchronize()
    # oracle: each sequence is a run of `steps` tokens
    cat = lambda name: np.stack([getattr(i, name) for i in ins], axis=1).reshape(
        N * steps, *getattr(ins[0], name).shape[1:])
    cu = np.arange(N + 1) * steps
    ro, rS = oracle.recurrent_full(cat("q"), cat("k"), cat("v"), cat("log_alpha"), cat("beta"),
                                   S0, cu)
    go = np.stack(outs, axis=1).reshape(N * steps, H, dv)
    tol = TOL[dtype]
    assert rel_err(go, ro) <= tol
    assert rel_err(S.cpu().numpy(), rS) <= tol


def test_decode_workload_all_steps():
    """The decode workload as configured: 1,000 steps on the full state (256 sequences x 32
    heads x 128 x 128 fp32).  Each step's inputs are drawn on the host and uploaded in turn.
    For 16 sampled (sequence, head) pairs the oracle runs the same 1,000 tokens from the same
    initial state; o is compared at every step (per pair over all steps, and step by step)
    and the state after the last step."""
    _, decode = kda()
    w = WORKLOADS["decode"]
    N, H, dk, dv, steps = w["B"], w["H"], w["dk"], w["dv"], w["T"]
    S0 = make_decode_state(N, H, dk, dv, w["index"])
    S = torch.from_numpy(S0).cuda()
    rng = np.random.default_rng(31)
    pairs = sorted({(0, 0), (N - 1, H - 1)} | {(int(a), int(b)) for a, b in
                                                zip(rng.integers(N, size=14), rng.integers(H, size=14))})
    pn = torch.tensor([p[0] for p in pairs], device="cuda")
    ph = torch.tensor([p[1] for p in pairs], device="cuda")
    keep = {name: [] for name in ("q", "k", "v", "log_alpha", "beta")}
    go = []
    for t in range(steps):
        inp = make_decode_step(N, H, dk, dv, "bf16", w["index"], t)
        d = to_torch(inp)
        o = decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S)
        go.append(o[pn, ph].float())
        for name in keep:
            keep[name].append(np.stack([getattr(inp, name)[n, h] for n, h in pairs]))
    go = torch.stack(go, 1).cpu().numpy()                           # [pairs, steps, dv]
    Sg = S[pn, ph].cpu().numpy()
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0
    P = len(pairs)
    packed = {name: np.stack(x, 1).reshape(P * steps, 1, *x[0].shape[1:])
              for name, x in keep.items()}                          # pair-major token axis
    packed["beta"] = packed["beta"].reshape(P * steps, 1)
    S0p = np.stack([S0[n, h] for n, h in pairs])[:, None]
    ro, rS = oracle.recurrent_full(packed["q"], packed["k"], packed["v"], packed["log_alpha"],
                                   packed["beta"], S0p, np.arange(P + 1) * steps)
    ro = ro.reshape(P, steps, dv)
    per_pair = [rel_err(go[i], ro[i]) for i in range(P)]
    per_step = [max(rel_err(go[i, t], ro[i, t]) for i in range(P)) for t in range(steps)]
    s_err = [rel_err(Sg[i], rS[i, 0]) for i in range(P)]
    print(f"[parity] decode 1000 steps, {P} pairs: o worst pair {max(per_pair):.3e}, "
          f"worst single step {max(per_step):.3e} (steps 0-99 {max(per_step[:100]):.3e}, "
          f"900-999 {max(per_step[-100:]):.3e}); final state worst pair {max(s_err):.3e}")
    assert max(per_pair) <= TOL["bf16"] and max(s_err) <= TOL["bf16"]
    assert max(per_step) <= TOL["bf16"]


def test_decode_workload_sampled():
    """The decode workload's full state (256 sequences x 32 heads x 128 x 128 fp32),
    a few steps; the oracle recomputes sampled (sequence, head) pairs."""
    _, decode = kda()
    w = WORKLOADS["decode"]
    N, H, dk, dv, steps = w["B"], w["H"], w["dk"], w["dv"], 4
    S0 = make_decode_state(N, H, dk, dv, w["index"])
    S = torch.from_numpy(S0).cuda()
    ins = [make_decode_step(N, H, dk, dv, "bf16", w["index"], t) for t in range(steps)]
    outs = []
    for inp in ins:
        d = to_torch(inp)
        outs.append(decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S).float()
                    .cpu().numpy())
    Sg = S.cpu().numpy()
    rng = np.random.default_rng(3)
    for n, h in zip(rng.integers(N, size=6), rng.integers(H, size=6)):
        pick = lambda name: np.stack([getattr(i, name)[n, h] for i in ins])[:, None]
        ro, rS = oracle.recurrent_full(pick("q"), pick("k"), pick("v"), pick("log_alpha"),
                                       pick("beta"), S0[n:n + 1, h:h + 1].copy())
        assert rel_err(np.stack([o[n, h] for o in outs]), ro[:, 0]) <= TOL["bf16"]
        assert rel_err(Sg[n, h], rS[0, 0]) <= TOL["bf16"]


def test_decode_matches_prefill():
    """T decode steps == one prefill over the same T tokens (both on the GPU)."""
    chunk_fwd, decode = kda()
    inp = make_inputs(3, 70, 2, 128, 128, "bf16", 31, state=True)
    o_pre, S_pre = run_chunk(inp)
    d = to_torch(inp)
    S = d["S0"].clone()
    outs = []
    for t in range(inp.T):
        outs.append(decode(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                           d["v"][:, t].contiguous(), d["log_alpha"][:, t].contiguous(),
                           d["beta"][:, t].contiguous(), S))
    o_dec = torch.stack(outs, 1).float().cpu().numpy().reshape(-1, inp.H, inp.dv)
    assert rel_err(o_dec, o_pre) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_pre) <= TOL["bf16"]


# ------------------------------------------------------ errors with real memory
def test_errors_with_device_tensors():
    from gated_delta_rule_119_b200 import KDAError
    chunk_fwd, decode = kda()
    inp = make_inputs(1, 64, 1, 128, 128, "bf16", 3)
    d = to_torch(inp)
    with pytest.raises(KDAError, match="KDA_ERR_ALIAS"):
        chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], out=d["v"])
    raw = torch.empty(64 * 128 + 1, dtype=torch.bfloat16, device="cuda")
    qm = raw[1:].view(1, 64, 1, 128)                      # 2-byte offset: misaligned
    qm.copy_(d["q"])
    with pytest.raises(KDAError, match="KDA_ERR_ALIGN"):
        chunk_fwd(qm, d["k"], d["v"], d["log_alpha"], d["beta"])
    with pytest.raises(KDAError, match="KDA_ERR_CHUNK"):
        chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], C=128)
