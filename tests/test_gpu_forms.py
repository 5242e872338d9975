"""GPU parity of the extended entry points (kda_chunk_fwd_ex, kda_decode_ex) through the C ABI.

* Gate forms: the scalar gate (Gated DeltaNet, "22,580" §08), no gate (DeltaNet, "22,580"
  §5-§6) and the fused gate of "Ten questions" Q9 with in-kernel key / query normalisation
  and beta logits, each against the fp64 oracle fed the oracle's own gate front-end
  (oracle/gates.py), pooled and per (sequence, head) pair, at the dtype's bar.
* The scalar and no-gate forms run the per-channel arithmetic on the broadcast gate, so their
  results must be bit-identical to kda_chunk_fwd given log_alpha broadcast over the channels
  (or zero).
* Decode from an indexed state pool with L tokens per call ("Ten questions" Q10): parity with
  the oracle; one call over L tokens bit-identical to L calls of one token; padding entries
  (-1) and the slots no sequence names left untouched; an index past the pool reported by
  kda_device_status.
"""
import numpy as np
import pytest

import oracle
from oracle import gates
from gated_delta_rule_119_b200.inputs import (WORKLOADS, make_decode_state, make_form_inputs,
                                             to_torch)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}
KIND = {"channel": 0, "scalar": 1, "none": 2, "fused": 3}


def rel_err(x, r):
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def oracle_inputs(inp):
    """q, k, log_alpha [T, H, dk], beta as the oracle reads them, from the form's inputs."""
    dk = inp.dk
    if inp.form == "channel":
        la = inp.log_alpha
    elif inp.form == "scalar":
        la = gates.broadcast_scalar(inp.log_alpha, dk)
    elif inp.form == "none":
        la = np.zeros(inp.q.shape)
    else:
        la = gates.fused_log_alpha(inp.f, inp.A_log, inp.dt_bias)
    q = gates.l2_normalize(inp.q) if inp.flags & 1 else inp.q
    k = gates.l2_normalize(inp.k) if inp.flags & 2 else inp.k
    beta = gates.sigmoid(inp.beta) if inp.flags & 4 else inp.beta
    return q, k, la, beta


def run_form(inp, d=None):
    from gated_delta_rule_119_b200 import kda_chunk_fwd_ex
    d = to_torch(inp) if d is None else d
    gate = {"channel": d["log_alpha"], "scalar": d["log_alpha"], "none": None, "fused": d["f"]}[inp.form]
    out, Sf = kda_chunk_fwd_ex(d["q"], d["k"], d["v"], gate, d["beta"], d["S0"], d["cu_seqlens"],
                               gate_kind=KIND[inp.form], A_log=d["A_log"], dt_bias=d["dt_bias"],
                               norm_q=bool(inp.flags & 1), norm_k=bool(inp.flags & 2),
                               beta_logits=bool(inp.flags & 4))
    torch.cuda.synchronize()
    return out, Sf


def check_form(inp, tasks=None):
    out, Sf = run_form(inp)
    o = out.float().cpu().numpy().reshape(inp.total_tokens, inp.H, inp.dv)
    S = Sf.cpu().numpy()
    cu = inp.offsets()
    if tasks is None:
        tasks = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H)]
    q, k, la, beta = oracle_inputs(inp)
    outs, sts = oracle.recurrent(q, k, inp.v, la, beta, inp.S0, cu, tasks=tasks)
    po, ps, go, ro = [], [], [], []
    for (n, h), on, sn in zip(tasks, outs, sts):
        if cu[n + 1] > cu[n]:
            x = o[cu[n]:cu[n + 1], h]
            po.append(rel_err(x, on))
            go.append(x.ravel())
            ro.append(on.ravel())
        ps.append(rel_err(S[n, h], sn))
    eo = rel_err(np.concatenate(go), np.concatenate(ro)) if go else 0.0
    es = rel_err(np.stack([S[n, h] for n, h in tasks]), np.stack(sts))
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0
    tol = TOL[inp.dtype]
    print(f"[forms] {inp.form} flags={inp.flags} {inp.dtype} T={inp.total_tokens} H={inp.H} "
          f"d={inp.dk}x{inp.dv} pairs={len(tasks)}: o {eo:.3e} (worst pair {max(po, default=0):.3e}) "
          f"S {es:.3e} (worst pair {max(ps):.3e})")
    assert eo <= tol and max(po, default=0.0) <= tol
    assert es <= tol and max(ps) <= tol


# ------------------------------------------------------------------ gate forms, small shapes
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("form", ["scalar", "none", "fused"])
@pytest.mark.parametrize("T", [1, 65, 130])
@pytest.mark.parametrize("d", [32, 128])
def test_forms_small(dtype, form, T, d):
    check_form(make_form_inputs(2, T, 3, d, d, dtype, 300 + T + d, form, state=T != 65,
                                raw=form == "fused"))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("form", ["scalar", "fused"])
def test_forms_varlen_ragged(dtype, form):
    cu = [0, 0, 1, 65, 200, 263, 263]
    check_form(make_form_inputs(6, 0, 3, 128, 128, dtype, 401, form, state=True, cu_seqlens=cu,
                                raw=form == "fused"))


def test_fused_gate_without_normalisation():
    """The fused gate alone (flags 0): unit keys from the generator, beta as given."""
    check_form(make_form_inputs(2, 200, 4, 128, 128, "bf16", 402, "fused"))


# ------------------------------------------------- fused gates on the workload shapes
def _sample(inp, k, seed):
    rng = np.random.default_rng(seed)
    lens = np.diff(inp.offsets())
    tasks = {(int(np.argmax(lens)), 0), (inp.n_seqs - 1, inp.H - 1)}
    while len(tasks) < k:
        tasks.add((int(rng.integers(inp.n_seqs)), int(rng.integers(inp.H))))
    return sorted(tasks)


@pytest.mark.parametrize("name", ["tiny_f32", "prefill", "varlen", "extremes"])
def test_fused_gates_on_workload_shapes(name):
    """The prefill workloads' shapes (sizes, varlen cut points, states) with the fused gate,
    unnormalised q and k and beta logits; the oracle recomputes every pair of the small
    workload and 16 sampled pairs of the large ones."""
    w = WORKLOADS[name]
    inp = make_form_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"], w["index"], "fused",
                           state=w["state"], varlen=w["varlen"], raw=True)
    check_form(inp, None if name == "tiny_f32" else _sample(inp, 16, 77))


# ----------------------------------------------------- scalar / no gate: bit-identical
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "bf16"), (32, "f32")])
def test_scalar_and_no_gate_are_the_broadcast_channel_gate(d, dtype):
    from gated_delta_rule_119_b200 import kda_chunk_fwd
    inp = make_form_inputs(2, 300, 4, d, d, dtype, 410, "scalar", state=True)
    t = to_torch(inp)
    o_s, S_s = run_form(inp, t)
    la_b = t["log_alpha"].unsqueeze(-1).expand(*t["log_alpha"].shape, d).contiguous()
    o_c, S_c = kda_chunk_fwd(t["q"], t["k"], t["v"], la_b, t["beta"], t["S0"])
    inp.form = "none"
    inp.log_alpha = None
    o_n, S_n = run_form(inp, {**t, "log_alpha": None})
    o_z, S_z = kda_chunk_fwd(t["q"], t["k"], t["v"], torch.zeros_like(la_b), t["beta"], t["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_c) and torch.equal(S_s, S_c)
    assert torch.equal(o_n, o_z) and torch.equal(S_n, S_z)


# ------------------------------------------------------------------- indexed decode
def _decode_case(N, L, H, d, dtype, seed, form="channel", raw=False):
    """N sequences x L new tokens as a packed batch (sequence-major), the gate form's inputs."""
    inp = make_form_inputs(N, L, H, d, d, dtype, seed, form, raw=raw)
    return inp


def _decode_call(inp, N, L, pool, idx, d_in=None):
    from gated_delta_rule_119_b200 import kda_decode_ex
    t = to_torch(inp) if d_in is None else d_in
    gate = {"channel": t["log_alpha"], "scalar": t["log_alpha"], "none": None, "fused": t["f"]}[inp.form]
    return kda_decode_ex(t["q"], t["k"], t["v"], gate, t["beta"], pool, idx, gate_kind=KIND[inp.form],
                         A_log=t["A_log"], dt_bias=t["dt_bias"], norm_q=bool(inp.flags & 1),
                         norm_k=bool(inp.flags & 2), beta_logits=bool(inp.flags & 4))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("form,raw", [("channel", False), ("scalar", False), ("fused", True)])
@pytest.mark.parametrize("L", [1, 3])
def test_decode_indexed_pool(dtype, form, raw, L):
    """Sequences on scattered pool slots (one of them padding): o and the updated slots
    against the oracle run from each slot's state; padding and unnamed slots untouched."""
    N, H, d, P = 6, 3, 128, 20
    inp = _decode_case(N, L, H, d, dtype, 500 + L, form, raw)
    pool0 = make_decode_state(P, H, d, d, 501)
    idx = np.array([7, 2, -1, 19, 0, 11], dtype=np.int32)
    pool = torch.from_numpy(pool0).cuda()
    t = to_torch(inp)
    out = _decode_call(inp, N, L, pool, torch.from_numpy(idx).cuda(), t)
    torch.cuda.synchronize()
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0
    q, k, la, beta = oracle_inputs(inp)
    S0 = np.stack([pool0[max(i, 0)] for i in idx])
    ro, rS = oracle.recurrent_full(q, k, inp.v, la, beta, S0, np.arange(N + 1) * L)
    o = out.float().cpu().numpy().reshape(N * L, H, d)
    pg = pool.cpu().numpy()
    tol = TOL[dtype]
    for n, i in enumerate(idx):
        if i < 0:
            continue
        assert rel_err(o[n * L:(n + 1) * L], ro[n * L:(n + 1) * L]) <= tol
        assert rel_err(pg[i], rS[n]) <= tol
    named = {int(i) for i in idx if i >= 0}
    for slot in range(P):
        if slot not in named:
            np.testing.assert_array_equal(pg[slot], pool0[slot])


def test_decode_padding_leaves_out_untouched():
    from gated_delta_rule_119_b200 import kda_decode_ex
    N, L, H, d = 3, 2, 2, 64
    inp = _decode_case(N, L, H, d, "bf16", 510)
    t = to_torch(inp)
    pool = torch.from_numpy(make_decode_state(4, H, d, d, 511)).cuda()
    out = torch.full((N, L, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    idx = torch.tensor([1, -1, 3], dtype=torch.int32, device="cuda")
    kda_decode_ex(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], pool, idx, out)
    torch.cuda.synchronize()
    assert torch.all(out[1] == 7.0) and not torch.all(out[0] == 7.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("form,raw", [("channel", False), ("fused", True)])
@pytest.mark.parametrize("L", [4, 7])
def test_multi_token_step_equals_single_steps(dtype, form, raw, L):
    """One call over L tokens == L calls of one token each, bit for bit (L = 7 spans two
    batches of staged tokens, the second one partial)."""
    N, H, d, P = 5, 2, 128, 9
    inp = _decode_case(N, L, H, d, dtype, 520, form, raw)
    t = to_torch(inp)
    idx = torch.tensor([4, 0, 8, 2, 6], dtype=torch.int32, device="cuda")
    pool0 = torch.from_numpy(make_decode_state(P, H, d, d, 521)).cuda()
    pool_a, pool_b = pool0.clone(), pool0.clone()
    out_a = _decode_call(inp, N, L, pool_a, idx, t)
    outs = []
    for l in range(L):
        one = {k_: (None if v_ is None or k_ in ("A_log", "dt_bias", "S0", "cu_seqlens")
                    else v_[:, l:l + 1].contiguous())            # [N, L, ...] -> token l
               for k_, v_ in t.items()}
        one["A_log"], one["dt_bias"] = t["A_log"], t["dt_bias"]
        outs.append(_decode_call(inp, N, 1, pool_b, idx, one))
    torch.cuda.synchronize()
    assert torch.equal(out_a, torch.cat(outs, 1))
    assert torch.equal(pool_a, pool_b)


def test_decode_matches_prefill_for_the_same_tokens():
    """L decode tokens from S0 == a prefill over the same L tokens from S0 (both on the GPU,
    different algorithms: within the bf16 bar)."""
    from gated_delta_rule_119_b200 import kda_chunk_fwd
    N, L, H, d = 3, 70, 2, 128
    inp = _decode_case(N, L, H, d, "bf16", 530)
    t = to_torch(inp)
    S0 = make_decode_state(N, H, d, d, 531)
    pool = torch.from_numpy(S0).cuda()
    o_dec = _decode_call(inp, N, L, pool, None, t)
    o_pre, S_pre = kda_chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"],
                                 torch.from_numpy(S0).cuda())
    torch.cuda.synchronize()
    assert rel_err(o_dec.float().cpu().numpy(), o_pre.float().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(pool.cpu().numpy(), S_pre.cpu().numpy()) <= TOL["bf16"]


def test_decode_index_past_the_pool_is_reported():
    """An entry >= P is skipped (nothing read or written for it) and reported once."""
    from gated_delta_rule_119_b200 import kda_decode_ex, kda_device_status
    N, H, d, P = 2, 2, 32, 3
    inp = _decode_case(N, 1, H, d, "f32", 540)
    t = to_torch(inp)
    pool0 = torch.from_numpy(make_decode_state(P, H, d, d, 541)).cuda()
    pool = pool0.clone()
    idx = torch.tensor([1, 3], dtype=torch.int32, device="cuda")
    kda_decode_ex(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], pool, idx)
    assert kda_device_status() == -11
    assert kda_device_status() == 0
    assert torch.equal(pool[0], pool0[0]) and torch.equal(pool[2], pool0[2])
    assert not torch.equal(pool[1], pool0[1])


def test_decode_workload_indexed_sampled():
    """The decode workload's full pool (256 x 32 x 128 x 128 fp32) with the sequences on a
    seeded permutation of the slots and the fused gate, 3 steps of L = 2 tokens; the oracle
    recomputes 12 sampled (sequence, head) pairs."""
    w = WORKLOADS["decode"]
    N, H, d = w["B"], w["H"], w["dk"]
    pool0 = make_decode_state(N, H, d, d, w["index"])
    pool = torch.from_numpy(pool0).cuda()
    perm = np.random.default_rng(5).permutation(N).astype(np.int32)
    idx = torch.from_numpy(perm).cuda()
    steps, L = 3, 2
    ins = [_decode_case(N, L, H, d, "bf16", (w["index"], s), "fused", True) for s in range(steps)]
    outs = [_decode_call(i, N, L, pool, idx).float().cpu().numpy() for i in ins]
    torch.cuda.synchronize()
    pg = pool.cpu().numpy()
    rng = np.random.default_rng(6)
    for n, h in zip(rng.integers(N, size=12), rng.integers(H, size=12)):
        cat = []
        for i in ins:
            q, k, la, beta = oracle_inputs(i)
            sl = slice(n * L, (n + 1) * L)
            cat.append((q[sl, h:h + 1], k[sl, h:h + 1], i.v[sl, h:h + 1], la[sl, h:h + 1], beta[sl, h:h + 1]))
        q, k, v, la, beta = (np.concatenate([c[j] for c in cat]) for j in range(5))
        ro, rS = oracle.recurrent_full(q, k, v, la, beta, pool0[perm[n], h][None, None].copy())
        go = np.concatenate([o[n, :, h] for o in outs])
        assert rel_err(go, ro[:, 0]) <= TOL["bf16"]
        assert rel_err(pg[perm[n], h], rS[0, 0]) <= TOL["bf16"]
