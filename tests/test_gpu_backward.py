"""GPU parity of the backward pass (kda_chunk_bwd, through the C ABI) against the fp64 oracle's
gradients (oracle.backward, pinned by finite differences on the forward oracle).

For L = sum(dO * o) + sum(dS_final * S_final) every gradient -- dq, dk, dv, dlog_alpha (or the
scalar gate's, summed over channels), dbeta, dS0 -- is compared per tensor and per (sequence,
head) pair, max|x - r| / max|r|, with the dtype's bar (1e-4 fp32, 2e-2 bf16)."""
import numpy as np
import pytest

import oracle
from oracle import gates
from gated_delta_rule_119_b200.inputs import make_form_inputs, to_storage, storage_to_torch, to_torch

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}
KIND = {"channel": 0, "scalar": 1, "none": 2}


def rel_err(x, r):
    x, r = np.asarray(x, np.float64), np.asarray(r, np.float64)
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def grad_inputs(inp, seed, final=True):
    """dO in the input dtype (bf16 bits or fp32) and dS_final fp32, seeded."""
    rng = np.random.default_rng([seed, 99])
    dO = to_storage(rng.standard_normal((inp.total_tokens, inp.H, inp.dv), dtype=np.float32), inp.dtype)
    dSf = rng.standard_normal((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=np.float32) if final else None
    return dO, dSf


def run_bwd(inp, dO, dSf):
    from gated_delta_rule_119_b200 import kda_chunk_bwd
    t = to_torch(inp)
    dO_t = storage_to_torch(dO, inp.dtype, "cuda").view(t["v"].shape)
    dSf_t = None if dSf is None else torch.from_numpy(dSf).cuda()
    gate = None if inp.form == "none" else t["log_alpha"]
    g = kda_chunk_bwd(t["q"], t["k"], t["v"], gate, t["beta"], dO_t, t["S0"], t["cu_seqlens"], dSf_t,
                      gate_kind=KIND[inp.form])
    torch.cuda.synchronize()
    Tt, H = inp.total_tokens, inp.H
    out = {"dq": g["dq"].float().cpu().numpy().reshape(Tt, H, inp.dk),
           "dk": g["dk"].float().cpu().numpy().reshape(Tt, H, inp.dk),
           "dv": g["dv"].float().cpu().numpy().reshape(Tt, H, inp.dv),
           "dbeta": g["dbeta"].cpu().numpy().reshape(Tt, H), "dS0": g["dS0"].cpu().numpy()}
    if g["dgate"] is not None:
        out["dgate"] = g["dgate"].cpu().numpy().reshape(Tt, H, *g["dgate"].shape[len(t["beta"].shape):])
    return out


def check_bwd(inp, seed, final=True, tasks=None):
    dO, dSf = grad_inputs(inp, seed, final)
    g = run_bwd(inp, dO, dSf)
    la = {"channel": inp.log_alpha, "scalar": None, "none": None}[inp.form]
    if inp.form == "scalar":
        la = gates.broadcast_scalar(inp.log_alpha, inp.dk)
    elif inp.form == "none":
        la = np.zeros(inp.q.shape)
    cu = inp.offsets()
    r = oracle.backward(inp.q, inp.k, inp.v, la, inp.beta, inp.S0, cu, dO, dSf, tasks=tasks)
    ref = {"dq": r["dq"], "dk": r["dk"], "dv": r["dv"], "dbeta": r["dbeta"], "dS0": r["dS0"]}
    if inp.form == "channel":
        ref["dgate"] = r["dlog_alpha"]
    elif inp.form == "scalar":
        ref["dgate"] = r["dlog_alpha"].sum(-1)
    if tasks is None:
        tasks = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H)]
    tol = TOL[inp.dtype]
    worst = {}
    for name, rv in ref.items():
        gv = g[name]
        if name == "dS0":
            xs = [gv[n, h] for n, h in tasks]
            rs = [rv[n, h] for n, h in tasks]
        else:
            xs = [gv[cu[n]:cu[n + 1], h] for n, h in tasks if cu[n + 1] > cu[n]]
            rs = [rv[cu[n]:cu[n + 1], h] for n, h in tasks if cu[n + 1] > cu[n]]
        if not xs:
            continue
        pooled = rel_err(np.concatenate([x.ravel() for x in xs]), np.concatenate([x.ravel() for x in rs]))
        per = max(rel_err(x, y) for x, y in zip(xs, rs) if np.abs(y).max() > 0) \
            if any(np.abs(y).max() > 0 for y in rs) else 0.0
        worst[name] = (pooled, per)
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0
    print(f"[backward] {inp.form} {inp.dtype} T={inp.total_tokens} H={inp.H} d={inp.dk}x{inp.dv}: " +
          "  ".join(f"{k} {p:.2e}/{w:.2e}" for k, (p, w) in worst.items()))
    for name, (p, w) in worst.items():
        assert p <= tol and w <= tol, (name, p, w)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 17, 64, 100])
@pytest.mark.parametrize("d", [32, 128])
def test_backward_small(dtype, T, d):
    inp = make_form_inputs(2, T, 2, d, d, dtype, 700 + T + d, "channel", state=True)
    check_bwd(inp, 701 + T, final=T % 2 == 0)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (32, 64)])
def test_backward_rectangular(dk, dv):
    check_bwd(make_form_inputs(2, 50, 2, dk, dv, "f32", 710 + dk, "channel", state=True), 711)


@pytest.mark.parametrize("form", ["scalar", "none"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_scalar_and_no_gate(form, dtype):
    check_bwd(make_form_inputs(2, 90, 3, 128, 128, dtype, 720, form, state=True), 721)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_varlen_ragged(dtype):
    cu = [0, 0, 1, 17, 80, 80, 130]
    check_bwd(make_form_inputs(6, 0, 2, 128, 128, dtype, 730, "channel", state=True, cu_seqlens=cu), 731)


def test_backward_extreme_gates():
    inp = make_form_inputs(2, 200, 4, 128, 128, "f32", 740, "channel", state=True, gates="extremes")
    check_bwd(inp, 741)


def test_backward_prefill_shape_sampled():
    """The prefill workload's shape (B=4, T=4096, H=16, 128 x 128, bf16); the oracle
    recomputes 6 sampled (sequence, head) pairs."""
    inp = make_form_inputs(4, 4096, 16, 128, 128, "bf16", 1, "channel")
    check_bwd(inp, 750, tasks=[(0, 0), (1, 5), (2, 9), (3, 15), (0, 12), (3, 3)])


def test_backward_is_deterministic():
    inp = make_form_inputs(2, 300, 4, 128, 128, "bf16", 760, "channel", state=True)
    dO, dSf = grad_inputs(inp, 761)
    a, b = run_bwd(inp, dO, dSf), run_bwd(inp, dO, dSf)
    for name in a:
        np.testing.assert_array_equal(a[name], b[name])


def test_backward_malformed_cu_seqlens_stay_in_bounds():
    """Offsets that are not non-decreasing ([0, T, 0, T]: two clamped sequences over the same
    tokens) ask for more checkpoint blocks than the workspace holds; each sequence's blocks are
    capped to what is left, so the call completes without a device error (its gradients are
    unspecified: two sequences write the same tokens' shares)."""
    from gated_delta_rule_119_b200 import kda_chunk_bwd, kda_device_status
    T, H = 512, 2
    inp = make_form_inputs(1, T, H, 128, 128, "bf16", 780, "channel", state=True)
    t = to_torch(inp)
    packed = {k_: t[k_].reshape(T, *t[k_].shape[2:]) for k_ in ("q", "k", "v", "log_alpha", "beta")}
    dO, _ = grad_inputs(inp, 781, final=False)
    dO_t = storage_to_torch(dO, inp.dtype, "cuda").view(packed["v"].shape)
    cu = torch.tensor([0, T, 0, T], dtype=torch.int32, device="cuda")
    S0 = torch.cat([t["S0"]] * 3)
    g = kda_chunk_bwd(packed["q"], packed["k"], packed["v"], packed["log_alpha"], packed["beta"], dO_t,
                      S0, cu)
    torch.cuda.synchronize()
    assert kda_device_status() == 0
    assert g["dv"].shape == packed["v"].shape
