"""GPU behaviour of the C ABI beyond single-call parity: calls on a side stream, run-to-run
determinism of the tensor-core prefill, many heads with short sequences, one sequence split
into several calls (S_final fed back as S0), concurrent calls from several host threads.
All through libkda.so; oracle values where a value is checked (max|x - r| / max|r| within
the dtype's bar)."""
import numpy as np
import pytest

import oracle
from gated_delta_rule_119_b200.inputs import make_inputs, to_torch

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(x, r):
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def call(d, **kw):
    from gated_delta_rule_119_b200 import kda_chunk_fwd
    return kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                         d["cu_seqlens"], **kw)


def test_side_stream_gives_the_default_stream_result():
    inp = make_inputs(2, 700, 4, 128, 128, "bf16", 1201, state=True)
    d = to_torch(inp)
    o_ref, s_ref = call(d)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o, s = call(d)
    side.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0


@pytest.mark.parametrize("gates", ["default", "extremes", "clear"])
def test_tensor_core_path_is_deterministic(gates):
    """Three calls give bit-identical results.  "clear" puts log_alpha = -1e4 on whole heads
    and on scattered tokens, so that blocks take the exact per-channel path (decay spread
    beyond the rescaled factors' range) beside the fast and the block paths."""
    inp = make_inputs(2, 1000, 4, 128, 128, "bf16", 1202, state=True,
                      gates="default" if gates == "clear" else gates)
    if gates == "clear":
        inp.log_alpha[:, 0] = -1e4
        inp.log_alpha[::5, 1, ::3] = -1e4
        inp.log_alpha[3::11, 2] = -1e4
    d = to_torch(inp)
    outs = [call(d) for _ in range(3)]
    torch.cuda.synchronize()
    for o, s in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(s, outs[0][1])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_many_heads_short_sequences(dtype):
    inp = make_inputs(3, 70, 64, 128, 128, dtype, 1203, state=True)
    d = to_torch(inp)
    o, s = call(d)
    torch.cuda.synchronize()
    ro, rs = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, inp.offsets())
    o = o.float().cpu().numpy().reshape(inp.total_tokens, inp.H, inp.dv)
    eo, es = rel_err(o, ro), rel_err(s.cpu().numpy(), rs)
    print(f"[behaviour] many heads {dtype}: o {eo:.3e}  S_final {es:.3e}")
    assert eo <= TOL[dtype] and es <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sequence_split_across_calls(dtype):
    """Prefill of tokens [0, 300) then [300, 700) with the first call's S_final as the
    second's S0 equals one call over [0, 700) (both checked against the oracle)."""
    full = make_inputs(1, 700, 3, 128, 128, dtype, 1204, state=True)
    cut = 300

    def part(lo, hi, S0):
        p = make_inputs(1, hi - lo, 3, 128, 128, dtype, 1204)
        for name in ("q", "k", "v", "log_alpha", "beta"):
            setattr(p, name, np.ascontiguousarray(getattr(full, name)[lo:hi]))
        p.S0 = S0
        return p

    first = part(0, cut, full.S0)
    d1 = to_torch(first)
    o1, s1 = call(d1)
    second = part(cut, 700, s1.cpu().numpy())
    d2 = to_torch(second)
    o2, s2 = call(d2)
    torch.cuda.synchronize()
    ro, rs = oracle.recurrent_full(full.q, full.k, full.v, full.log_alpha, full.beta, full.S0,
                                   full.offsets())
    o = np.concatenate([o1.float().cpu().numpy().reshape(cut, 3, 128),
                        o2.float().cpu().numpy().reshape(700 - cut, 3, 128)])
    eo, es = rel_err(o, ro), rel_err(s2.cpu().numpy(), rs)
    print(f"[behaviour] split {dtype}: o {eo:.3e}  S_final {es:.3e}")
    assert eo <= TOL[dtype] and es <= TOL[dtype]


def test_bounded_wait_selftest_reports_timeout_and_context_survives():
    """A wait that nothing ends gives up after its limit: kda_device_status() reports
    KDA_ERR_TIMEOUT once, then clears, and the next prefill still runs and matches."""
    from gated_delta_rule_119_b200 import kda_device_status, kda_selftest_wait_timeout
    assert kda_device_status() == 0
    assert kda_selftest_wait_timeout(2000) == 0
    assert kda_device_status() == -8
    assert kda_device_status() == 0
    inp = make_inputs(1, 200, 2, 128, 128, "bf16", 1205, state=True)
    o, s = call(to_torch(inp))
    torch.cuda.synchronize()
    ro, rs = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, inp.offsets())
    o = o.float().cpu().numpy().reshape(inp.total_tokens, inp.H, inp.dv)
    assert rel_err(o, ro) <= TOL["bf16"] and rel_err(s.cpu().numpy(), rs) <= TOL["bf16"]
    assert kda_device_status() == 0


def test_concurrent_host_threads_match_sequential_calls():
    """Four host threads, each with its own stream and problem (fixed-length and varlen,
    bf16 tensor-core path and fp32 SIMT path), call the library at the same time: every
    result equals the one the same call gives alone.  The ctypes call releases the GIL, so
    the calls really overlap on the host, set-up included."""
    import threading
    cases = [make_inputs(2, 900, 4, 128, 128, "bf16", 1206, state=True),
             make_inputs(3, 1500, 2, 128, 128, "bf16", 1207, state=True, varlen=True),
             make_inputs(1, 650, 3, 128, 128, "bf16", 1208, gates="extremes"),
             make_inputs(2, 300, 2, 64, 64, "f32", 1209, state=True)]
    data = [to_torch(c) for c in cases]
    alone = [call(d) for d in data]
    torch.cuda.synchronize()
    results, errors = [None] * len(data), []
    start = threading.Barrier(len(data))

    def worker(i):
        try:
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            start.wait()
            with torch.cuda.stream(st):
                outs = [call(data[i]) for _ in range(3)]
            st.synchronize()
            results[i] = outs
        except Exception as exc:      # reported below, with the thread's case
            errors.append((i, repr(exc)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(data))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    for (o_ref, s_ref), outs in zip(alone, results):
        for o, s in outs:
            assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    from gated_delta_rule_119_b200 import kda_device_status
    assert kda_device_status() == 0


def test_malformed_cu_seqlens_stay_in_bounds():
    """Offsets that are not non-decreasing ([0, T, 0, T]: two clamped sequences of T tokens
    over the same tokens) ask for more workspace slots than the call holds; the slot table
    caps them, so the call completes without a device error.  Results of such a call are
    unspecified except that the first sequence, whose slots come first, is still exact."""
    T, H = 2048, 2
    inp = make_inputs(1, T, H, 128, 128, "bf16", 1290, state=True)
    from gated_delta_rule_119_b200 import kda_chunk_fwd, kda_device_status
    d = to_torch(inp)
    packed = {k_: d[k_].reshape(T, *d[k_].shape[2:]) for k_ in ("q", "k", "v", "log_alpha", "beta")}
    cu = torch.tensor([0, T, 0, T], dtype=torch.int32, device="cuda")
    S0 = torch.cat([d["S0"]] * 3)
    o, S = kda_chunk_fwd(packed["q"], packed["k"], packed["v"], packed["log_alpha"],
                         packed["beta"], S0, cu)
    torch.cuda.synchronize()
    assert kda_device_status() == 0
    _, rs = oracle.recurrent_full(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0,
                                  inp.offsets())
    assert rel_err(S[0].cpu().numpy(), rs[0]) <= TOL["bf16"]
    np.testing.assert_array_equal(S[1].cpu().numpy(), inp.S0[0])     # the empty sequence
