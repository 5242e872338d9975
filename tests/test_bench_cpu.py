"""bench.py's command-line contract where no GPU is needed: the reference arm (the fp64
oracle on the host cores) prints one JSON line with the keys the driver reads, ranks other
than 0 print nothing, and too few warm-up steps are refused."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def run_bench(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, BENCH, *args], capture_output=True, text=True,
                          cwd=ROOT, env=env, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    import oracle
    oracle.build()
    r = run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1", "--warmup", "3",
                   "--ref-step-budget", "0.2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny_f32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1", "--warmup", "3"],
                  env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("impl", ["ours", "reference"])
def test_too_few_warmup_steps_are_refused(impl):
    r = run_bench(["--impl", impl, "--warmup", "2"])
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr


def test_sample_parity_reports_the_max_relative_error():
    """The bench's parity check on the CPU-baseline sample: max|x - r| / max|r| over the
    sampled pairs together and for the worst pair on its own, and a failure to read the GPU
    side reported in the line instead of raised."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    rng = np.random.default_rng(5)
    tasks = [(0, 0), (0, 1), (1, 0)]
    outs = [rng.normal(size=(4, 3)) for _ in tasks]
    outs[1] *= 0.1                                   # a pair with small outputs of its own
    states = [rng.normal(size=(2, 3)) for _ in tasks]
    o_scale = max(np.abs(o).max() for o in outs)
    perturbed = {t: (o + (0.5e-3 * o_scale if t == (0, 1) else 0.0), s * (1 + 1e-3))
                 for t, o, s in zip(tasks, outs, states)}
    p = bench.sample_parity(tasks, outs, states, lambda n, h: perturbed[(n, h)], "bf16")
    assert abs(p["o_max_rel_err"] - 0.5e-3) < 1e-12
    assert abs(p["S_final_max_rel_err"] - 1e-3) < 1e-12
    # the worst pair on its own: pair (0, 1)'s shift relative to its own largest |o|
    assert abs(p["o_worst_pair_rel_err"] - 0.5e-3 * o_scale / np.abs(outs[1]).max()) < 1e-12
    assert p["o_worst_pair_rel_err"] > p["o_max_rel_err"]
    assert abs(p["S_final_worst_pair_rel_err"] - 1e-3) < 1e-12
    assert p["pass"] is True and p["bar"] == 2e-2 and p["pairs"] == 3
    assert bench.sample_parity(tasks, outs, states, lambda n, h: (outs[0] * 2, states[0]), "f32")["pass"] is False

    def broken(n, h):
        raise RuntimeError("no device")
    assert "error" in bench.sample_parity(tasks, outs, states, broken, "bf16")


def test_cpu_baseline_parity_of_the_oracle_against_itself_is_zero():
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    from gated_delta_rule_119_b200.inputs import make_inputs
    oracle.build()
    inp = make_inputs(2, 40, 2, 32, 32, "f32", 77, state=True, varlen=True)
    cu = inp.offsets()
    pairs = [(n, h) for n in range(inp.n_seqs) for h in range(inp.H)]
    outs, states = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.S0, cu,
                                    tasks=pairs)
    ref = {t: (o, s) for t, o, s in zip(pairs, outs, states)}
    cb = bench.cpu_baseline(inp, 0.2, lambda n, h: ref[(n, h)])
    assert cb["parity"]["o_max_rel_err"] == 0.0 and cb["parity"]["S_final_max_rel_err"] == 0.0
    assert cb["parity"]["pass"] is True and cb["kind"] == "oracle"


def test_decode_parity_pairs_replay_the_steps_on_a_copy_of_the_state():
    """decode_pairs runs the given decode steps from the initial state on a copy and returns,
    per (sequence, head), the o of every step and the state after them (a stand-in step on
    CPU tensors here: S += 1 per step, o = row sums of S)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import bench

    def fake_step(q, k, v, log_alpha, beta, S):
        S += 1.0
        return S.sum(dim=2)
    S0 = np.arange(2 * 3 * 4 * 5, dtype=np.float32).reshape(2, 3, 4, 5)
    dev_in = [dict(q=None, k=None, v=None, log_alpha=None, beta=None) for _ in range(3)]
    pair = bench.decode_pairs(dev_in, S0, torch.device("cpu"), fake_step)
    o, S = pair(1, 2)
    assert o.shape == (3, 5) and S.shape == (4, 5)
    np.testing.assert_allclose(S, S0[1, 2] + 3)
    np.testing.assert_allclose(o[0], (S0[1, 2] + 1).sum(0))
    assert S0[1, 2, 0, 0] == 1 * 60 + 2 * 20          # the initial state is untouched


def test_prefill_parity_pairs_index_the_packed_token_axis():
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import bench
    from gated_delta_rule_119_b200.inputs import make_inputs
    inp = make_inputs(3, 50, 2, 32, 32, "f32", 78, varlen=True)
    cu = inp.offsets()
    out = torch.arange(inp.total_tokens * 2 * 32, dtype=torch.float32).view(inp.total_tokens, 2, 32)
    Sf = torch.randn(3, 2, 32, 32)
    o, S = bench.prefill_pairs(out, Sf, inp)(2, 1)
    np.testing.assert_array_equal(o, out[cu[2]:cu[3], 1].numpy())
    np.testing.assert_array_equal(S, Sf[2, 1].numpy())
    fixed = make_inputs(2, 7, 3, 32, 32, "f32", 79)
    out4 = torch.randn(2, 7, 3, 32)                    # the [B, T, H, dv] view of a fixed-length call
    o, _ = bench.prefill_pairs(out4, torch.zeros(2, 3, 32, 32), fixed)(1, 2)
    np.testing.assert_array_equal(o, out4[1, :, 2].numpy())


def test_decode_variant_oracle_replays_each_sequences_tokens_in_order():
    """cpu_baseline_decode_ex packs, per sequence, the L tokens of every call in call order and
    starts from that sequence's state; checked against the oracle run by hand on one pair."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    from gated_delta_rule_119_b200.inputs import make_decode_state, make_form_inputs
    oracle.build()
    N, L, H, d = 3, 2, 2, 32
    ins = [make_form_inputs(N, L, H, d, d, "f32", (9, c), "fused", raw=True) for c in range(2)]
    S0 = make_decode_state(N, H, d, d, 9)
    n, h = 2, 1
    views = [bench.oracle_view(i) for i in ins]
    pick = lambda name: np.concatenate([np.asarray(getattr(v, name))[n * L:(n + 1) * L, h:h + 1]
                                        for v in views])
    ro, rs = oracle.recurrent_full(pick("q"), pick("k"), pick("v"), pick("log_alpha"), pick("beta"),
                                   S0[n:n + 1, h:h + 1].copy())
    cb = bench.cpu_baseline_decode_ex(ins, S0, L, 0.05, lambda a, b: (ro[:, 0], rs[0, 0]))
    assert cb["kind"] == "oracle" and cb["value"] > 0 and "parity" in cb
    # the function's packing of that pair equals the hand-built token stream
    outs, states = oracle.recurrent(*[np.stack([np.asarray(getattr(v, x)).reshape(N, L, *np.shape(getattr(v, x))[1:])
                                                for v in views], 1).reshape(N * 2 * L, *np.shape(getattr(views[0], x))[1:])
                                      for x in ("q", "k", "v", "log_alpha", "beta")],
                                    S0, np.arange(N + 1) * 2 * L, tasks=[(n, h)])
    np.testing.assert_allclose(outs[0], ro[:, 0], rtol=0, atol=0)
    np.testing.assert_allclose(states[0], rs[0, 0], rtol=0, atol=0)


def test_oracle_view_applies_the_gate_front_end():
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from oracle import gates
    from gated_delta_rule_119_b200.inputs import make_form_inputs
    inp = make_form_inputs(2, 20, 2, 32, 32, "bf16", 10, "fused", raw=True)
    v = bench.oracle_view(inp)
    np.testing.assert_array_equal(v.log_alpha, gates.fused_log_alpha(inp.f, inp.A_log, inp.dt_bias))
    np.testing.assert_allclose(np.linalg.norm(v.k, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_array_equal(v.beta, gates.sigmoid(inp.beta))
    s = make_form_inputs(2, 20, 2, 32, 32, "f32", 11, "scalar")
    assert bench.oracle_view(s).log_alpha.shape == (40, 2, 32)


@pytest.mark.parametrize("N", [1, 3, 4, 8, 9])
def test_e2e_groups_partition_the_batch(N):
    """The end-to-end path's groups cover every sequence once, in order, and (packed tokens)
    every token once, each group's cu_seqlens rebased to start at 0 with its own lengths."""
    sys.path.insert(0, ROOT)
    import bench
    rng = np.random.default_rng(N)
    lens = rng.integers(0, 50, size=N)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    for packed in (False, True):
        groups = bench.e2e_groups(N, cu if packed else None)
        assert 1 <= len(groups) <= 4
        assert groups[0][0] == 0 and groups[-1][1] == N
        for (a0, a1, _, _), (b0, b1, _, _) in zip(groups, groups[1:]):
            assert a1 == b0 and a0 < a1
        for b0, b1, sl, cg in groups:
            if not packed:
                assert (sl.start, sl.stop) == (b0, b1) and cg is None
            else:
                assert (sl.start, sl.stop) == (int(cu[b0]), int(cu[b1]))
                assert cg.dtype == np.int32 and cg[0] == 0 and len(cg) == b1 - b0 + 1
                np.testing.assert_array_equal(np.diff(cg), lens[b0:b1])
