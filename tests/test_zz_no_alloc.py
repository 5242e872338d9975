"""kda_chunk_fwd_noalloc, called through the C ABI.

The call runs the same kernels on the same inputs as kda_chunk_fwd, only with its
workspace in the fixed scratch buffer, so it must give bit-identical o and S_final on two
calls in a row (the second one reuses the buffer the first one wrote: a stale slot would
show as a difference); and a problem whose workspace does not fit the buffer must be
refused on the host.  This file is collected last so that its GPU
tests also run after everything else in the suite.
"""
import numpy as np
import pytest

from gated_delta_rule_119_b200 import binding
from gated_delta_rule_119_b200.inputs import make_inputs, to_torch

SLOT_BYTES = 66560       # workspace bytes per (chunk, head) of the bf16 128 x 128 path


def rel_err(x, r):
    x, r = np.asarray(x, np.float64), np.asarray(r, np.float64)
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-30))


def test_oversize_refused_on_host():
    """No CUDA call happens before the size check: fake aligned addresses are never used."""
    A = [(i + 1) << 36 for i in range(8)]      # far apart: no spans overlap
    T = 64 * 1009           # 1,009 chunks x 1 head: one slot more than the buffer holds
    rc = binding.chunk_fwd_noalloc_raw(A[0], A[1], A[2], A[3], A[4], 0, 0, A[5], A[6],
                                       1, T, 1, 128, 128, 64, binding.KDA_BF16, 0)
    assert rc == -9
    assert binding.kda_status_string(rc).startswith("KDA_ERR_SCRATCH")
    assert 1008 * SLOT_BYTES + 1024 <= binding.NOALLOC_SCRATCH_BYTES < 1009 * SLOT_BYTES + 1024


CASES = {
    # name: (B, T, H, dk, dv, dtype, seed, state, varlen)
    "bf16_fixed": (2, 1000, 4, 128, 128, "bf16", 901, False, False),
    "bf16_varlen_state": (5, 1500, 3, 128, 128, "bf16", 902, True, True),
    "bf16_at_limit": (1, 4032, 16, 128, 128, "bf16", 903, False, False),
    "f32_no_scratch": (2, 200, 2, 64, 128, "f32", 904, True, False),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_chunk_fwd(name):
    import torch
    B, T, H, dk, dv, dtype, seed, state, varlen = CASES[name]
    inp = make_inputs(B, T, H, dk, dv, dtype, seed, state=state, varlen=varlen)
    d = to_torch(inp)
    ref_o, ref_s = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                         d["S0"], d["cu_seqlens"])
    torch.cuda.synchronize()
    ref_o, ref_s = ref_o.float().cpu().numpy(), ref_s.cpu().numpy()
    code = binding.KDA_BF16 if dtype == "bf16" else binding.KDA_F32
    N = inp.n_seqs
    Bc, Tc = (N, inp.total_tokens) if varlen else (B, T)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: 0 if t is None else t.data_ptr()
    for call in range(2):
        out = torch.full_like(d["v"], float("nan"))
        S_final = torch.full((N, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
        rc = binding.chunk_fwd_noalloc_raw(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]),
                                           ptr(d["log_alpha"]), ptr(d["beta"]), ptr(d["S0"]),
                                           ptr(d["cu_seqlens"]), ptr(out), ptr(S_final), Bc, Tc,
                                           H, dk, dv, 64, code, stream)
        assert rc == 0, binding.kda_status_string(rc)
        torch.cuda.synchronize()
        eo = rel_err(out.float().cpu().numpy(), ref_o)
        es = rel_err(S_final.cpu().numpy(), ref_s)
        print(f"[noalloc] {name} call {call}: o {eo:.3e}  S_final {es:.3e}")
        assert np.array_equal(out.float().cpu().numpy(), ref_o), (call, eo)
        assert np.array_equal(S_final.cpu().numpy(), ref_s), (call, es)
    assert binding.kda_device_status() == 0


@pytest.mark.gpu
def test_noalloc_oversize_refused_with_device_buffers():
    import torch
    inp = make_inputs(1, 64 * 1009, 1, 128, 128, "bf16", 905)
    d = to_torch(inp)
    out = torch.empty_like(d["v"])
    rc = binding.chunk_fwd_noalloc_raw(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(),
                                       d["log_alpha"].data_ptr(), d["beta"].data_ptr(), 0, 0,
                                       out.data_ptr(), 0, 1, 64 * 1009, 1, 128, 128, 64,
                                       binding.KDA_BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == -9
