"""The C ABI without a GPU: the library loads, exports every symbol that
include/kda.h declares, and rejects bad arguments on the host (every case
below fails validation before anything could be launched)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_119_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        s = binding.kda_status_string(code)
        assert s and (code == -7 or s.startswith(name)), (code, s)
    assert binding.kda_status_string(12345) == "unknown kda status"


# Fake, 16-byte aligned "device" addresses: never dereferenced, because every
# call below is rejected by host-side validation first.
A = [0x10000 * (i + 1) for i in range(12)]
BIG = 1 << 40


def chunk(**kw):
    args = dict(q=A[0], k=A[1], v=A[2], log_alpha=A[3], beta=A[4], S0=0, cu_seqlens=0,
                out=A[5], S_final=A[6], B=1, T=64, H=1, dk=128, dv=128, C=64, dtype=1,
                stream=0)
    args.update(kw)
    return binding.chunk_fwd_raw(**args)


def decode(**kw):
    args = dict(q=A[0], k=A[1], v=A[2], log_alpha=A[3], beta=A[4], S_inout=BIG, out=A[5],
                N=1, H=1, dk=128, dv=128, dtype=1, stream=0)
    args.update(kw)
    return binding.decode_step_raw(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(v=0), -1), (dict(log_alpha=0), -1),
    (dict(beta=0), -1), (dict(out=0), -1), (dict(q=0, cu_seqlens=A[8], T=5, B=2), -1),
    (dict(dtype=2), -5), (dict(dtype=-1), -5),
    (dict(B=0), -2), (dict(H=0), -2), (dict(T=-1), -2), (dict(dk=96), -2), (dict(dv=16), -2),
    (dict(dk=256), -2),
    (dict(C=32), -3), (dict(C=128), -3),
    (dict(q=A[0] + 8), -4), (dict(out=A[5] + 2), -4), (dict(S0=A[7] + 4), -4),
    (dict(cu_seqlens=A[8] + 4), -4),
    (dict(out=A[0]), -6), (dict(out=A[1] + 16), -6), (dict(S_final=A[3]), -6),
    (dict(S0=A[7], S_final=A[7] + 16), -6),
])
def test_chunk_fwd_rejects(lib, kw, code):
    assert chunk(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(S_inout=0), -1), (dict(out=0), -1),
    (dict(dtype=7), -5), (dict(N=0), -2), (dict(H=-3), -2), (dict(dk=48), -2),
    (dict(k=A[1] + 2), -4), (dict(S_inout=BIG + 8), -4),
    (dict(out=A[2]), -6), (dict(S_inout=A[4]), -6), (dict(out=BIG + 64), -6),
])
def test_decode_step_rejects(lib, kw, code):
    assert decode(**kw) == code


def test_product_path_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="libkda.so not found"):
        binding.load_library(str(tmp_path / "libkda.so"))


@pytest.mark.parametrize("limit_us", [0, -5, 1000001])
def test_wait_selftest_rejects_out_of_range_limits(lib, limit_us):
    assert binding.kda_selftest_wait_timeout(limit_us) == -2      # KDA_ERR_DIM, before any CUDA call


def chunk_ex(**kw):
    args = dict(q=A[0], k=A[1], v=A[2], gate_kind=0, gate=A[3], A_log=0, dt_bias=0, flags=0,
                beta=A[4], S0=0, cu_seqlens=0, out=A[5], S_final=A[6], B=1, T=64, H=1, dk=128,
                dv=128, C=64, dtype=1, stream=0)
    args.update(kw)
    return binding.chunk_fwd_ex_raw(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(gate_kind=4), -10), (dict(gate_kind=-1), -10), (dict(flags=8), -10),
    (dict(gate_kind=2), -10),                               # no decay, yet a gate tensor
    (dict(gate=0), -10), (dict(gate_kind=1, gate=0), -10),  # a decay form without its tensor
    (dict(gate_kind=3), -10), (dict(gate_kind=3, A_log=A[9]), -10),   # fused without A_log / dt_bias
    (dict(gate_kind=3, A_log=A[9], dt_bias=A[10] + 4), -4),
    (dict(q=0), -1), (dict(beta=0), -1), (dict(dtype=3), -5), (dict(C=16), -3),
    (dict(out=A[3]), -6), (dict(gate_kind=3, A_log=A[9], dt_bias=A[10], S_final=A[9]), -6),
    (dict(gate_kind=1, gate=A[3], out=A[3] + 16), -6),
])
def test_chunk_fwd_ex_rejects(lib, kw, code):
    assert chunk_ex(**kw) == code


def decode_ex(**kw):
    args = dict(q=A[0], k=A[1], v=A[2], gate_kind=0, gate=A[3], A_log=0, dt_bias=0, flags=0,
                beta=A[4], state_pool=BIG, state_idx=0, out=A[5], N=1, L=1, H=1, dk=128, dv=128,
                P=1, dtype=1, stream=0)
    args.update(kw)
    return binding.decode_ex_raw(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(L=0), -2), (dict(P=0), -2), (dict(N=2, P=1), -2),       # slot n needs P >= N
    (dict(gate_kind=7), -10), (dict(gate_kind=2), -10), (dict(gate=0), -10),
    (dict(gate_kind=3), -10), (dict(flags=16), -10),
    (dict(state_pool=0), -1), (dict(state_idx=A[8] + 4, N=2, P=1), -4),
    (dict(out=A[3]), -6), (dict(state_pool=A[4]), -6), (dict(state_idx=BIG + 64, N=2, P=4), -6),
    (dict(out=BIG + 128), -6),
])
def test_decode_ex_rejects(lib, kw, code):
    assert decode_ex(**kw) == code


def test_new_status_strings(lib):
    assert binding.kda_status_string(-10).startswith("KDA_ERR_GATE")
    assert binding.kda_status_string(-11).startswith("KDA_ERR_INDEX")


def chunk_bwd(**kw):
    args = dict(q=A[0], k=A[1], v=A[2], gate_kind=0, gate=A[3], beta=A[4], S0=0, cu_seqlens=0,
                dO=A[5], dS_final=0, dq=A[6], dk=A[7], dv=A[8], dgate=A[9], dbeta=A[10], dS0=0,
                B=1, T=64, H=1, dk_=128, dv_=128, C=64, dtype=1, stream=0)
    args.update(kw)
    return binding.chunk_bwd_raw(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(gate_kind=3), -10), (dict(gate_kind=5), -10), (dict(gate=0), -10),
    (dict(dO=0), -1), (dict(dq=0), -1), (dict(dbeta=0), -1), (dict(dgate=0), -1),
    (dict(dq=A[6] + 2), -4), (dict(C=32), -3), (dict(dk_=48), -2), (dict(dtype=4), -5),
    (dict(dq=A[0]), -6), (dict(dv=A[5]), -6), (dict(dk=A[6] + 64), -6), (dict(dS0=A[3]), -6),
])
def test_chunk_bwd_rejects(lib, kw, code):
    assert chunk_bwd(**kw) == code


def test_chunk_bwd_no_gate_needs_no_gate_gradient(lib):
    """Without decay the gate gradient may be NULL (the call then fails only later, on the
    fake addresses, which this host-side test never reaches: KDA_ERR_GATE for a gate given)."""
    assert chunk_bwd(gate_kind=2, gate=A[3]) == -10
