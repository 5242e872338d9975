"""The end-to-end path of bench.py: the sequences in groups on three streams (copies in, the
calls, copies out).  Every (sequence, head) pair is computed by the same kernels whatever the
batch around it, so the grouped calls must return exactly what one call over the whole batch
returns; a missing wait between the streams would show up as stale or partial results."""
import os
import sys
from types import SimpleNamespace

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["prefill", "varlen"])
def test_grouped_e2e_equals_one_call(name):
    import torch
    import bench
    from gated_delta_rule_119_b200 import kda_chunk_fwd
    device = torch.device("cuda", 0)
    args = SimpleNamespace(steps=3, e2e_steps=3)
    res, host, out_host, S_host = bench.run_e2e(args, name, device, torch.cuda.current_stream(device), 0,
                                                return_outputs=True)
    assert res["value"] > 0 and res["h2d_bytes_per_step"] > 0 and res["d2h_bytes_per_step"] > 0
    d = {k: (None if t is None else t.to(device)) for k, t in host.items()}
    o, Sf = kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"])
    torch.cuda.synchronize()
    assert torch.equal(out_host, o.cpu())
    assert torch.equal(S_host, Sf.cpu())


def test_grouped_e2e_decode_equals_one_call():
    """Decode keeps the state on the device; the last grouped step's o equals a direct step
    taken from the same state."""
    import torch
    import bench
    from gated_delta_rule_119_b200 import kda_decode_step
    device = torch.device("cuda", 0)
    args = SimpleNamespace(steps=1, e2e_steps=1)
    res, host, out_host, S_host = bench.run_e2e(args, "decode", device, torch.cuda.current_stream(device), 0,
                                                return_outputs=True)
    assert res["value"] > 0
    # run_e2e took two steps (one untimed, one timed) from S_host: replay them directly
    S = S_host.to(device)
    d = {k: (None if t is None else t.to(device)) for k, t in host.items()}
    for _ in range(2):
        o = kda_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S)
    torch.cuda.synchronize()
    assert torch.equal(out_host, o.cpu())
