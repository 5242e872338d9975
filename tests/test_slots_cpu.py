"""The varlen slot bookkeeping of the tensor-core prefill, mirrored on the host: whatever
cu_seqlens holds (decreasing, negative or out-of-range entries), every workspace slot the
intra-chunk kernel writes and the scan reads lies inside the workspace, which holds
ceil(T / 64) + N slots per head.

The mirror follows the device code step by step: each sequence's bounds are clamped to
[0, T] (an end below its start is raised to the start); the slot kernel gives sequence n
min(ceil(len_n / 64), slots left) slots from a running sum capped at the workspace size; the
intra kernel maps slot s < base[N] to the last n with base[n] <= s and chunk s - base[n];
the scan walks min(ceil(len_n / 64), base[n + 1] - base[n]) chunks from base[n]."""
import numpy as np

CH = 64


def seq_bounds(cu, n, T):
    a = min(max(int(cu[n]), 0), T)
    b = int(cu[n + 1])
    b = a if b < a else min(b, T)
    return a, b


def slot_table(cu, T):
    N = len(cu) - 1
    max_slots = (T + CH - 1) // CH + N
    base, acc = [], 0
    for n in range(N):
        t0, t1 = seq_bounds(cu, n, T)
        base.append(acc)
        acc += min((t1 - t0 + CH - 1) // CH, max_slots - acc)
    base.append(acc)
    return base, max_slots


def touched_slots(cu, T):
    """Slots written by the intra kernel and read by the scan, per the device code."""
    base, max_slots = slot_table(cu, T)
    N = len(cu) - 1
    written = []
    for s in range(max_slots):                 # the intra grid spans max_slots
        if s >= base[N]:
            continue
        n = max(m for m in range(N) if base[m] <= s)
        ci = s - base[n]
        t0, t1 = seq_bounds(cu, n, T)
        assert t0 + ci * CH < t1                # the chunk has at least one token
        written.append(s)
    read = []
    for n in range(N):
        t0, t1 = seq_bounds(cu, n, T)
        nch = min((t1 - t0 + CH - 1) // CH, base[n + 1] - base[n])
        read += [base[n] + c for c in range(nch)]
    return written, read, max_slots


def test_well_formed_offsets_get_every_chunk():
    rng = np.random.default_rng(0)
    for _ in range(200):
        T = int(rng.integers(0, 5000))
        N = int(rng.integers(1, 20))
        cuts = np.sort(rng.integers(0, T + 1, size=N - 1))
        cu = [0, *cuts.tolist(), T]
        base, max_slots = slot_table(cu, T)
        for n in range(N):                     # no cap: each sequence has all its chunks
            assert base[n + 1] - base[n] == (cu[n + 1] - cu[n] + CH - 1) // CH
        written, read, _ = touched_slots(cu, T)
        assert sorted(written) == sorted(read) == list(range(base[N]))


def test_malformed_offsets_stay_inside_the_workspace():
    rng = np.random.default_rng(1)
    cases = [([0, 4096, 0, 4096], 4096), ([0, 100, 50, 200], 200), ([-50, 10_000, -7, 3], 64),
             ([5000, 0, 5000, 0, 5000], 5000), ([0, 0, 0, 0], 1)]
    for _ in range(300):
        T = int(rng.integers(1, 3000))
        N = int(rng.integers(1, 12))
        cases.append((rng.integers(-T - 10, 2 * T + 10, size=N + 1).tolist(), T))
    capped = 0
    for cu, T in cases:
        written, read, max_slots = touched_slots(cu, T)
        assert all(0 <= s < max_slots for s in written + read), cu
        assert set(read) <= set(written), cu   # the scan reads only slots the intra kernel wrote
        base, _ = slot_table(cu, T)
        want = sum((b - a + CH - 1) // CH for a, b in (seq_bounds(cu, n, T) for n in range(len(cu) - 1)))
        capped += want > base[-1]
    assert capped > 0                          # the cap was exercised


BWD_CH = 16


def bwd_blocks(cu, T):
    """The backward kernel's checkpoint blocks per sequence, per the device code: the workspace
    holds ceil(T / 16) + N blocks per (head, half); sequence n's first block is the running sum
    of the sequences before it, each capped to what is left, and it walks
    min(ceil(len_n / 16), blocks left) chunks from there."""
    N = len(cu) - 1
    max_chunks = (T + BWD_CH - 1) // BWD_CH + N
    out = []
    for n in range(N):
        base = 0
        for m in range(n):
            s0, s1 = seq_bounds(cu, m, T)
            want = (s1 - s0 + BWD_CH - 1) // BWD_CH
            base += min(want, max_chunks - base)
        t0, t1 = seq_bounds(cu, n, T)
        nch = min((t1 - t0 + BWD_CH - 1) // BWD_CH, max_chunks - base)
        out.append((base, nch, t0, t1))
    return out, max_chunks


def test_backward_checkpoints_stay_inside_the_workspace():
    """Whatever cu_seqlens holds, every checkpoint block the backward writes or reads lies inside
    its workspace and every token it touches inside [0, T); well-formed offsets get all their
    chunks, each sequence its own blocks."""
    rng = np.random.default_rng(2)
    cases = [([0, 4096, 0, 4096], 4096), ([0, 100, 50, 200], 200), ([-50, 10_000, -7, 3], 64),
             ([5000, 0, 5000, 0, 5000], 5000), ([0, 0, 0, 0], 1)]
    for _ in range(300):
        T = int(rng.integers(1, 3000))
        N = int(rng.integers(1, 12))
        cases.append((rng.integers(-T - 10, 2 * T + 10, size=N + 1).tolist(), T))
    for cu, T in cases:
        blocks, max_chunks = bwd_blocks(cu, T)
        for base, nch, t0, t1 in blocks:
            assert 0 <= base and nch >= 0 and base + nch <= max_chunks
            for ci in range(nch):
                c0 = t0 + ci * BWD_CH
                assert 0 <= c0 < t1 <= T               # the chunk's tokens are in [0, T)
    for _ in range(200):
        T = int(rng.integers(0, 3000))
        N = int(rng.integers(1, 12))
        cuts = np.sort(rng.integers(0, T + 1, size=N - 1))
        cu = [0, *cuts.tolist(), T]
        blocks, _ = bwd_blocks(cu, T)
        used = []
        for n, (base, nch, t0, t1) in enumerate(blocks):
            assert nch == (cu[n + 1] - cu[n] + BWD_CH - 1) // BWD_CH
            used += list(range(base, base + nch))
        assert len(used) == len(set(used))               # no block shared by two sequences
