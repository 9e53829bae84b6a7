"""GPU parity of the chunk-boundary state snapshots (prefix caching) with the fp64 oracle.

kda_chunk_fwd with a snapshot buffer writes the state after every multiple of the interval of
every sequence; the oracle records the same states in its sequential loop.  Covered: ragged varlen
batches on both kernels, boundaries inside split segments, the fp32 path, resuming a sequence from
a snapshot, and sampled units of the full-size workload in the benchmark's launch configuration.
"""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
import oracle
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import (TOL_F32, TOL_OUT_BF16, TOL_STATE_BF16, host, oracle_full, oracle_units,
                               rel_l2)

pytestmark = pytest.mark.gpu

PATHS = {"default": 0, "simt": kda.KDA_FLAG_FORCE_SIMT}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _run(inp, interval, flags=0, split=0, extra_rows=2):
    """Prefill with snapshots into a NaN-filled buffer with extra_rows spare rows."""
    rows = kda.snapshot_count(inp.q, inp.v, interval, cu_seqlens=inp.cu_seqlens)
    H, dk, dv = inp.q.shape[1], inp.q.shape[2], inp.v.shape[2]
    snaps = torch.full((rows + extra_rows, H, dk, dv), float("nan"), device="cuda")
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     flags=flags, split_segments=split, snapshots=snaps,
                                     snapshot_interval=interval)
    st = kda.kda_read_device_error(ws)
    assert st == kda.KDA_OK, kda.kda_status_string(st)
    return out, fin, snaps, rows


def _oracle_snaps(inp, interval):
    a = {n: host(getattr(inp, n)) for n in ("q", "k", "v", "g", "beta", "gate")}
    s0 = None if inp.initial_state is None else inp.initial_state.double().cpu().numpy()
    return oracle.forward_snapshots(a["q"], a["k"], a["v"], a["g"], a["beta"], interval,
                                    cu_seqlens=inp.cu_seqlens, gate=a["gate"], initial_state=s0)


def _check(inp, interval, flags=0, split=0):
    out, fin, snaps, rows = _run(inp, interval, flags=flags, split=split)
    o_ref, f_ref, s_ref = _oracle_snaps(inp, interval)
    assert s_ref.shape[0] == rows
    ts = TOL_F32 if inp.q.dtype == torch.float32 else TOL_STATE_BF16
    to = TOL_F32 if inp.q.dtype == torch.float32 else TOL_OUT_BF16
    got = host(snaps)
    for r in range(rows):  # every snapshot row on its own
        assert rel_l2(got[r], s_ref[r]) <= ts, r
    assert np.isnan(got[rows:]).all()  # rows past the last snapshot untouched
    # the outputs and final states are unchanged by the snapshots
    assert rel_l2(host(out), o_ref) <= to
    assert rel_l2(host(fin), f_ref) <= ts
    return out, fin, snaps


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("interval", [64, 192])
def test_snapshots_ragged_varlen(path, interval):
    """Lengths 64, 200, 0, 130, 1000, 20, 256 (a boundary at a sequence end, inside, none at all)
    with initial states and the gate."""
    lengths = np.array([64, 200, 0, 130, 1000, 20, 256])
    inp = synth.make_prefill(H=3, dk=128, dv=128, dtype="bf16", seed=41, device="cuda",
                             lengths=lengths, gate=True, init_state=True)
    _, fin, snaps = _check(inp, interval, flags=PATHS[path])
    # a snapshot at the end of a sequence is that sequence's final state, bit for bit
    cu = inp.cu_seqlens
    row = 0
    for n, L in enumerate(lengths):
        k = L // interval
        if k and L % interval == 0:
            torch.testing.assert_close(snaps[row + k - 1], fin[n], rtol=0, atol=0)
        row += k


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("split", [2, 3])
def test_snapshots_in_split_segments(path, split):
    """Forced sequence split: the boundaries fall in the head and in carried-state segments."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=42, device="cuda",
                             lengths=np.array([1000, 700]), gate=True, init_state=True)
    _check(inp, 128, flags=PATHS[path], split=split)


def test_snapshots_fp32():
    inp = synth.make_prefill(H=2, dk=64, dv=64, dtype="f32", seed=43, device="cuda",
                             lengths=np.array([256, 100, 64]), gate=False, init_state=True)
    _check(inp, 64)


@pytest.mark.parametrize("path", list(PATHS))
def test_resume_from_snapshot(path):
    """Prefix caching: the tokens after a snapshot, run from that snapshot as the initial state,
    give the same outputs and final state as the uninterrupted run (both against the oracle)."""
    inp = synth.make_prefill(H=4, dk=128, dv=128, dtype="bf16", seed=44, device="cuda",
                             lengths=np.array([640]), gate=True, init_state=True)
    out, fin, snaps, rows = _run(inp, 256, flags=PATHS[path], extra_rows=0)
    assert rows == 2
    o_ref, f_ref = oracle_full(inp)
    p = 256
    tail = {n: getattr(inp, n)[p:].contiguous() for n in ("q", "k", "v", "g", "beta", "gate")}
    out2, fin2, ws = kda.kda_chunk_fwd(tail["q"], tail["k"], tail["v"], tail["g"], tail["beta"],
                                       gate=tail["gate"], cu_seqlens=[0, 640 - p],
                                       initial_state=snaps[0:1].contiguous(), flags=PATHS[path])
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    assert rel_l2(host(out2), o_ref[p:]) <= TOL_OUT_BF16
    assert rel_l2(host(fin2), f_ref) <= TOL_STATE_BF16


def test_snapshots_full_size_sampled():
    """B4 H32 T4096 (the benchmark's prefill batch and launch configuration) with a snapshot every
    1024 tokens: sampled units against the oracle on the prefix, the last snapshot of every
    sequence equal to its final state."""
    inp = synth.make_workload("prefill_bf16", device="cuda")
    interval = 1024
    rows = kda.snapshot_count(inp.q, inp.v, interval, cu_seqlens=inp.cu_seqlens)
    assert rows == 4 * 4
    H = inp.q.shape[1]
    snaps = torch.empty((rows, H, 128, 128), device="cuda")
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     snapshots=snaps, snapshot_interval=interval)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    for n in range(4):
        torch.testing.assert_close(snaps[4 * n + 3], fin[n], rtol=0, atol=0)
    units = [(0, 0), (1, 17), (3, 31)]
    for k in (1, 2):  # snapshots after 1024 and 2048 tokens
        ref = oracle_units(inp, units, tok_limit=k * interval)
        for (n, h) in units:
            assert rel_l2(host(snaps[4 * n + k - 1, h]), ref[(n, h)][1]) <= TOL_STATE_BF16
