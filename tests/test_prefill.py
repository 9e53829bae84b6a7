"""GPU parity of kda_chunk_fwd (through the C ABI) with the fp64 oracle.

Small cases compare every element; the full-size workloads (in the launch
configuration the benchmark times) compare sampled (sequence, head) units, which the
oracle computes one by one.  Both the default path (tensor cores for bf16 at
dk = dv = 128) and the fp32 CUDA-core path are covered.
"""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import (TOL_F32, TOL_OUT_BF16, TOL_STATE_BF16, gpu_unit, host, oracle_full,
                               oracle_units, rel_l2)

pytestmark = pytest.mark.gpu

PATHS = {"default": 0, "simt": kda.KDA_FLAG_FORCE_SIMT}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _run(inp, flags=0, norm_weight=None, split=0, eps=1e-6):
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     norm_weight=norm_weight, flags=flags, split_segments=split,
                                     eps=eps)
    st = kda.kda_read_device_error(ws)
    assert st == kda.KDA_OK, kda.kda_status_string(st)
    return out, fin


def _tol(inp):
    if inp.q.dtype == torch.float32:
        return TOL_F32, TOL_F32
    return TOL_OUT_BF16, TOL_STATE_BF16


def test_tiny_fp32_workload():
    """B1 H2 T256 d64 fp32, no output gate, zero initial state: every element <= 1e-4."""
    inp = synth.make_workload("tiny_fp32", device="cuda")
    out, fin = _run(inp)
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_F32
    assert rel_l2(host(fin), f_ref) <= TOL_F32


@pytest.mark.parametrize("split", [0, 3])
@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 128), ("bf16", 64, 128),
                                         ("f32", 64, 64), ("bf16", 128, 64)])
def test_ragged_varlen_small(path, dtype, dk, dv, split):
    """Chunk-boundary edge cases in one packed batch: lengths 0, 1, 15, 16, 17, 63, 64, 65,
    127, 200 with initial states, gate and a norm weight; every element compared.  With a forced
    split of 3 the sequences longer than one chunk are cut into two segments (64 + 1, 64 + 63,
    128 + 72) while the others run whole beside them, the empty one included."""
    lengths = np.array([1, 15, 0, 16, 17, 63, 64, 65, 127, 200])
    inp = synth.make_prefill(H=3, dk=dk, dv=dv, dtype=dtype, seed=31, device="cuda",
                             lengths=lengths, gate=True, init_state=True)
    w = torch.linspace(0.5, 1.5, dv, device="cuda")
    out, fin = _run(inp, flags=PATHS[path], norm_weight=w, split=split)
    o_ref, f_ref = oracle_full(inp, norm_weight=w)
    to, ts = _tol(inp)
    assert rel_l2(host(out), o_ref) <= to
    assert rel_l2(host(fin), f_ref) <= ts
    # the zero-length sequence returns its initial state unchanged
    np.testing.assert_array_equal(host(fin[2]), host(inp.initial_state[2]))
    # each sequence on its own (guards against a small error hidden by a large sequence)
    cu = inp.cu_seqlens
    for n in range(len(lengths)):
        if lengths[n] == 0:
            continue
        sl = slice(cu[n], cu[n + 1])
        assert rel_l2(host(out[sl]), o_ref[sl]) <= to
        assert rel_l2(host(fin[n]), f_ref[n]) <= ts


@pytest.mark.parametrize("path", list(PATHS))
def test_no_gate_no_initial_state(path):
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=32, device="cuda",
                             lengths=np.array([300, 77]), gate=False, init_state=False)
    out, fin = _run(inp, flags=PATHS[path])
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


@pytest.mark.parametrize("path", list(PATHS))
def test_slow_decay_long_carry(path):
    """g = -5 sigmoid(N(0,1) - 6): the state carries over many chunks."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=33, device="cuda",
                             lengths=np.array([1000, 333]), gate=True, init_state=True,
                             decay_shift=-6.0)
    out, fin = _run(inp, flags=PATHS[path])
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("split", [2, 3, 5])
def test_sequence_split_matches_oracle(path, split):
    """Forced split of each sequence into segments (pass 1, combine, pass 2)."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=34, device="cuda",
                             lengths=np.array([700, 64, 1100, 130]), gate=True, init_state=True,
                             decay_shift=-6.0)
    out, fin = _run(inp, flags=PATHS[path], split=split)
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


def test_sequence_split_fp32():
    inp = synth.make_prefill(H=2, dk=64, dv=64, dtype="f32", seed=35, device="cuda",
                             lengths=np.array([400, 190]), gate=True, init_state=True, decay_shift=-6.0)
    out, fin = _run(inp, split=4)
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_F32
    assert rel_l2(host(fin), f_ref) <= TOL_F32


def test_checked_decay_reports_out_of_range():
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=36, device="cuda",
                             lengths=np.array([40]), gate=True)
    inp.g[17, 1, 5] = -5.5
    _, _, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                 cu_seqlens=inp.cu_seqlens, flags=kda.KDA_FLAG_CHECK_DECAY)
    assert kda.kda_read_device_error(ws) == kda.binding.KDA_ERR_DECAY_OUT_OF_RANGE
    assert kda.kda_read_device_error(ws) == kda.KDA_OK  # reading clears it
    inp.g[17, 1, 5] = 0.25
    _, _, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                 cu_seqlens=inp.cu_seqlens, flags=kda.KDA_FLAG_CHECK_DECAY)
    assert kda.kda_read_device_error(ws) == kda.binding.KDA_ERR_DECAY_OUT_OF_RANGE


def test_empty_batch():
    e = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    b = torch.empty((0, 2), dtype=torch.bfloat16, device="cuda")
    out, fin, ws = kda.kda_chunk_fwd(e, e, e, e, b, cu_seqlens=np.array([0, 0, 0]))
    assert out.shape == (0, 2, 128) and fin.shape == (2, 2, 128, 128)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    assert torch.count_nonzero(fin) == 0


# ---------------------------------------------------------------- full-size workloads
def _check_units(inp, out, fin, units, tok_limit=None, check_state=True):
    ref = oracle_units(inp, units, tok_limit=tok_limit)
    for u in units:
        o, f = gpu_unit(out, fin, inp.cu_seqlens, *u, tok_limit=tok_limit)
        assert rel_l2(o, ref[u][0]) <= TOL_OUT_BF16, u
        if check_state:
            assert rel_l2(f, ref[u][1]) <= TOL_STATE_BF16, u


def test_prefill_bf16_full_size():
    """B4 H32 T4096 d128 with gate: 8 sampled (sequence, head) units, outputs and states."""
    inp = synth.make_workload("prefill_bf16", device="cuda")
    out, fin = _run(inp)
    rng = np.random.default_rng(0)
    units = [(int(rng.integers(4)), int(rng.integers(32))) for _ in range(6)] + [(0, 0), (3, 31)]
    _check_units(inp, out, fin, units)


def test_varlen_bf16_full_size():
    """64 sequences of U[128, 8192] tokens, H32, initial states: shortest, longest and
    random units."""
    inp = synth.make_workload("varlen_bf16", device="cuda")
    out, fin = _run(inp)
    lens = np.diff(inp.cu_seqlens)
    rng = np.random.default_rng(1)
    units = [(int(np.argmin(lens)), 3), (int(np.argmax(lens)), 17)]
    units += [(int(rng.integers(64)), int(rng.integers(32))) for _ in range(6)]
    _check_units(inp, out, fin, units)


@pytest.mark.slow
def test_long_context_prefix_and_full_run():
    """B1 H16 T=2^20: (a) a 65,536-token prefix, outputs and final states of 4 heads against the
    oracle; (b) the full run, final states of 2 heads against the oracle."""
    full = synth.make_workload("long_bf16", device="cuda")
    P = 65536
    pre = synth.PrefillInputs(full.q[:P], full.k[:P], full.v[:P], full.g[:P], full.beta[:P],
                              full.gate[:P], None, np.array([0, P]))
    out, fin = _run(pre)
    _check_units(pre, out, fin, [(0, 0), (0, 5), (0, 10), (0, 15)])
    del out, fin
    out, fin = _run(full)
    heads = [(0, 3), (0, 12)]
    ref = oracle_units(full, heads, num_threads=len(heads))
    for u in heads:
        assert rel_l2(fin[u].cpu().numpy(), ref[u][1]) <= TOL_STATE_BF16, u
        o, _ = gpu_unit(out, None, full.cu_seqlens, *u)
        assert rel_l2(o[-4096:], ref[u][0][-4096:]) <= TOL_OUT_BF16, u


def test_forced_timeout_reports_and_recovers():
    """The test-only flag makes the tensor-core kernel's bounded waits give up at once: the call
    reports KDA_ERR_TIMEOUT in the error word, drains its own copies, frees TMEM and returns;
    the next call on the same context is correct."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=37, device="cuda",
                             lengths=np.array([300, 100]), gate=True, init_state=True)
    _, _, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                 cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                 flags=kda.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert kda.kda_read_device_error(ws) == kda.binding.KDA_ERR_TIMEOUT
    out, fin = _run(inp)
    o_ref, f_ref = oracle_full(inp)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


@pytest.mark.parametrize("path", list(PATHS))
def test_varlen_neighbour_nan_does_not_leak(path):
    """Packed sequences are independent.  The middle sequence holds NaN in every input; the last,
    partial chunk of the sequence before it is staged as a full tile that overlaps the NaN rows.
    Its neighbours' outputs and states must stay finite and match the oracle."""
    lengths = np.array([100, 77, 150])
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=38, device="cuda",
                             lengths=lengths, gate=True, init_state=True)
    cu = inp.cu_seqlens
    bad = slice(cu[1], cu[2])
    for t in (inp.q, inp.k, inp.v, inp.g, inp.gate):
        t[bad] = float("nan")
    inp.beta[bad] = float("nan")
    out, fin = _run(inp, flags=PATHS[path])
    for n in (0, 2):
        sl = slice(cu[n], cu[n + 1])
        one = synth.PrefillInputs(inp.q[sl], inp.k[sl], inp.v[sl], inp.g[sl], inp.beta[sl],
                                  inp.gate[sl], inp.initial_state[n:n + 1], np.array([0, lengths[n]]))
        o_ref, f_ref = oracle_full(one)
        assert torch.isfinite(out[sl]).all() and torch.isfinite(fin[n]).all(), n
        assert rel_l2(host(out[sl]), o_ref) <= TOL_OUT_BF16, n
        assert rel_l2(host(fin[n]), f_ref[0]) <= TOL_STATE_BF16, n


_SPLIT_REF = {}


@pytest.mark.parametrize("split", [1, 2, 9, 32])
def test_split_error_against_segment_count(split):
    """One 65,536-token sequence with slow decay (the state carries across segments), two heads:
    the same call cut into 1, 2, 9 and 32 segments.  Each segment boundary adds a combine step
    S_start(q+1) = M_q S_start(q) + S_loc(q) with M_q and S_loc from bf16 tensor-core passes, so
    the error can grow with the segment count; every count must stay within the tolerances
    (outputs of the last 4,096 tokens and of the first 4,096, final states)."""
    T = 65536
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=39, device="cuda",
                             lengths=np.array([T]), gate=True, init_state=True, decay_shift=-6.0)
    if "ref" not in _SPLIT_REF:
        _SPLIT_REF["ref"] = oracle_full(inp, num_threads=2)
    o_ref, f_ref = _SPLIT_REF["ref"]
    out, fin = _run(inp, split=split)
    for sl in (slice(0, 4096), slice(T - 4096, T)):
        assert rel_l2(host(out[sl]), o_ref[sl]) <= TOL_OUT_BF16, (split, sl)
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16, split
