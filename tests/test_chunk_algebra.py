"""The chunkwise algebra the GPU kernels implement equals the sequential oracle.

tests/chunk_model.py restates the chunk form (decayed Gram blocks with 16-token
sub-tile reference points, UT inverse, W/U, output and state carry) in numpy
fp64.  In exact arithmetic it must equal the oracle to rounding; with the
operands rounded to bf16 it must stay inside the parity tolerances, which is the
error budget of the tensor-core design.
"""
import numpy as np
import pytest

import oracle
from linear_attention_serving_rule_b200 import synth
from tests import chunk_model as cm


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _inputs(lengths, dk, dv, seed, dtype="f32", decay_shift=0.0):
    inp = synth.make_prefill(H=2, dk=dk, dv=dv, dtype=dtype, seed=seed, lengths=np.array(lengths),
                             gate=False, init_state=True, decay_shift=decay_shift)
    a = {n: getattr(inp, n).float().numpy() for n in ("q", "k", "v", "g", "beta")}
    return a, inp.initial_state.double().numpy(), inp.cu_seqlens


@pytest.mark.parametrize("C", [16, 64])
def test_chunk_form_equals_oracle(C):
    a, s0, cu = _inputs([1, 15, 16, 17, 63, 64, 65, 150], 32, 24, seed=21)
    o_ref, f_ref = oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                                  initial_state=s0)
    o, f = cm.chunk_forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu, S0=s0, C=C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f, f_ref, rtol=1e-10, atol=1e-12)


def test_subtile_factors_stay_in_bf16_range():
    """With g >= -5 every row factor is <= 1 and every column factor <= e^80 < bf16 max."""
    a, _, _ = _inputs([64], 128, 128, seed=22, dtype="bf16")
    g = np.maximum(a["g"][:, 0], -5.0)
    gam = np.cumsum(g, axis=0)
    ref = np.concatenate([np.zeros((1, 128)), gam[15:63:16]])
    own = np.repeat(np.arange(4), 16)
    assert np.all(gam - ref[own] <= 0) and np.all(gam - ref[own] >= -80)
    worst = -5.0 * 16
    assert np.exp(-worst) < 3.38e38


@pytest.mark.parametrize("decay_shift", [0.0, -6.0])
def test_bf16_operand_error_budget(decay_shift):
    a, s0, cu = _inputs([300, 211], 128, 128, seed=23, dtype="bf16", decay_shift=decay_shift)
    o_ref, f_ref = oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                                  initial_state=s0)
    o, f = cm.chunk_forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu, S0=s0, C=64, rnd=cm.bf16)
    assert _rel(o, o_ref) < 5e-3
    assert _rel(f, f_ref) < 3.5e-3


def test_stacked_output_form_equals_oracle_and_keeps_the_budget():
    """O = Q~ S + P U rewritten as P T' V + (Q~ - P T' K~) S (the operands [T'; P T'] and
    [-W; Q~ - P W] stacked over 128 rows): exact to rounding, and inside the same bf16 error
    budget as the form the kernel uses now."""
    a, s0, cu = _inputs([1, 15, 16, 17, 63, 64, 65, 150], 32, 24, seed=24)
    o_ref, f_ref = oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                                  initial_state=s0)
    o, f = cm.chunk_forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu, S0=s0, C=64, stacked=True)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f, f_ref, rtol=1e-10, atol=1e-12)
    for shift in (0.0, -6.0):
        a, s0, cu = _inputs([300, 211], 128, 128, seed=23, dtype="bf16", decay_shift=shift)
        o_ref, f_ref = oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                                      initial_state=s0)
        o, f = cm.chunk_forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu, S0=s0, C=64, rnd=cm.bf16,
                                stacked=True)
        assert _rel(o, o_ref) < 5e-3, shift
        assert _rel(f, f_ref) < 3.5e-3, shift
