"""GPU parity with the fp64 oracle of the unbounded-decay path (KDA_FLAG_UNBOUNDED_DECAY): any
g <= 0, as with the negative-softplus decay, including decays far beyond what a factor split
could represent; the oracle takes g as given."""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
import oracle
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import TOL_F32, TOL_OUT_BF16, TOL_STATE_BF16, host, oracle_full, rel_l2

pytestmark = pytest.mark.gpu
UNB = kda.KDA_FLAG_UNBOUNDED_DECAY


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _run(inp, flags, split=0):
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     flags=flags, split_segments=split)
    return out, fin, kda.kda_read_device_error(ws)


def _check(inp, flags=UNB, split=0):
    out, fin, st = _run(inp, flags, split)
    assert st == kda.KDA_OK, kda.kda_status_string(st)
    o_ref, f_ref = oracle_full(inp)
    f32 = inp.q.dtype == torch.float32
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()
    assert rel_l2(host(out), o_ref) <= (TOL_F32 if f32 else TOL_OUT_BF16)
    assert rel_l2(host(fin), f_ref) <= (TOL_F32 if f32 else TOL_STATE_BF16)


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("bf16", 64, 128)])
def test_softplus_decay(dtype, dk, dv):
    inp = synth.make_prefill(H=3, dk=dk, dv=dv, dtype=dtype, seed=81, device="cuda",
                             lengths=np.array([1, 15, 16, 17, 64, 200, 333]), gate=True,
                             init_state=True, decay="softplus")
    _check(inp)


def test_extreme_decays():
    """Channels that forget with g = -300 or -1e4 on some tokens, next to slow ones: a split
    factor e^{-gamma} would overflow fp32 within one token."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=82, device="cuda",
                             lengths=np.array([100, 250]), gate=True, init_state=True,
                             decay="softplus", decay_shift=-4.0)
    g = inp.g.clone()
    gen = torch.Generator(device="cuda").manual_seed(5)
    mask = torch.rand(g.shape, generator=gen, device="cuda") < 0.02
    g[mask] = -300.0
    g[:, :, 7] = -1.0e4  # one channel forgets everything at every token
    inp = synth.PrefillInputs(inp.q, inp.k, inp.v, g.contiguous(), inp.beta, inp.gate, inp.initial_state,
                              inp.cu_seqlens)
    _check(inp)


@pytest.mark.parametrize("split", [3])
def test_unbounded_split(split):
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=83, device="cuda",
                             lengths=np.array([900, 500]), gate=True, init_state=True, decay="softplus")
    _check(inp, split=split)


def test_checked_unbounded_reports_only_positive_decay():
    inp = synth.make_prefill(H=2, dk=64, dv=64, dtype="f32", seed=84, device="cuda",
                             lengths=np.array([40]), gate=False, decay="softplus")
    g = inp.g.clone()
    g[3, 1, 5] = -400.0
    ok = synth.PrefillInputs(inp.q, inp.k, inp.v, g, inp.beta, inp.gate, inp.initial_state, inp.cu_seqlens)
    assert _run(ok, UNB | kda.KDA_FLAG_CHECK_DECAY)[2] == kda.KDA_OK
    g2 = g.clone()
    g2[10, 0, 2] = 0.5
    bad = synth.PrefillInputs(inp.q, inp.k, inp.v, g2, inp.beta, inp.gate, inp.initial_state, inp.cu_seqlens)
    assert _run(bad, UNB | kda.KDA_FLAG_CHECK_DECAY)[2] == kda.binding.KDA_ERR_DECAY_OUT_OF_RANGE


def test_decode_unbounded():
    N, H = 5, 3
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=85, device="cuda")
    s64 = state.double().cpu().numpy()
    tok = synth.make_decode_token(N=N, H=H, dk=128, dv=128, dtype="bf16", seed=86, device="cuda")
    g = tok.g.clone()
    g[:, :, :4] = -300.0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kda.kda_decode_step(tok.q, tok.k, tok.v, g, tok.beta, state, gate=tok.gate, error_word=err,
                              flags=UNB | kda.KDA_FLAG_CHECK_DECAY)
    a = {n: host(getattr(tok, n)) for n in ("q", "k", "v", "beta", "gate")}
    o_ref = oracle.decode_step(a["q"], a["k"], a["v"], host(g), a["beta"], s64, gate=a["gate"])
    assert kda.kda_read_device_error(err) == kda.KDA_OK
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16
