"""GPU parity of the in-kernel pre-processing of the raw projections with the fp64 oracle.

With KDA_FLAG_G_LOGITS, KDA_FLAG_BETA_LOGITS and KDA_FLAG_QK_L2NORM the kernels take decay
logits, beta logits and unnormalised q, k; the oracle applies the same maps in fp64 (its
G_LOGITS, BETA_LOGITS and QK_L2NORM modes, pinned in test_oracle.py).  Inputs are the same seeded
draws as the standard workloads, taken before their last step (synth raw=True).
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
ALL_LIB = kda.KDA_FLAG_G_LOGITS | kda.KDA_FLAG_BETA_LOGITS | kda.KDA_FLAG_QK_L2NORM
ALL_REF = oracle.G_LOGITS | oracle.BETA_LOGITS | oracle.QK_L2NORM
# one flag at a time: (library flag, oracle mode, which inputs stay raw)
SINGLE = {"g_logits": (kda.KDA_FLAG_G_LOGITS, oracle.G_LOGITS),
          "beta_logits": (kda.KDA_FLAG_BETA_LOGITS, oracle.BETA_LOGITS),
          "qk_l2norm": (kda.KDA_FLAG_QK_L2NORM, oracle.QK_L2NORM)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _mixed(raw, done, which):
    """Inputs whose `which` tensors are raw and the rest processed (the same draws)."""
    pick = {"g_logits": ("g",), "beta_logits": ("beta",), "qk_l2norm": ("q", "k")}[which]
    fields = {n: getattr(raw if n in pick else done, n) for n in ("q", "k", "v", "g", "beta", "gate")}
    return synth.PrefillInputs(fields["q"], fields["k"], fields["v"], fields["g"], fields["beta"],
                               fields["gate"], done.initial_state, done.cu_seqlens)


def _run(inp, flags, split=0):
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     flags=flags, split_segments=split)
    st = kda.kda_read_device_error(ws)
    assert st == kda.KDA_OK, kda.kda_status_string(st)
    return out, fin


LENGTHS = np.array([1, 15, 0, 16, 17, 63, 64, 65, 127, 200, 333])


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("bf16", 64, 128)])
def test_all_flags_ragged(path, dtype, dk, dv):
    inp = synth.make_prefill(H=3, dk=dk, dv=dv, dtype=dtype, seed=51, device="cuda",
                             lengths=LENGTHS, gate=True, init_state=True, raw=True)
    out, fin = _run(inp, ALL_LIB | PATHS[path])
    o_ref, f_ref = oracle_full(inp, mode=ALL_REF)
    to, ts = (TOL_F32, TOL_F32) if dtype == "f32" else (TOL_OUT_BF16, TOL_STATE_BF16)
    assert rel_l2(host(out), o_ref) <= to
    assert rel_l2(host(fin), f_ref) <= ts
    cu = inp.cu_seqlens
    for n in range(len(LENGTHS)):
        if LENGTHS[n]:
            assert rel_l2(host(out[cu[n]:cu[n + 1]]), o_ref[cu[n]:cu[n + 1]]) <= to
            assert rel_l2(host(fin[n]), f_ref[n]) <= ts


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("which", list(SINGLE))
def test_each_flag_alone(path, which):
    raw = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=52, device="cuda",
                             lengths=np.array([300, 77]), gate=True, init_state=True, raw=True)
    done = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=52, device="cuda",
                              lengths=np.array([300, 77]), gate=True, init_state=True)
    inp = _mixed(raw, done, which)
    flag, mode = SINGLE[which]
    out, fin = _run(inp, flag | PATHS[path])
    o_ref, f_ref = oracle_full(inp, mode=mode)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


@pytest.mark.parametrize("split", [3])
def test_all_flags_split(split):
    """The split's pass 1 (local state and transition) sees the same pre-processing."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=53, device="cuda",
                             lengths=np.array([1000, 700]), gate=True, init_state=True, raw=True)
    out, fin = _run(inp, ALL_LIB, split=split)
    o_ref, f_ref = oracle_full(inp, mode=ALL_REF)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


def test_all_flags_slow_decay():
    """Decay logits shifted by -6 (g near 0): long carry through the fused pre-processing."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=54, device="cuda",
                             lengths=np.array([512]), gate=True, init_state=True, raw=True,
                             decay_shift=-6.0)
    out, fin = _run(inp, ALL_LIB)
    o_ref, f_ref = oracle_full(inp, mode=ALL_REF)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(fin), f_ref) <= TOL_STATE_BF16


def test_all_flags_full_size_sampled():
    """B4 H32 T4096 raw projections in the benchmark's launch configuration: sampled units."""
    inp = synth.make_workload("prefill_bf16", device="cuda", raw=True)
    out, fin = _run(inp, ALL_LIB)
    units = [(0, 0), (1, 9), (2, 22), (3, 31)]
    ref = oracle_units(inp, units, tok_limit=1024, mode=ALL_REF)
    for (n, h) in units:
        o_ref, _ = ref[(n, h)]
        t0 = int(inp.cu_seqlens[n])
        assert rel_l2(host(out[t0:t0 + 1024, h]), o_ref) <= TOL_OUT_BF16
    ref = oracle_units(inp, units[:2], mode=ALL_REF)
    for (n, h) in units[:2]:
        assert rel_l2(host(fin[n, h]), ref[(n, h)][1]) <= TOL_STATE_BF16


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_decode_all_flags(dtype, dk, dv):
    N, H, slots = 6, 3, 8
    state = synth.make_states(slots=slots, H=H, dk=dk, dv=dv, seed=55, device="cuda")
    idx = torch.tensor([7, 0, 3, 5, 4, 1], dtype=torch.int32, device="cuda")
    s64 = state.double().cpu().numpy()
    for step in range(3):
        tok = synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, dtype=dtype, seed=56 + step,
                                      device="cuda", raw=True)
        out = kda.kda_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, state, gate=tok.gate,
                                  state_indices=idx, flags=ALL_LIB)
        a = {n: host(getattr(tok, n)) for n in ("q", "k", "v", "g", "beta", "gate")}
        o_ref = oracle.decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], s64, gate=a["gate"],
                                   state_indices=host(idx).astype(np.int64), mode=ALL_REF)
        tol = TOL_F32 if dtype == "f32" else TOL_OUT_BF16
        assert rel_l2(host(out), o_ref) <= tol
        assert rel_l2(state.cpu().numpy(), s64) <= (1e-5 if dtype == "f32" else TOL_STATE_BF16)


def test_prefill_then_decode_with_flags():
    """Raw projections: prefill of T tokens then one decode step = prefill of T + 1 tokens."""
    inp = synth.make_prefill(H=2, dk=128, dv=128, dtype="bf16", seed=57, device="cuda",
                             lengths=np.array([129]), gate=True, init_state=True, raw=True)
    T = 128
    head = {n: getattr(inp, n)[:T].contiguous() for n in ("q", "k", "v", "g", "beta", "gate")}
    _, fin, ws = kda.kda_chunk_fwd(head["q"], head["k"], head["v"], head["g"], head["beta"],
                                   gate=head["gate"], cu_seqlens=[0, T], initial_state=inp.initial_state,
                                   flags=ALL_LIB)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    state = fin.clone()
    last = {n: getattr(inp, n)[T:T + 1].contiguous() for n in ("q", "k", "v", "g", "beta", "gate")}
    out = kda.kda_decode_step(last["q"], last["k"], last["v"], last["g"], last["beta"], state,
                              gate=last["gate"], flags=ALL_LIB)
    o_ref, f_ref = oracle_full(inp, mode=ALL_REF)
    assert rel_l2(host(out[0]), o_ref[T]) <= TOL_OUT_BF16
    assert rel_l2(host(state[0]), f_ref[0]) <= TOL_STATE_BF16
