"""GPU parity of kda_decode_step (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
import oracle
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import TOL_F32, TOL_OUT_BF16, TOL_STATE_BF16, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _oracle_step(tok, state64, idx=None, w=None):
    a = {n: host(getattr(tok, n)) for n in ("q", "k", "v", "g", "beta", "gate")}
    return oracle.decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], state64, gate=a["gate"],
                              state_indices=None if idx is None else host(idx).astype(np.int64),
                              norm_weight=host(w))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("gate", [True, False])
def test_decode_small(dtype, dk, dv, gate):
    N, H, slots = 6, 3, 10
    state = synth.make_states(slots=slots, H=H, dk=dk, dv=dv, seed=40, device="cuda")
    idx = torch.tensor([7, 0, 3, 9, 4, 1], dtype=torch.int32, device="cuda")
    w = torch.linspace(0.5, 1.5, dv, device="cuda")
    s64 = state.double().cpu().numpy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(3):
        tok = synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, dtype=dtype, seed=41 + step,
                                      device="cuda", gate=gate)
        out = kda.kda_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, state, gate=tok.gate,
                                  state_indices=idx, norm_weight=w, error_word=err)
        o_ref = _oracle_step(tok, s64, idx, w)
        tol = TOL_F32 if dtype == "f32" else TOL_OUT_BF16
        assert rel_l2(host(out), o_ref) <= tol
        assert rel_l2(state.cpu().numpy(), s64) <= (1e-5 if dtype == "f32" else TOL_STATE_BF16)
    assert kda.kda_read_device_error(err) == kda.KDA_OK


def test_decode_full_size_one_step():
    """N512 x H32 d128, fp32 states ~ N(0, 0.02) updated in place, all units compared."""
    cfg = synth.WORKLOADS["decode_bf16"]
    N, H, dk, dv = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"]
    state = synth.make_states(slots=N, H=H, dk=dk, dv=dv, seed=cfg["seed"], device="cuda")
    s64 = state.double().cpu().numpy()
    tok = synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, dtype="bf16", seed=cfg["seed"] + 1,
                                  device="cuda")
    out = kda.kda_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, state, gate=tok.gate)
    o_ref = _oracle_step(tok, s64)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16
    for n in (0, 255, 511):  # per-sequence check
        assert rel_l2(host(out[n]), o_ref[n]) <= TOL_OUT_BF16


def test_bad_state_index_reports_error():
    state = synth.make_states(slots=4, H=2, dk=128, dv=128, seed=42, device="cuda")
    before = state.clone()
    tok = synth.make_decode_token(N=2, H=2, dk=128, dv=128, seed=43, device="cuda")
    idx = torch.tensor([1, 4], dtype=torch.int32, device="cuda")  # 4 is out of range
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, state, gate=tok.gate,
                        state_indices=idx, error_word=err)
    assert kda.kda_read_device_error(err) == kda.binding.KDA_ERR_BAD_STATE_INDEX
    assert torch.equal(state[[0, 2, 3]], before[[0, 2, 3]])  # only slot 1 was touched
    assert not torch.equal(state[1], before[1])


def test_checked_decode_decay():
    state = synth.make_states(slots=2, H=1, dk=128, dv=128, seed=44, device="cuda")
    tok = synth.make_decode_token(N=2, H=1, dk=128, dv=128, seed=45, device="cuda")
    tok.g[1, 0, 3] = -7.0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, state, gate=tok.gate,
                        flags=kda.KDA_FLAG_CHECK_DECAY, error_word=err)
    assert kda.kda_read_device_error(err) == kda.binding.KDA_ERR_DECAY_OUT_OF_RANGE


@pytest.mark.parametrize("flags", [0, kda.KDA_FLAG_FORCE_SIMT])
def test_prefill_then_decode_equals_longer_prefill(flags):
    """prefill(T) then one decode step == prefill(T + 1) (outputs of the last token, states)."""
    T = 203
    full = synth.make_prefill(H=4, dk=128, dv=128, dtype="bf16", seed=46, device="cuda", B=1, T=T + 1,
                              gate=True, init_state=True)
    o_full, f_full, _ = kda.kda_chunk_fwd(full.q, full.k, full.v, full.g, full.beta, gate=full.gate,
                                          cu_seqlens=full.cu_seqlens, initial_state=full.initial_state,
                                          flags=flags)
    _, f_pre, _ = kda.kda_chunk_fwd(full.q[:T], full.k[:T], full.v[:T], full.g[:T], full.beta[:T],
                                    gate=full.gate[:T], cu_seqlens=np.array([0, T]),
                                    initial_state=full.initial_state, flags=flags)
    sl = slice(T, T + 1)
    o_dec = kda.kda_decode_step(full.q[sl], full.k[sl], full.v[sl], full.g[sl], full.beta[sl], f_pre,
                                gate=full.gate[sl])
    assert rel_l2(host(o_dec), host(o_full[sl])) <= TOL_OUT_BF16
    assert rel_l2(host(f_pre), host(f_full)) <= TOL_STATE_BF16


def test_decode_1000_steps_sampled_sequences():
    """The benchmark's decode loop: N512 x H32, 1,000 consecutive in-place steps over a ring of 16
    input sets, every step on the whole batch.  Four sampled sequences (all heads) are replayed
    by the oracle step by step; the outputs of the last step and the states after it must agree."""
    cfg = synth.WORKLOADS["decode_bf16"]
    N, H, dk, dv, ring = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"], cfg["ring"]
    steps = cfg["steps"]
    seed = cfg["seed"]
    state = synth.make_states(slots=N, H=H, dk=dk, dv=dv, seed=seed, device="cuda")
    picks = np.array([0, 137, 300, 511])
    s64 = state[picks].double().cpu().numpy()
    toks = [synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, seed=seed + 1 + i, device="cuda")
            for i in range(ring)]
    sub = [{n: host(getattr(t, n))[picks] for n in ("q", "k", "v", "g", "beta", "gate")} for t in toks]
    out = torch.empty((N, H, dv), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i in range(steps):
        t = toks[i % ring]
        kda.kda_decode_step(t.q, t.k, t.v, t.g, t.beta, state, gate=t.gate, out=out, error_word=err)
    torch.cuda.synchronize()
    assert kda.kda_read_device_error(err) == kda.KDA_OK
    for i in range(steps):
        a = sub[i % ring]
        o_ref = oracle.decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], s64, gate=a["gate"])
    assert rel_l2(host(out[picks]), o_ref) <= TOL_OUT_BF16
    got = state[picks].cpu().numpy()
    assert rel_l2(got, s64) <= TOL_STATE_BF16
    for j in range(len(picks)):  # per sequence
        assert rel_l2(got[j], s64[j]) <= TOL_STATE_BF16, picks[j]
