"""GPU parity of the multi-token decode (K tokens per sequence in one call, for verifying
speculative drafts) with the fp64 oracle: K consecutive oracle decode steps give the outputs of
every position, the state after each position and the final state."""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
import oracle
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import TOL_F32, TOL_OUT_BF16, TOL_STATE_BF16, host, oracle_full, rel_l2

pytestmark = pytest.mark.gpu

FIELDS = ("q", "k", "v", "g", "beta", "gate")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _tokens(N, K, H, dk, dv, dtype, seed, raw=False, gate=True):
    """[N, K, H, d] inputs: N sequences of K tokens (the prefill generator, reshaped)."""
    p = synth.make_prefill(H=H, dk=dk, dv=dv, dtype=dtype, seed=seed, device="cuda",
                           lengths=np.full(N, K, dtype=np.int64), gate=gate, raw=raw)
    t = {}
    for n in FIELDS:
        x = getattr(p, n)
        t[n] = None if x is None else x.reshape((N, K) + tuple(x.shape[1:])).contiguous()
    return t


def _oracle_steps(t, s64, idx, mode=0):
    """K oracle decode steps; returns outputs [N, K, H, dv] and states after each position
    [N, K, H, dk, dv] (s64 advanced in place)."""
    a = {n: host(x) for n, x in t.items()}
    N, K = a["q"].shape[:2]
    outs, states = [], []
    slots = host(idx).astype(np.int64) if idx is not None else np.arange(N)
    for tk in range(K):
        o = oracle.decode_step(a["q"][:, tk], a["k"][:, tk], a["v"][:, tk], a["g"][:, tk], a["beta"][:, tk],
                               s64, gate=None if a["gate"] is None else a["gate"][:, tk],
                               state_indices=None if idx is None else slots, mode=mode)
        outs.append(o)
        states.append(s64[slots].copy())
    return np.stack(outs, axis=1), np.stack(states, axis=1)


def _run(t, state, idx=None, flags=0, pos=None):
    g = t["gate"]
    return kda.kda_decode_step(t["q"], t["k"], t["v"], t["g"], t["beta"], state, gate=g,
                               state_indices=idx, flags=flags, position_states=pos)


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 7, 8])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 128), ("bf16", 128, 64), ("bf16", 64, 64)])
def test_multi_token_matches_sequential_steps(K, dtype, dk, dv):
    """K tokens in groups of up to four: K = 3 leaves a partial first group, K = 5 and 7 a partial
    second group (one and three tokens), so every split of a group's tokens over the threads of
    a channel is reached."""
    N, H, slots = 5, 3, 9
    state = synth.make_states(slots=slots, H=H, dk=dk, dv=dv, seed=60, device="cuda")
    idx = torch.tensor([8, 0, 3, 6, 1], dtype=torch.int32, device="cuda")
    s64 = state.double().cpu().numpy()
    t = _tokens(N, K, H, dk, dv, dtype, seed=61 + K)
    pos = torch.full((N, K, H, dk, dv), float("nan"), device="cuda")
    out = _run(t, state, idx, pos=pos)
    o_ref, p_ref = _oracle_steps(t, s64, idx)
    to = TOL_F32 if dtype == "f32" else TOL_OUT_BF16
    ts = 1e-5 if dtype == "f32" else TOL_STATE_BF16
    assert out.shape == (N, K, H, dv)
    for tk in range(K):
        assert rel_l2(host(out[:, tk]), o_ref[:, tk]) <= to, tk
        assert rel_l2(host(pos[:, tk]), p_ref[:, tk]) <= ts, tk
    assert rel_l2(state.cpu().numpy(), s64) <= ts
    # the committed state is the last position state, bit for bit
    torch.testing.assert_close(state[idx.long()], pos[:, K - 1], rtol=0, atol=0)


def test_no_commit_leaves_state_unchanged():
    N, H, K = 4, 2, 4
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=62, device="cuda")
    before = state.clone()
    t = _tokens(N, K, H, 128, 128, "bf16", seed=63)
    out_nc = _run(t, state, flags=kda.KDA_FLAG_DECODE_NO_COMMIT)
    torch.testing.assert_close(state, before, rtol=0, atol=0)
    out_c = _run(t, state)
    torch.testing.assert_close(out_nc, out_c, rtol=0, atol=0)


def test_verify_then_roll_back_or_commit_prefix():
    """Speculative decoding: verify K = 4 drafts without committing; accept m = 2.  Taking the
    position-1 state and re-running the 2 accepted tokens with commit give the same state, and
    both continue like the oracle that saw only the accepted tokens.  (The position states come
    from the token-by-token update, the committed state from the same recurrence unrolled over
    the group, so they agree to fp32 rounding rather than bit for bit.)"""
    N, H, K, m = 6, 2, 4, 2
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=64, device="cuda")
    s64 = state.double().cpu().numpy()
    t = _tokens(N, K, H, 128, 128, "bf16", seed=65)
    pos = torch.empty((N, K, H, 128, 128), device="cuda")
    _run(t, state, flags=kda.KDA_FLAG_DECODE_NO_COMMIT, pos=pos)
    rolled = pos[:, m - 1].contiguous()
    acc = {n: x[:, :m].contiguous() for n, x in t.items()}
    _run(acc, state)  # commit the accepted prefix
    torch.testing.assert_close(state, rolled, rtol=1e-5, atol=1e-6)
    _, _ = _oracle_steps(acc, s64, None)
    assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16
    nxt = _tokens(N, 1, H, 128, 128, "bf16", seed=66)
    out = _run(nxt, state)
    o_ref, _ = _oracle_steps(nxt, s64, None)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16


def test_multi_token_equals_prefill_of_the_tokens():
    """Decoding K tokens from S0 = the chunkwise prefill of the same K tokens from S0."""
    N, H, K = 3, 4, 8
    lengths = np.full(N, K, dtype=np.int64)
    p = synth.make_prefill(H=H, dk=128, dv=128, dtype="bf16", seed=67, device="cuda", lengths=lengths,
                           gate=True, init_state=True)
    out_p, fin_p, ws = kda.kda_chunk_fwd(p.q, p.k, p.v, p.g, p.beta, gate=p.gate, cu_seqlens=p.cu_seqlens,
                                         initial_state=p.initial_state)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    state = p.initial_state.clone()
    t = {n: getattr(p, n).reshape((N, K) + tuple(getattr(p, n).shape[1:])).contiguous() for n in FIELDS}
    out_d = _run(t, state)
    o_ref, f_ref = oracle_full(p)
    assert rel_l2(host(out_d).reshape(o_ref.shape), o_ref) <= TOL_OUT_BF16
    assert rel_l2(host(out_p), o_ref) <= TOL_OUT_BF16
    assert rel_l2(state.cpu().numpy(), f_ref) <= TOL_STATE_BF16


def test_multi_token_with_preprocessing_flags():
    N, H, K = 4, 2, 3
    flags = kda.KDA_FLAG_G_LOGITS | kda.KDA_FLAG_BETA_LOGITS | kda.KDA_FLAG_QK_L2NORM
    mode = oracle.G_LOGITS | oracle.BETA_LOGITS | oracle.QK_L2NORM
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=68, device="cuda")
    s64 = state.double().cpu().numpy()
    t = _tokens(N, K, H, 128, 128, "bf16", seed=69, raw=True)
    out = _run(t, state, flags=flags)
    o_ref, _ = _oracle_steps(t, s64, None, mode=mode)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16


def test_multi_token_full_size():
    """N512 x H32 d128 with K = 4 draft tokens per sequence (the decode benchmark's batch)."""
    cfg = synth.WORKLOADS["decode_bf16"]
    N, H, K = cfg["N"], cfg["H"], 4
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=cfg["seed"], device="cuda")
    s64 = state.double().cpu().numpy()
    t = _tokens(N, K, H, 128, 128, "bf16", seed=70)
    out = _run(t, state)
    o_ref, _ = _oracle_steps(t, s64, None)
    assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16
    assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16


def test_multi_token_bad_state_index_reports_error():
    """A slot outside the pool is reported on the error word and skipped: no other slot changes,
    and the valid sequence is still decoded."""
    N, H, K, slots = 2, 2, 3, 4
    state = synth.make_states(slots=slots, H=H, dk=128, dv=128, seed=71, device="cuda")
    before = state.clone()
    t = _tokens(N, K, H, 128, 128, "bf16", seed=72)
    idx = torch.tensor([1, 4], dtype=torch.int32, device="cuda")  # 4 is out of range
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_decode_step(t["q"], t["k"], t["v"], t["g"], t["beta"], state, gate=t["gate"],
                        state_indices=idx, error_word=err)
    assert kda.kda_read_device_error(err) == kda.binding.KDA_ERR_BAD_STATE_INDEX
    assert torch.equal(state[[0, 2, 3]], before[[0, 2, 3]])  # only slot 1 was touched
    s64 = before.double().cpu().numpy()
    one = {n: x[:1].contiguous() for n, x in t.items()}
    _oracle_steps(one, s64, torch.tensor([1], dtype=torch.int32))
    assert rel_l2(state[1].cpu().numpy(), s64[1]) <= TOL_STATE_BF16
