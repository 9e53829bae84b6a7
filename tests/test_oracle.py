"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test targets a plausible mistake in the oracle: decay applied after the
write or on the value axis, a wrong sign in the prediction error, the read-out
taken before the write, a missing beta or scale, a wrong cumulative-decay
index, a broken epilogue.  None of these tests re-types the oracle's loop: they
use closed forms, dense transition-matrix products, exact algebraic identities
and a library RMSNorm.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_serving_rule_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _exact_unit_rows(rng, n, d, nnz=16):
    """Rows with nnz entries of +-1/sqrt(nnz) (nnz a power of 4): unit norm exactly in fp32."""
    x = np.zeros((n, d), dtype=np.float32)
    a = np.float32(1.0 / math.sqrt(nnz))
    for i in range(n):
        idx = rng.choice(d, size=nnz, replace=False)
        x[i, idx] = a * rng.choice([-1.0, 1.0], size=nnz)
    return x


def _hadamard(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


# --- I1: exact delta write (generalised Householder projection) --------------------------
def pin_delta_write_is_exact_for_unit_keys(ref, dk=16, dv=8):
    """With ||k||=1 and beta=1 the write makes S_t^T k_t = v_t whatever the decay and the
    previous state ("Kimi K3 from Moonshot AI", section KDA: delta rule on the generalised
    Householder transformation).  Read-out with q = k and scale 1 gives o_t = v_t."""
    rng = _rng(1)
    T, H = 40, 2
    k = _exact_unit_rows(rng, T * H, dk).reshape(T, H, dk)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    g = (-5.0 * rng.random((T, H, dk))).astype(np.float32)
    beta = np.ones((T, H), np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    out, fin = ref.forward(k, k, v, g, beta, initial_state=s0, scale=1.0)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)
    # the last write holds in the final state as well
    np.testing.assert_allclose(np.einsum("hij,hi->hj", fin[0], k[-1].astype(np.float64)), v[-1],
                               rtol=0, atol=1e-12)


# --- I2a: beta = 0 leaves pure decay --------------------------------------------------------
def pin_beta_zero_is_pure_decay(ref):
    """beta = 0 removes both erase and write: S_t = Diag(e^{gamma_t}) S0 with gamma_t the
    inclusive cumulative log-decay, o_t = scale * S0^T (e^{gamma_t} * q_t).  dk != dv so that a
    decay applied to the value axis fails."""
    rng = _rng(2)
    T, H, dk, dv = 33, 3, 12, 7
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    g = (-0.3 * rng.random((T, H, dk))).astype(np.float32)
    beta = np.zeros((T, H), np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    out, fin = ref.forward(q, k, v, g, beta, initial_state=s0)
    gam = np.cumsum(g.astype(np.float64), axis=0)  # [T, H, dk]
    scale = 1.0 / math.sqrt(dk)
    want = scale * np.einsum("hij,thi->thj", s0[0], np.exp(gam) * q)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fin[0], np.exp(gam[-1])[:, :, None] * s0[0], rtol=1e-12, atol=0)


# --- I2b: erase off = gated linear attention (quadratic form) ------------------------------
def pin_erase_off_equals_gated_linear_attention(ref):
    """Without the erase term the recurrence is gated linear attention:
    o_t = scale * [ S0^T(e^{gamma_t} q_t) + sum_{s<=t} beta_s ((q_t e^{gamma_t - gamma_s}) . k_s) v_s ]."""
    rng = _rng(3)
    T, H, dk, dv = 24, 2, 8, 5
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    g = (-0.5 * rng.random((T, H, dk))).astype(np.float32)
    beta = rng.random((T, H)).astype(np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    out, fin = ref.forward(q, k, v, g, beta, initial_state=s0, mode=ref.ERASE_OFF)
    q64, k64, v64, b64 = (a.astype(np.float64) for a in (q, k, v, beta))
    gam = np.cumsum(g.astype(np.float64), axis=0)
    scale = 1.0 / math.sqrt(dk)
    want = np.zeros((T, H, dv))
    for h in range(H):
        for t in range(T):
            acc = s0[0, h].T @ (np.exp(gam[t, h]) * q64[t, h])
            for s in range(t + 1):
                w = np.dot(q64[t, h] * np.exp(gam[t, h] - gam[s, h]), k64[s, h])
                acc = acc + b64[s, h] * w * v64[s, h]
            want[t, h] = scale * acc
    np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-12)
    fin_want = np.exp(gam[-1])[:, :, None] * s0[0] + np.einsum(
        "th,thi,thj->hij", b64, np.exp(gam[-1][None] - gam) * k64, v64)
    np.testing.assert_allclose(fin[0], fin_want, rtol=1e-11, atol=1e-12)


# --- I3: unrolled product of explicit transition matrices -----------------------------------
def pin_unrolled_transition_product(ref, seed=4):
    """S_T = (prod_r M_r) S0 + sum_t (prod_{r>t} M_r) beta_t k_t v_t^T with the dense
    M_r = (I - beta_r k_r k_r^T) Diag(e^{g_r}); outputs o_t = scale S_t^T q_t from the
    same unrolled products, on tiny shapes with dk != dv."""
    rng = _rng(seed)
    T, dk, dv = 7, 3, 4
    q = rng.standard_normal((T, 1, dk)).astype(np.float32)
    k = rng.standard_normal((T, 1, dk)).astype(np.float32)
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    g = (-rng.random((T, 1, dk))).astype(np.float32)
    beta = rng.random((T, 1)).astype(np.float32)
    s0 = rng.standard_normal((1, 1, dk, dv))
    scale = 0.37
    out, fin = ref.forward(q, k, v, g, beta, initial_state=s0, scale=scale)
    q64, k64, v64, g64, b64 = (a[:, 0].astype(np.float64) for a in (q, k, v, g, beta[:, :, None]))
    M = [(np.eye(dk) - b64[r, 0] * np.outer(k64[r], k64[r])) @ np.diag(np.exp(g64[r]))
         for r in range(T)]

    def prod(lo, hi):  # M_{hi-1} ... M_lo
        P = np.eye(dk)
        for r in range(lo, hi):
            P = M[r] @ P
        return P

    for t in range(T):
        St = prod(0, t + 1) @ s0[0, 0]
        for s in range(t + 1):
            St = St + prod(s + 1, t + 1) @ (b64[s, 0] * np.outer(k64[s], v64[s]))
        np.testing.assert_allclose(out[t, 0], scale * St.T @ q64[t], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fin[0, 0], St, rtol=1e-11, atol=1e-12)


# --- I3b: chunk-boundary snapshots are the unrolled prefix states -------------------------------
def pin_snapshots_are_unrolled_prefix_states(ref, seed=7):
    """Snapshot p of a sequence is S_p = (prod_{r<p} M_r) S0 + sum_{t<p} (prod_{t<r<p} M_r)
    beta_t k_t v_t^T, computed here from the dense transition matrices for every boundary of two
    ragged sequences (lengths 130 and 70, interval 64), each head with its own initial state."""
    rng = _rng(seed)
    lens, H, dk, dv, I = (130, 70), 2, 3, 2, 64
    Tt = sum(lens)
    cu = np.array([0, lens[0], Tt], dtype=np.int64)
    q = rng.standard_normal((Tt, H, dk)).astype(np.float32)
    k = rng.standard_normal((Tt, H, dk)).astype(np.float32)
    v = rng.standard_normal((Tt, H, dv)).astype(np.float32)
    g = (-0.05 * rng.random((Tt, H, dk))).astype(np.float32)  # slow decay: early tokens still count
    beta = rng.random((Tt, H)).astype(np.float32)
    s0 = rng.standard_normal((2, H, dk, dv))
    out, fin, snaps = ref.forward_snapshots(q, k, v, g, beta, I, cu_seqlens=cu, initial_state=s0)
    assert snaps.shape == (lens[0] // I + lens[1] // I, H, dk, dv)
    row = 0
    for n in range(2):
        for p_ in range(I, lens[n] + 1, I):
            for h in range(H):
                S = s0[n, h].copy()
                for t in range(cu[n], cu[n] + p_):
                    kk = k[t, h].astype(np.float64)
                    M = (np.eye(dk) - float(beta[t, h]) * np.outer(kk, kk)) @ np.diag(np.exp(g[t, h].astype(np.float64)))
                    S = M @ S + float(beta[t, h]) * np.outer(kk, v[t, h].astype(np.float64))
                np.testing.assert_allclose(snaps[row, h], S, rtol=1e-10, atol=1e-12)
            row += 1
    assert row == snaps.shape[0]


# --- pre-processing of the raw projections (decay logits, beta logits, q/k L2 norm) ----------
def _small(seed, T=40, H=2, dk=8, dv=5):
    rng = _rng(seed)
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    g = (-rng.random((T, H, dk))).astype(np.float32)
    beta = rng.random((T, H)).astype(np.float32)
    gate = rng.standard_normal((T, H, dv)).astype(np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    return q, k, v, g, beta, gate, s0


def pin_decay_logits_are_the_scaled_sigmoid(ref):
    """g = -5 sigmoid(a): a = 0 gives g = -2.5 exactly, a = +40 the floor -5, a = -40 no decay
    (sigmoid(-40) = 4e-18), each against a run given that g directly."""
    q, k, v, g, beta, gate, s0 = _small(11)
    for a_val, g_val, tol in ((0.0, -2.5, 1e-13), (40.0, -5.0, 1e-12), (-40.0, 0.0, 1e-12)):
        a = np.full_like(g, a_val)
        o1, f1 = ref.forward(q, k, v, a, beta, gate=gate, initial_state=s0, mode=ref.G_LOGITS)
        o2, f2 = ref.forward(q, k, v, np.full_like(g, g_val), beta, gate=gate, initial_state=s0)
        np.testing.assert_allclose(o1, o2, rtol=tol, atol=tol)
        np.testing.assert_allclose(f1, f2, rtol=tol, atol=tol)


def pin_beta_logits_are_the_sigmoid(ref):
    """beta = sigmoid(b): b = 0 gives beta = 1/2 exactly; b = -40 removes the write (the pure
    decay closed form of S0); b = +40 gives beta = 1."""
    q, k, v, g, beta, gate, s0 = _small(12)
    o1, f1 = ref.forward(q, k, v, g, np.zeros_like(beta), gate=gate, initial_state=s0, mode=ref.BETA_LOGITS)
    o2, f2 = ref.forward(q, k, v, g, np.full_like(beta, 0.5), gate=gate, initial_state=s0)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(f1, f2, rtol=1e-13, atol=1e-13)
    o1, f1 = ref.forward(q, k, v, g, np.full_like(beta, 40.0), initial_state=s0, mode=ref.BETA_LOGITS)
    o2, f2 = ref.forward(q, k, v, g, np.ones_like(beta), initial_state=s0)
    np.testing.assert_allclose(f1, f2, rtol=1e-12, atol=1e-12)
    _, f1 = ref.forward(q, k, v, g, np.full_like(beta, -40.0), initial_state=s0, mode=ref.BETA_LOGITS)
    decay = np.exp(g.astype(np.float64).sum(axis=0))  # [H, dk]
    np.testing.assert_allclose(f1[0], decay[:, :, None] * s0[0], rtol=1e-12, atol=1e-14)


def pin_qk_l2norm_gives_unit_keys(ref):
    """q, k <- x / sqrt(|x|^2 + 1e-6): (a) with beta = 1, g = 0 and keys of norm 3 the delta write
    is the exact Householder projection of the normalised key, S_t^T k_t/|k_t| = v_t (to the
    1e-7 the eps leaves); (b) scaling q by 4 and k by 1/4 changes nothing (to that eps)."""
    rng = _rng(13)
    T, dk, dv = 12, 16, 6
    k = _exact_unit_rows(rng, T, dk)[:, None, :] * 3.0
    q = rng.standard_normal((T, 1, dk)).astype(np.float32)
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    g = np.zeros((T, 1, dk), np.float32)
    s0 = rng.standard_normal((1, 1, dk, dv))
    S = s0[0, 0].copy()
    for t in range(T):
        _, fin = ref.forward(q[:t + 1], k[:t + 1], v[:t + 1], g[:t + 1], np.ones((t + 1, 1), np.float32),
                             initial_state=s0, mode=ref.QK_L2NORM)
        kt = k[t, 0].astype(np.float64) / 3.0
        np.testing.assert_allclose(fin[0, 0].T @ kt, v[t, 0], rtol=0, atol=2e-6)
    q, k2, v, g, beta, gate, s0 = _small(14)
    o1, f1 = ref.forward(q, k2, v, g, beta, gate=gate, initial_state=s0, mode=ref.QK_L2NORM)
    o2, f2 = ref.forward(q * 4, k2 * 0.25, v, g, beta, gate=gate, initial_state=s0, mode=ref.QK_L2NORM)
    # (the 1e-6 inside the root moves the scaled keys' norm by ~1e-6 relative; the RMSNorm
    # epilogue can amplify that on small outputs)
    np.testing.assert_allclose(o1, o2, rtol=2e-4, atol=2e-5)
    np.testing.assert_allclose(f1, f2, rtol=2e-4, atol=2e-5)
    # and the normalisation does act: the unnormalised run differs at order 1
    o3, _ = ref.forward(q * 4, k2 * 0.25, v, g, beta, gate=gate, initial_state=s0)
    assert np.abs(o3 - o1).max() > 1e-2


# --- I4: orthonormal keys form an exact associative memory ----------------------------------
def pin_orthonormal_keys_are_recalled_exactly(ref):
    """g = 0, beta = 1, keys = distinct rows of a normalised 16x16 Hadamard matrix (exactly
    orthonormal in fp32): after all writes S_T^T k_s = v_s for every written key s."""
    rng = _rng(7)
    dk, dv, T = 16, 6, 11
    Hd = (_hadamard(dk) / 4.0).astype(np.float32)
    rows = rng.permutation(dk)[:T]
    k = Hd[rows][:, None, :]
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    g = np.zeros((T, 1, dk), np.float32)
    beta = np.ones((T, 1), np.float32)
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, fin = ref.forward(k, k, v, g, beta, initial_state=s0)
    recalled = k[:, 0].astype(np.float64) @ fin[0, 0]
    np.testing.assert_allclose(recalled, v[:, 0], rtol=0, atol=1e-12)


# --- I5: joint linearity in (V, S0) --------------------------------------------------------
def pin_linear_in_values_and_initial_state(ref):
    rng = _rng(8)
    T, H, dk, dv = 20, 2, 8, 8
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32) * 0.5
    g = (-rng.random((T, H, dk))).astype(np.float32)
    beta = rng.random((T, H)).astype(np.float32)
    # values on a coarse grid so that v1 + v2 is exact in fp32
    v1 = (rng.integers(-512, 512, (T, H, dv)) / 64.0).astype(np.float32)
    v2 = (rng.integers(-512, 512, (T, H, dv)) / 64.0).astype(np.float32)
    s1 = rng.standard_normal((1, H, dk, dv))
    s2 = rng.standard_normal((1, H, dk, dv))
    o1, f1 = ref.forward(q, k, v1, g, beta, initial_state=s1)
    o2, f2 = ref.forward(q, k, v2, g, beta, initial_state=s2)
    o3, f3 = ref.forward(q, k, v1 + v2, g, beta, initial_state=s1 + s2)
    np.testing.assert_allclose(o3, o1 + o2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(f3, f1 + f2, rtol=1e-10, atol=1e-11)


# --- I6 / I7: split invariance and varlen = separate sequences ------------------------------
def pin_split_invariance_and_varlen_packing(ref):
    inp = synth.make_prefill(H=3, dk=16, dv=12, dtype="f32", seed=9,
                             lengths=np.array([37, 1, 64, 0, 19]), gate=True, init_state=True)
    a = {n: getattr(inp, n).numpy() for n in ("q", "k", "v", "g", "beta", "gate")}
    s0 = inp.initial_state.double().numpy()
    cu = inp.cu_seqlens
    out, fin = ref.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                              gate=a["gate"], initial_state=s0)
    for n in range(len(cu) - 1):
        sl = slice(cu[n], cu[n + 1])
        L = cu[n + 1] - cu[n]
        sub = {x: a[x][sl] for x in a}
        o_n, f_n = ref.forward(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"],
                                  gate=sub["gate"], initial_state=s0[n:n + 1])
        np.testing.assert_array_equal(o_n, out[sl])
        np.testing.assert_array_equal(f_n[0], fin[n])
        if L >= 2:
            c = L // 3 + 1
            first = {x: sub[x][:c] for x in sub}
            rest = {x: sub[x][c:] for x in sub}
            oa, fa = ref.forward(first["q"], first["k"], first["v"], first["g"], first["beta"],
                                    gate=first["gate"], initial_state=s0[n:n + 1])
            ob, fb = ref.forward(rest["q"], rest["k"], rest["v"], rest["g"], rest["beta"],
                                    gate=rest["gate"], initial_state=fa)
            np.testing.assert_array_equal(np.concatenate([oa, ob]), out[sl])
            np.testing.assert_array_equal(fb[0], fin[n])


# --- epilogue: head-wise RMSNorm then sigmoid gate (library RMSNorm) --------------------------
def pin_epilogue_matches_library_rmsnorm(ref):
    """out = rms_norm(o_raw, eps) * w * sigmoid(gate) per (token, head) over dv
    ("Kimi K3 Architecture Explained", section Token mixing: head-wise RMSNorm, then gate)."""
    inp = synth.make_prefill(H=2, dk=16, dv=24, dtype="f32", seed=10, B=1, T=30, gate=True)
    a = {n: getattr(inp, n).numpy() for n in ("q", "k", "v", "g", "beta", "gate")}
    w = np.random.default_rng(0).uniform(0.5, 1.5, 24).astype(np.float32)
    eps = 1e-6
    raw, _ = ref.forward(a["q"], a["k"], a["v"], a["g"], a["beta"])
    gated, _ = ref.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], gate=a["gate"],
                              norm_weight=w, eps=eps)
    t_raw = torch.from_numpy(raw)
    want = torch.nn.functional.rms_norm(t_raw, (24,), weight=torch.from_numpy(w).double(), eps=eps)
    want = want * torch.sigmoid(torch.from_numpy(a["gate"]).double())
    np.testing.assert_allclose(gated, want.numpy(), rtol=1e-12, atol=1e-14)
    # gate logit 0 gives exactly half of the normalised output
    half, _ = ref.forward(a["q"], a["k"], a["v"], a["g"], a["beta"],
                             gate=np.zeros_like(a["gate"]), eps=eps)
    rms = np.sqrt((raw ** 2).mean(-1, keepdims=True) + eps)
    np.testing.assert_allclose(half, 0.5 * raw / rms, rtol=1e-13, atol=1e-15)


# --- decode: one recurrent step equals one token of the packed form --------------------------
def pin_decode_step_matches_one_token_forward(ref):
    rng = _rng(11)
    N, H, dk, dv, slots = 5, 2, 16, 8, 9
    inp = synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, dtype="f32", seed=12)
    a = {n: getattr(inp, n).numpy() for n in ("q", "k", "v", "g", "beta", "gate")}
    idx = rng.permutation(slots)[:N].astype(np.int64)
    state = rng.standard_normal((slots, H, dk, dv))
    before = state.copy()
    out = ref.decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], state, gate=a["gate"],
                             state_indices=idx)
    cu = np.arange(N + 1)
    o_f, f_f = ref.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                              gate=a["gate"], initial_state=before[idx])
    np.testing.assert_array_equal(out, o_f)
    np.testing.assert_array_equal(state[idx], f_f)
    untouched = np.setdiff1d(np.arange(slots), idx)
    np.testing.assert_array_equal(state[untouched], before[untouched])


# --- worked scalar example (hand-derived, tests/golden) --------------------------------------
def pin_scalar_worked_example(ref):
    """dk = dv = 1 values derived by hand from S_t = (1 - b k^2) e^g S + b k v; o = scale S q."""
    with open(os.path.join(GOLDEN, "scalar_recurrence.json")) as f:
        gold = json.load(f)
    x = {n: np.array(gold[n], dtype=np.float32).reshape(-1, 1, 1) for n in ("q", "k", "v", "g")}
    beta = np.array(gold["beta"], dtype=np.float32).reshape(-1, 1)
    s0 = np.array(gold["s0"], dtype=np.float64).reshape(1, 1, 1, 1)
    out, fin = ref.forward(x["q"], x["k"], x["v"], x["g"], beta, initial_state=s0,
                              scale=gold["scale"])
    e = math.exp(-1.0)
    want = [a + b * e for a, b in gold["expected_out"]]
    a, b = gold["expected_final_state"]
    np.testing.assert_allclose(out.reshape(-1), want, rtol=1e-15, atol=1e-16)
    np.testing.assert_allclose(fin.reshape(-1), [a + b * e], rtol=1e-15)


def pin_default_scale_is_one_over_sqrt_dk(ref):
    """The read-out is o_t = S_t^T q_t / sqrt(dk) when no scale is passed.  Worked by hand: dk = 4,
    dv = 1, one token with k = q = (1/2, 1/2, 1/2, 1/2) (unit norm), v = 2, g = 0, beta = 1 from
    S0 = 0.  The write gives S_1 = k v = 2 k, so o = scale * 2 (k . q) = 2 scale = 2 / sqrt(4) = 1,
    and the decode step gives the same.  (A 1/dk default would give 0.5.)"""
    half = np.full((1, 1, 4), 0.5, dtype=np.float32)
    v = np.full((1, 1, 1), 2.0, dtype=np.float32)
    g = np.zeros((1, 1, 4), dtype=np.float32)
    beta = np.ones((1, 1), dtype=np.float32)
    out, fin = ref.forward(half, half, v, g, beta)
    assert out.reshape(-1).tolist() == [1.0]
    assert fin.reshape(-1).tolist() == [1.0, 1.0, 1.0, 1.0]
    state = np.zeros((1, 1, 4, 1))
    o = ref.decode_step(half, half, v, g, beta, state)
    assert np.asarray(o).reshape(-1).tolist() == [1.0]


# --- I9: the decay floor keeps 16-token factors inside the bf16 range ------------------------
def pin_decay_floor_bound_on_generated_inputs(ref):
    """g = -5 sigmoid(.) >= -5 after bf16 rounding, so any 16-token cumulative log-decay is
    >= -80 and e^80 < bf16 max ("Kimi K3: Engineering ...", section Dimension 1)."""
    inp = synth.make_prefill(H=4, dk=128, dv=128, dtype="bf16", seed=13, B=2, T=256)
    g = inp.g.float()
    assert float(g.min()) >= -5.0 and float(g.max()) <= 0.0
    cs = g.reshape(2, 16, 16, 4, 128).sum(2)
    assert float(cs.min()) >= -80.0
    assert math.exp(80.0) < float(torch.finfo(torch.bfloat16).max)


PINS = [pin_delta_write_is_exact_for_unit_keys, pin_beta_zero_is_pure_decay,
        pin_erase_off_equals_gated_linear_attention, pin_unrolled_transition_product,
        pin_orthonormal_keys_are_recalled_exactly, pin_linear_in_values_and_initial_state,
        pin_split_invariance_and_varlen_packing, pin_epilogue_matches_library_rmsnorm,
        pin_decode_step_matches_one_token_forward, pin_scalar_worked_example,
        pin_snapshots_are_unrolled_prefix_states, pin_decay_logits_are_the_scaled_sigmoid,
        pin_beta_logits_are_the_sigmoid, pin_qk_l2norm_gives_unit_keys,
        pin_default_scale_is_one_over_sqrt_dk]


@pytest.fixture(scope="module")
def ref():
    oracle.build()
    return oracle.Oracle()


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__[4:])
def test_pin(ref, pin):
    pin(ref)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (32, 8)])
def test_delta_write_other_shapes(ref, dk, dv):
    pin_delta_write_is_exact_for_unit_keys(ref, dk, dv)


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_unrolled_transition_product_more_seeds(ref, seed):
    pin_unrolled_transition_product(ref, seed)


def test_decay_floor_bound():
    pin_decay_floor_bound_on_generated_inputs(None)
