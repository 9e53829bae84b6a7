"""Test-only numpy model of the chunkwise ("piecewise parallel") form of the KDA recurrence.

This is the algebra the GPU chunk kernels implement, written in plain numpy so
that it can be checked against the sequential oracle before (and independently
of) any CUDA.  It is not the oracle and is not used by the library.

Per (sequence, head) unit and chunk of C tokens with state S0 at the chunk start
(gamma_t = inclusive cumulative log-decay from the chunk start, per key channel):

  A_ts = sum_c k_t[c] k_s[c] e^{gamma_t[c]-gamma_s[c]}   (s < t)
  P_ts = sum_c q_t[c] k_s[c] e^{gamma_t[c]-gamma_s[c]}   (s <= t)
  T    = (I + Diag(beta) A)^-1,  T' = T Diag(beta)
  W    = T' (e^{gamma} * K),  U' = T' V,  U = U' - W S0
  O    = scale * ((e^{gamma} * Q) S0 + P U)
  S_C  = Diag(e^{gamma_C}) S0 + (e^{gamma_C - gamma} * K)^T U

The decayed Gram blocks A and P are formed as products of two bounded factors
with a reference point per 16-token sub-tile: for a row token t in sub-tile a
(reference r_a = cumulative decay before sub-tile a) the row factor is
e^{gamma_t - r_a} <= 1 and the column factor is e^{r_a - gamma_s}, which is
<= e^{80} inside sub-tile a and <= 1 before it.  This is the lower-bounded decay
of "Kimi K3: Engineering a 2.8 Trillion Parameter Frontier" (section Dimension 1:
g >= -5 keeps a 16-token tile's cumulative log-decay in (-80, 0) and the
reciprocal factors inside the BF16 range), which lets every causal tile be a
dense product.

`rnd` (optional) rounds the operands the tensor-core kernel stores in bf16, to
estimate the error of that design.
"""
import numpy as np
import torch


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def tf32(x):
    a = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).copy()
    # round to nearest even at 10 mantissa bits
    lsb = (a >> 13) & 1
    a = (a + 0xFFF + lsb) & np.uint32(0xFFFFE000)
    return a.view(np.float32).astype(np.float64)


def _ident(x):
    return x


def chunk_unit(q, k, v, g, beta, S0, *, C=64, sub=16, scale=None, rnd=None, state_rnd=None, stacked=False):
    """One unit: q, k, g [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv].  fp64 arithmetic.
    rnd: rounding applied to bf16 operands (None = exact); state_rnd: rounding of the
    state copy used as an MMA operand (defaults to rnd).
    stacked: the output through the stacked operands [T'; P T'] and [-W; Q~ - P W] (U and the
    whole O from one product with S, no separate P U term), with that form's own rounding
    points: P T' and Q~ - P W are rounded like the other bf16 operands, P U' stays fp32."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    T, dk = q.shape
    dv = v.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    R = rnd or _ident
    RS = state_rnd or R
    S = np.array(S0, dtype=np.float64, copy=True)
    out = np.zeros((T, dv))
    for c0 in range(0, T, C):
        L = min(C, T - c0)
        Q = np.zeros((C, dk)); K = np.zeros((C, dk)); V = np.zeros((C, dv))
        G = np.zeros((C, dk)); b = np.zeros(C)
        Q[:L], K[:L], V[:L], G[:L], b[:L] = q[c0:c0 + L], k[c0:c0 + L], v[c0:c0 + L], g[c0:c0 + L], beta[c0:c0 + L]
        gam = np.cumsum(G, axis=0)                       # inclusive, from the chunk start
        nsub = C // sub
        ref = np.zeros((nsub, dk))                        # r_a: cumulative decay before sub-tile a
        for a in range(1, nsub):
            ref[a] = gam[a * sub - 1]
        own = np.repeat(np.arange(nsub), sub)            # sub-tile of each row
        Kl = R(K * np.exp(gam - ref[own]))               # row factors <= 1
        Ql = R(Q * np.exp(gam - ref[own]))
        A = np.zeros((C, C)); P = np.zeros((C, C))
        for a in range(nsub):
            n = (a + 1) * sub
            Kc = R(K[:n] * np.exp(ref[a] - gam[:n]))     # column factors <= e^{80}
            rows = slice(a * sub, n)
            A[rows, :n] = Kl[rows] @ Kc.T
            P[rows, :n] = Ql[rows] @ Kc.T
        A = np.tril(A, -1)
        P = np.tril(P)
        Tm = np.linalg.inv(np.eye(C) + b[:, None] * A)   # (I + Diag(beta) A)^-1
        Tp = R(Tm * b[None, :])                          # T' = T Diag(beta)
        Kt = R(K * np.exp(gam))                          # e^{gamma} k
        Qt = R(Q * np.exp(gam))
        W = Tp @ Kt
        Up = Tp @ V
        Sb = RS(S)
        U = Up - R(W) @ Sb
        Ub = R(U)
        if stacked:
            PT = R(R(P) @ Tp)                            # second half of the stacked T' operand
            O = scale * (PT @ V + R(Qt - PT @ Kt) @ Sb)  # = scale (Q~ S + P U) in exact arithmetic
        else:
            O = scale * (Qt @ Sb + R(P) @ Ub)
        Kh = R(K * np.exp(gam[C - 1] - gam))             # e^{gamma_C - gamma} k
        S = np.exp(gam[C - 1])[:, None] * S + Kh.T @ Ub
        out[c0:c0 + L] = O[:L]
    return out, S


def chunk_forward(q, k, v, g, beta, cu_seqlens, S0=None, **kw):
    """Packed batch [T_tot, H, d] -> (out [T_tot, H, dv], final [N, H, dk, dv]); no epilogue."""
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu_seqlens) - 1
    out = np.zeros((T_tot, H, dv))
    fin = np.zeros((N, H, dk, dv))
    for n in range(N):
        sl = slice(cu_seqlens[n], cu_seqlens[n + 1])
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else S0[n, h]
            o, s = chunk_unit(q[sl, h], k[sl, h], v[sl, h], g[sl, h], beta[sl, h], s0, **kw)
            out[sl, h] = o
            fin[n, h] = s
    return out, fin
