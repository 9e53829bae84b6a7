"""Helpers shared by the GPU parity tests: relative L2 error and oracle runs on
selected (sequence, head) units of a packed batch."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Parity tolerances (relative L2 over the compared tensor, in fp64).
TOL_OUT_BF16 = 1e-2
TOL_STATE_BF16 = 5e-3
TOL_F32 = 1e-4


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def host(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_full(inp, norm_weight=None, eps=1e-6, num_threads=0, mode=0):
    """The oracle on every unit of a (small) packed PrefillInputs."""
    a = {n: host(getattr(inp, n)) for n in ("q", "k", "v", "g", "beta", "gate")}
    s0 = None if inp.initial_state is None else inp.initial_state.double().cpu().numpy()
    return oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=inp.cu_seqlens,
                          gate=a["gate"], initial_state=s0, norm_weight=host(norm_weight), eps=eps,
                          num_threads=num_threads, mode=mode)


def oracle_units(inp, units, *, tok_limit=None, norm_weight=None, eps=1e-6, num_threads=0, mode=0):
    """Oracle outputs and final states for the listed (n, h) units only.

    Returns {(n, h): (out [len, dv] float64, final [dk, dv] float64)}.  With tok_limit the
    unit is cut to its first tok_limit tokens.  All units run in one oracle call as a
    packed batch of single-head sequences.
    """
    cu = inp.cu_seqlens
    qs, ks, vs, gs, bs, gts, s0s, lens = [], [], [], [], [], [], [], []
    for n, h in units:
        t0, t1 = int(cu[n]), int(cu[n + 1])
        if tok_limit is not None:
            t1 = min(t1, t0 + tok_limit)
        sl = slice(t0, t1)
        qs.append(host(inp.q[sl, h:h + 1])); ks.append(host(inp.k[sl, h:h + 1]))
        vs.append(host(inp.v[sl, h:h + 1])); gs.append(host(inp.g[sl, h:h + 1]))
        bs.append(host(inp.beta[sl, h:h + 1]))
        if inp.gate is not None:
            gts.append(host(inp.gate[sl, h:h + 1]))
        if inp.initial_state is not None:
            s0s.append(inp.initial_state[n, h].double().cpu().numpy())
        lens.append(t1 - t0)
    cat = lambda xs: np.concatenate(xs, axis=0)
    cuu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s0 = np.stack(s0s)[:, None] if s0s else None
    out, fin = oracle.forward(cat(qs), cat(ks), cat(vs), cat(gs), cat(bs), cu_seqlens=cuu,
                              gate=cat(gts) if gts else None, initial_state=s0,
                              norm_weight=host(norm_weight), eps=eps, num_threads=num_threads,
                              mode=mode)
    res = {}
    for i, u in enumerate(units):
        res[u] = (out[cuu[i]:cuu[i + 1], 0], fin[i, 0])
    return res


def gpu_unit(out, final, cu, n, h, tok_limit=None):
    t0, t1 = int(cu[n]), int(cu[n + 1])
    if tok_limit is not None:
        t1 = min(t1, t0 + tok_limit)
    o = out[t0:t1, h].float().cpu().numpy()
    f = None if final is None else final[n, h].cpu().numpy()
    return o, f
