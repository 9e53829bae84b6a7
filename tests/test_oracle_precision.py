"""Precision cross-check of the oracle: its fp64 arithmetic against the same C source compiled
with every double promoted to x87 extended precision (long double, 64-bit significand).

The recurrence is a product of contractions (decay <= 1, Householder-type erase) and the
read-out is a plain sum, so the fp64 oracle should agree with a higher-precision evaluation to a
few units in the last place.  A large disagreement would mean the oracle loses accuracy somewhere
(cancellation, an unstable ordering) and could not serve as the reference at 1e-4.  Run on the
tiny fp32 workload (B1 H2 T256 d64, no gate, zero initial state) and on a gated variant with
initial states, slow decay and varlen lengths.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
from linear_attention_serving_rule_b200 import synth

LD = np.longdouble

PREAMBLE = """#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#define double long double
#define exp expl
#define sqrt sqrtl
"""


@pytest.fixture(scope="module")
def ld_lib(tmp_path_factory):
    if np.finfo(LD).nmant < 63:
        pytest.skip("long double is not the x87 extended format on this host")
    d = tmp_path_factory.mktemp("oracle_ld")
    path = oracle.compile_variant(PREAMBLE + oracle.source_text(), str(d / "libkda_ref_ld.so"))
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.kda_ref_forward.argtypes = [
        ctypes.c_int64, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        P, P, P, P, P, P, P, P, ctypes.c_longdouble, ctypes.c_longdouble,
        ctypes.c_uint32, ctypes.c_int32, P, P]
    lib.kda_ref_forward.restype = ctypes.c_int
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ld_forward(lib, inp):
    f = lambda t: None if t is None else np.ascontiguousarray(t.float().numpy())
    q, k, v, g, beta, gate = (f(getattr(inp, n)) for n in ("q", "k", "v", "g", "beta", "gate"))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = np.ascontiguousarray(inp.cu_seqlens.astype(np.int64))
    N = len(cu) - 1
    s0 = None
    if inp.initial_state is not None:
        s0 = np.ascontiguousarray(inp.initial_state.double().numpy().astype(LD))
    out = np.zeros((T, H, dv), dtype=LD)
    fin = np.zeros((N, H, dk, dv), dtype=LD)
    scale = LD(1) / np.sqrt(LD(dk))
    rc = lib.kda_ref_forward(N, _p(cu), H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(beta), _p(gate),
                             None, _p(s0), scale, LD(1e-6), 0, 1, _p(out), _p(fin))
    assert rc == 0
    return out, fin


def _f64_forward(inp):
    f = lambda t: None if t is None else t.float().numpy()
    s0 = None if inp.initial_state is None else inp.initial_state.double().numpy()
    return oracle.forward(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta), cu_seqlens=inp.cu_seqlens,
                          gate=f(inp.gate), initial_state=s0, num_threads=1)


def _max_rel(x, ref):
    x = np.asarray(x, dtype=LD)
    return float(np.max(np.abs(x - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("name", ["tiny_fp32", "gated_varlen"])
def test_fp64_oracle_agrees_with_extended_precision(ld_lib, name):
    if name == "tiny_fp32":
        inp = synth.make_workload("tiny_fp32", device="cpu")
    else:
        inp = synth.make_prefill(H=3, dk=64, dv=32, dtype="f32", seed=70, device="cpu",
                                 lengths=np.array([1, 90, 300]), gate=True, init_state=True,
                                 decay_shift=-6.0)
    o64, f64 = _f64_forward(inp)
    old, fld = _ld_forward(ld_lib, inp)
    # the two builds must really differ in precision (the promotion took effect) ...
    assert np.any(np.asarray(o64, dtype=LD) != old)
    # ... and agree far below every tolerance the oracle is used at
    assert _max_rel(o64, old) < 1e-12
    assert _max_rel(f64, fld) < 1e-12
