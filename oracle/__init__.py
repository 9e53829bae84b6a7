"""The oracle for the Kimi Delta Attention (KDA) core -- TEST INFRASTRUCTURE ONLY.

`kda_ref.c` is a plain sequential fp64 C statement of the gated delta rule with
its channel-wise forget gate and the head-wise RMSNorm * sigmoid-gate epilogue
(see `kda_ref.h` for the equations and the pages each step follows).  This
module compiles it with gcc and exposes it through ctypes over numpy arrays.

Only the test suite, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The GPU library never imports it and
shares no code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_ref.c")
_HDR = os.path.join(_HERE, "kda_ref.h")
_LIB = os.path.join(_HERE, "libkda_ref.so")
_lock = threading.Lock()
_lib = None

ERASE_OFF = 1
G_LOGITS = 2       # g holds decay logits a: g = -5 sigmoid(a)
BETA_LOGITS = 4    # beta holds logits: beta = sigmoid(b)
QK_L2NORM = 8      # q, k L2-normalised per (token, head): x / sqrt(sum x^2 + 1e-6)


def build(force: bool = False) -> str:
    """Compile kda_ref.c into oracle/libkda_ref.so (gcc -O2, no fast-math, OpenMP)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp",
               "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True, cwd=_HERE)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.kda_ref_forward.argtypes = [
        ctypes.c_int64, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        P, P, P, P, P, P, P, P, ctypes.c_double, ctypes.c_double,
        ctypes.c_uint32, ctypes.c_int32, P, P]
    lib.kda_ref_forward.restype = ctypes.c_int
    lib.kda_ref_forward_snapshots.argtypes = lib.kda_ref_forward.argtypes + [ctypes.c_int64, P]
    lib.kda_ref_forward_snapshots.restype = ctypes.c_int
    lib.kda_ref_decode_step.argtypes = [
        ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        P, P, P, P, P, P, P, P, P, ctypes.c_double, ctypes.c_double,
        ctypes.c_uint32, ctypes.c_int32, P]
    lib.kda_ref_decode_step.restype = ctypes.c_int
    lib.kda_ref_max_threads.argtypes = []
    lib.kda_ref_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


class Oracle:
    """The oracle bound to one compiled library (the default one, or a test's variant)."""

    ERASE_OFF = ERASE_OFF
    G_LOGITS, BETA_LOGITS, QK_L2NORM = G_LOGITS, BETA_LOGITS, QK_L2NORM

    def __init__(self, lib_path=None):
        self._lib = _bind(lib_path) if lib_path else None

    def _l(self):
        return self._lib if self._lib is not None else _load()

    def forward(self, *a, **kw):
        return forward(*a, _lib=self._l(), **kw)

    def forward_snapshots(self, *a, **kw):
        return forward_snapshots(*a, _lib=self._l(), **kw)

    def decode_step(self, *a, **kw):
        return decode_step(*a, _lib=self._l(), **kw)


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of kda_ref.c (used by the tests that check that the pins
    reject planted mistakes) into out_path with the same flags as build()."""
    d = os.path.dirname(out_path)
    src = os.path.join(d, "kda_ref_variant.c")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                    "-I", _HERE, "-o", out_path, src, "-lm"], check=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f32(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().kda_ref_max_threads())


def forward(q, k, v, g, beta, *, cu_seqlens=None, gate=None, norm_weight=None,
            initial_state=None, scale=None, eps=1e-6, mode=0, num_threads=0,
            return_final_state=True, _lib=None, _snapshot_interval=None):
    """Run the oracle over a packed batch.

    q, k, g: [T_tot, H, dk]; v, gate: [T_tot, H, dv]; beta: [T_tot, H] (any
    float dtype; values are taken as float32, which is exact for bf16/fp32).
    A 4-D input [B, T, H, d] is accepted and treated as B equal-length sequences.
    initial_state: [N, H, dk, dv] (float64 kept as is) or None.
    Returns (out [T_tot, H, dv] float64, final_state [N, H, dk, dv] float64 or None).
    """
    q = np.asarray(q)
    dense = q.ndim == 4
    if dense:
        B, T = q.shape[0], q.shape[1]
        rs = lambda a: None if a is None else np.asarray(a).reshape((B * T,) + np.asarray(a).shape[2:])
        q, k, v, g, beta, gate = map(rs, (q, k, v, g, beta, gate))
        if cu_seqlens is None:
            cu_seqlens = np.arange(B + 1, dtype=np.int64) * T
    q, k, v, g, beta, gate, norm_weight = map(_f32, (q, k, v, g, beta, gate, norm_weight))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T_tot], dtype=np.int64)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[-1] != T_tot:
        raise ValueError("cu_seqlens[-1] must equal the number of packed tokens")
    S0 = None
    if initial_state is not None:
        S0 = np.ascontiguousarray(np.asarray(initial_state, dtype=np.float64)).reshape(N, H, dk, dv)
    out = np.zeros((T_tot, H, dv), dtype=np.float64)
    fin = np.zeros((N, H, dk, dv), dtype=np.float64) if return_final_state else None
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    args = (N, _ptr(cu), H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
            _ptr(norm_weight), _ptr(S0), float(scale), float(eps), int(mode), int(num_threads),
            _ptr(out), _ptr(fin))
    snaps = None
    if _snapshot_interval is None:
        rc = (_lib or _load()).kda_ref_forward(*args)
    else:
        I = int(_snapshot_interval)
        if I <= 0:
            raise ValueError("snapshot_interval must be positive")
        rows = int(sum((int(cu[n + 1]) - int(cu[n])) // I for n in range(N)))
        snaps = np.zeros((max(rows, 1), H, dk, dv), dtype=np.float64)
        rc = (_lib or _load()).kda_ref_forward_snapshots(*args, I, _ptr(snaps))
        snaps = snaps[:rows]
    if rc != 0:
        raise ValueError(f"kda_ref_forward rejected its arguments (rc={rc})")
    if dense:
        out = out.reshape(B, T, H, dv)
    return (out, fin) if snaps is None else (out, fin, snaps)


def forward_snapshots(q, k, v, g, beta, snapshot_interval, **kw):
    """forward() that also returns the state after every multiple of snapshot_interval tokens of
    each sequence: (out, final_state, snapshots [rows, H, dk, dv] float64), rows ordered by
    sequence, then by position (the layout kda_ref.h gives)."""
    return forward(q, k, v, g, beta, _snapshot_interval=snapshot_interval, **kw)


def decode_step(q, k, v, g, beta, state, *, gate=None, norm_weight=None,
                state_indices=None, scale=None, eps=1e-6, mode=0, num_threads=0, _lib=None):
    """One decode token per sequence.  Inputs [N, H, d]; state [slots, H, dk, dv]
    float64, updated IN PLACE.  Returns out [N, H, dv] float64."""
    q, k, v, g, beta, gate, norm_weight = map(_f32, (q, k, v, g, beta, gate, norm_weight))
    N, H, dk = q.shape
    dv = v.shape[2]
    if state.dtype != np.float64 or not state.flags.c_contiguous:
        raise TypeError("state must be a C-contiguous float64 array (updated in place)")
    idx = None
    if state_indices is not None:
        idx = np.ascontiguousarray(np.asarray(state_indices, dtype=np.int64))
    out = np.zeros((N, H, dv), dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    rc = (_lib or _load()).kda_ref_decode_step(N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                     _ptr(gate), _ptr(norm_weight), _ptr(state), _ptr(idx),
                                     float(scale), float(eps), int(mode), int(num_threads),
                                     _ptr(out))
    if rc != 0:
        raise ValueError(f"kda_ref_decode_step rejected its arguments (rc={rc})")
    return out
