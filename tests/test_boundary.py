"""The C ABI boundary, without a GPU: libkda.so loads, exports every entry point that
include/*.h declares, and rejects bad arguments on the host before any CUDA call.

Pointers below are fake (never dereferenced): validation returns before the first
CUDA call, so these tests run on a machine without a GPU.  cu_seqlens is a real host
array because the host reads it.
"""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

import linear_attention_serving_rule_b200 as kda
from linear_attention_serving_rule_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def L():
    kda.build_library()
    return kda.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert {"kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
            "kda_read_device_error", "kda_status_string"} <= declared
    for name in declared:
        assert hasattr(L, name), f"libkda.so does not export {name}"
    assert set(B.EXPORTED) <= declared


def test_status_strings(L):
    for code, name in [(0, "KDA_OK"), (1, "KDA_ERR_INVALID_ARGUMENT"), (3, "KDA_ERR_WORKSPACE_TOO_SMALL"),
                       (5, "KDA_ERR_TIMEOUT"), (6, "KDA_ERR_DECAY_OUT_OF_RANGE"),
                       (7, "KDA_ERR_BAD_STATE_INDEX")]:
        assert kda.kda_status_string(code) == name
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"


def _args(**kw):
    a = B.KdaChunkArgs()
    a.num_seqs, a.total_tokens, a.cu_seqlens = 2, 256, None
    a.H, a.dk, a.dv, a.dtype = 4, 128, 128, B.KDA_BF16
    for f in ("q", "k", "v", "g", "beta", "gate", "out"):
        setattr(a, f, FAKE)
    a.norm_weight = a.initial_state = a.final_state = None
    a.scale, a.eps, a.flags, a.split_segments = 0.0, 1e-6, 0, 0
    a.workspace, a.workspace_bytes = FAKE, 1 << 30
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def _fwd(L, a):
    return L.kda_chunk_fwd(ctypes.byref(a), None)


def _ws(L, a):
    n = ctypes.c_size_t(0)
    rc = L.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n))
    return rc, n.value


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "beta", "out"])
def test_null_required_pointer(L, field):
    assert _fwd(L, _args(**{field: None})) == B.KDA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("field", ["q", "v", "gate", "out"])
def test_misaligned_pointer(L, field):
    assert _fwd(L, _args(**{field: FAKE + 2})) == B.KDA_ERR_INVALID_ARGUMENT


def test_beta_needs_element_alignment_only(L):
    assert _ws(L, _args(beta=FAKE + 2))[0] == B.KDA_OK
    assert _fwd(L, _args(beta=FAKE + 1)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(beta=FAKE + 2, dtype=B.KDA_F32)) == B.KDA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("dk,dv,code", [(96, 128, B.KDA_ERR_UNSUPPORTED), (128, 32, B.KDA_ERR_UNSUPPORTED),
                                        (0, 128, B.KDA_ERR_INVALID_ARGUMENT)])
def test_head_dims(L, dk, dv, code):
    assert _fwd(L, _args(dk=dk, dv=dv)) == code


def test_bad_scalars(L):
    assert _fwd(L, _args(H=0)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(dtype=7)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(eps=-1.0)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(eps=float("nan"))) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(scale=-0.5)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(split_segments=-1)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(total_tokens=255)) == B.KDA_ERR_INVALID_ARGUMENT  # not divisible by num_seqs
    assert _fwd(L, _args(num_seqs=0, total_tokens=5)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(total_tokens=1 << 31)) == B.KDA_ERR_UNSUPPORTED


def test_cu_seqlens_validation(L):
    good = np.array([0, 100, 100, 256], dtype=np.int32)
    bad_start = np.array([1, 100, 100, 256], dtype=np.int32)
    decreasing = np.array([0, 100, 90, 256], dtype=np.int32)
    wrong_total = np.array([0, 100, 100, 255], dtype=np.int32)
    for arr, code in [(bad_start, B.KDA_ERR_INVALID_ARGUMENT), (decreasing, B.KDA_ERR_INVALID_ARGUMENT),
                      (wrong_total, B.KDA_ERR_INVALID_ARGUMENT)]:
        assert _fwd(L, _args(num_seqs=3, cu_seqlens=arr.ctypes.data)) == code
    rc, n = _ws(L, _args(num_seqs=3, cu_seqlens=good.ctypes.data))
    assert rc == B.KDA_OK and n >= 4


def test_workspace_size_and_check(L):
    rc, n = _ws(L, _args())
    assert rc == B.KDA_OK and n == 256  # error word only: 8 units fill too little GPU to split 128-token sequences
    assert _fwd(L, _args(workspace=None)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(workspace=FAKE + 16)) == B.KDA_ERR_INVALID_ARGUMENT
    assert _fwd(L, _args(workspace_bytes=n - 1)) == B.KDA_ERR_WORKSPACE_TOO_SMALL
    # a forced split needs per-segment state buffers
    rc, n3 = _ws(L, _args(split_segments=3, total_tokens=2 * 1024))
    assert rc == B.KDA_OK
    segs = 3 * 2  # 1024 tokens -> 3 segments of 384 (multiple of 64) per sequence
    assert n3 == 256 + segs * 4 * (128 * 128 + 128 * 256) * 4


def test_automatic_split_for_long_context(L):
    # 1 sequence x 16 heads of 1M tokens: 16 units < half of 148 SMs -> split.  With P segments
    # the first launch holds 16 x (P - 1) units (pass 1 of every segment but the last) and the
    # second 16 x P (every segment with its outputs); P = 9 gives 128 and 144 units, one wave of
    # 148 each: 2/9 of the unsplit time, the least for P <= 64 (P = 18 ties at 4 waves / 18).
    rc, n = _ws(L, _args(num_seqs=1, total_tokens=1 << 20, H=16))
    assert rc == B.KDA_OK
    per_slot = 16 * (128 * 128 + 128 * 256) * 4
    assert (n - 256) % per_slot == 0 and (n - 256) // per_slot == 9


@pytest.mark.parametrize("H,T,P", [(8, 1 << 20, 18), (4, 1 << 20, 37), (32, 1 << 16, 9), (64, 1 << 20, 1)])
def test_automatic_split_segment_count(L, H, T, P):
    """The planner's model, in chunk times of one unit: waves(H (P - 1)) + waves(H P) launches of a
    segment's chunks plus 4 per combine step, against the unsplit T / 64.
    - H = 8, 2^20 tokens: P = 18 gives 136 and 144 units (one wave each): 2 x 911 + 68 = 1,890.
      P = 37 gives 288 and 296 units (two waves each): 4 x 443 + 144 = 1,916.
    - H = 4: P = 37 gives 144 and 148 units, 2 x 443 + 144 = 1,030.
    - H = 32, 2^16 tokens: P = 9 gives 256 and 288 units (two waves each): 4 x 114 + 32 = 488.
      P = 4 gives 96 and 128 units: 2 x 256 + 12 = 524.
    - H = 64: no count saves a fifth of 16,384 (P = 2 already takes 2 x 8,192 + 4), so there is no
      split."""
    rc, n = _ws(L, _args(num_seqs=1, total_tokens=T, H=H))
    assert rc == B.KDA_OK
    per_slot = H * (128 * 128 + 128 * 256) * 4
    if P == 1:
        assert n == 256
    else:
        assert (n - 256) % per_slot == 0 and (n - 256) // per_slot == P


def _dargs(**kw):
    a = B.KdaDecodeArgs()
    a.N, a.H, a.dk, a.dv, a.dtype = 8, 4, 128, 128, B.KDA_BF16
    for f in ("q", "k", "v", "g", "beta", "gate", "state", "out"):
        setattr(a, f, FAKE)
    a.norm_weight = a.state_indices = a.error_word = None
    a.num_slots = 8
    a.scale, a.eps, a.flags = 0.0, 1e-6, 0
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def test_decode_validation(L):
    f = lambda **kw: L.kda_decode_step(ctypes.byref(_dargs(**kw)), None)
    for field in ("q", "k", "v", "g", "beta", "state", "out"):
        assert f(**{field: None}) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(state=FAKE + 4) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(dk=96) == B.KDA_ERR_UNSUPPORTED
    assert f(num_slots=7) == B.KDA_ERR_INVALID_ARGUMENT       # identity slots need num_slots >= N
    assert f(num_slots=0, state_indices=FAKE) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(N=-1) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(N=0) == B.KDA_OK                                  # nothing to do, nothing launched
    assert L.kda_read_device_error(None, None) == B.KDA_ERR_INVALID_ARGUMENT
    # multi-token decode: K >= 0 (0 means 1), position states 16-byte aligned
    assert f(tokens=-1) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(tokens=4, position_states=FAKE + 8) == B.KDA_ERR_INVALID_ARGUMENT
    assert f(N=0, tokens=8) == B.KDA_OK
    assert f(N=1 << 20, H=64, tokens=64, num_slots=1 << 20) == B.KDA_ERR_UNSUPPORTED  # N K H > 2^31


def _count(L, a):
    n = ctypes.c_int64(-1)
    rc = L.kda_chunk_fwd_snapshot_count(ctypes.byref(a), ctypes.byref(n))
    return rc, n.value


def test_snapshot_arguments(L):
    # a snapshot buffer needs 16-byte alignment and an interval that is a positive multiple of 64
    assert _fwd(L, _args(snapshots=FAKE + 8, snapshot_interval=64)) == B.KDA_ERR_INVALID_ARGUMENT
    for bad in (0, -64, 32, 96):
        assert _fwd(L, _args(snapshots=FAKE, snapshot_interval=bad)) == B.KDA_ERR_INVALID_ARGUMENT
        assert _count(L, _args(snapshot_interval=bad))[0] == B.KDA_ERR_INVALID_ARGUMENT
    # without a buffer the interval is ignored
    assert _ws(L, _args(snapshots=None, snapshot_interval=32))[0] == B.KDA_OK


def test_snapshot_count(L):
    # sum over sequences of floor(len / interval); zero-length and short sequences contribute 0
    cu = np.array([0, 100, 300, 300, 1000], dtype=np.int32)
    a = _args(num_seqs=4, total_tokens=1000, cu_seqlens=cu.ctypes.data)
    for I, want in ((64, 1 + 3 + 0 + 10), (128, 0 + 1 + 0 + 5), (1024, 0)):
        a.snapshot_interval = I
        assert _count(L, a) == (B.KDA_OK, want)
    # dense batch: 2 sequences of 128 tokens
    assert _count(L, _args(snapshot_interval=64)) == (B.KDA_OK, 4)
    assert _count(L, _args(snapshot_interval=128)) == (B.KDA_OK, 2)
    # only the layout and the interval are read: no tensor pointers needed
    bare = B.KdaChunkArgs()
    bare.num_seqs, bare.total_tokens, bare.cu_seqlens, bare.snapshot_interval = 4, 1000, cu.ctypes.data, 64
    assert _count(L, bare) == (B.KDA_OK, 14)
    bad = np.array([0, 100, 90, 1000], dtype=np.int32)
    assert _count(L, _args(num_seqs=3, total_tokens=1000, cu_seqlens=bad.ctypes.data,
                           snapshot_interval=64))[0] == B.KDA_ERR_INVALID_ARGUMENT
