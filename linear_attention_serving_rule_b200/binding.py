"""ctypes binding of libkda.so -- argument marshalling only.

Every function here fills the C argument struct from torch tensors and calls the C
entry point of the same name; all computation runs in the library's CUDA kernels.
Tensors must already live on the GPU.  If libkda.so is missing the first call raises
(there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

from .build import LIB as _LIB_PATH

_lock = threading.Lock()
_lib = None

KDA_OK = 0
KDA_ERR_INVALID_ARGUMENT = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_WORKSPACE_TOO_SMALL = 3
KDA_ERR_CUDA = 4
KDA_ERR_TIMEOUT = 5
KDA_ERR_DECAY_OUT_OF_RANGE = 6
KDA_ERR_BAD_STATE_INDEX = 7

KDA_BF16 = 0
KDA_F32 = 1

KDA_FLAG_CHECK_DECAY = 0x1
KDA_FLAG_FORCE_SIMT = 0x2
KDA_FLAG_TEST_FORCE_TIMEOUT = 0x4
KDA_FLAG_G_LOGITS = 0x8       # g holds decay logits a: the kernels use g = -5 sigmoid(a)
KDA_FLAG_BETA_LOGITS = 0x10   # beta holds logits: the kernels use sigmoid(beta)
KDA_FLAG_QK_L2NORM = 0x20     # q, k L2-normalised per (token, head) in the kernels
KDA_FLAG_DECODE_NO_COMMIT = 0x40  # decode: leave the state unchanged (verify pass)
KDA_FLAG_UNBOUNDED_DECAY = 0x80   # any g <= 0 (negative-softplus decay): exact fp32 prefill path

EXPORTED = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_decode_step",
            "kda_read_device_error", "kda_status_string", "kda_chunk_fwd_noalloc",
            "kda_chunk_fwd_snapshot_count")
KDA_NOALLOC_SCRATCH_BYTES = 32 << 20

_P = ctypes.c_void_p


class KdaChunkArgs(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int64),
        ("cu_seqlens", _P),
        ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
        ("dtype", ctypes.c_int),
        ("q", _P), ("k", _P), ("v", _P), ("g", _P), ("beta", _P), ("gate", _P),
        ("norm_weight", _P), ("initial_state", _P), ("out", _P), ("final_state", _P),
        ("scale", ctypes.c_float), ("eps", ctypes.c_float), ("flags", ctypes.c_uint32),
        ("split_segments", ctypes.c_int32),
        ("workspace", _P), ("workspace_bytes", ctypes.c_size_t),
        ("snapshots", _P), ("snapshot_interval", ctypes.c_int32),
    ]


class KdaDecodeArgs(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
        ("dtype", ctypes.c_int),
        ("q", _P), ("k", _P), ("v", _P), ("g", _P), ("beta", _P), ("gate", _P),
        ("norm_weight", _P), ("state", _P), ("num_slots", ctypes.c_int32),
        ("state_indices", _P), ("out", _P),
        ("scale", ctypes.c_float), ("eps", ctypes.c_float), ("flags", ctypes.c_uint32),
        ("error_word", _P), ("tokens", ctypes.c_int32), ("position_states", _P),
    ]


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {kda_status_string(status)} ({status})")


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libkda.so (built in-tree by build.build())."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"libkda.so is not built ({_LIB_PATH}); run "
                                   "`python -m linear_attention_serving_rule_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            L.kda_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(KdaChunkArgs),
                                                       ctypes.POINTER(ctypes.c_size_t)]
            L.kda_chunk_fwd_workspace_size.restype = ctypes.c_int
            L.kda_chunk_fwd_snapshot_count.argtypes = [ctypes.POINTER(KdaChunkArgs),
                                                       ctypes.POINTER(ctypes.c_int64)]
            L.kda_chunk_fwd_snapshot_count.restype = ctypes.c_int
            L.kda_chunk_fwd.argtypes = [ctypes.POINTER(KdaChunkArgs), _P]
            L.kda_chunk_fwd.restype = ctypes.c_int
            L.kda_decode_step.argtypes = [ctypes.POINTER(KdaDecodeArgs), _P]
            L.kda_decode_step.restype = ctypes.c_int
            L.kda_read_device_error.argtypes = [_P, _P]
            L.kda_read_device_error.restype = ctypes.c_int
            L.kda_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(KdaChunkArgs), _P, ctypes.POINTER(ctypes.c_void_p)]
            L.kda_chunk_fwd_noalloc.restype = ctypes.c_int
            L.kda_status_string.argtypes = [ctypes.c_int]
            L.kda_status_string.restype = ctypes.c_char_p
            _lib = L
    return _lib


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors passed to libkda must be CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors passed to libkda must be contiguous")


def make_chunk_args(q, k, v, g, beta, *, gate=None, cu_seqlens=None, initial_state=None,
                    norm_weight=None, out=None, final_state=None, scale=0.0, eps=1e-6,
                    flags=0, split_segments=0, workspace=None, snapshots=None, snapshot_interval=0):
    """Fill a KdaChunkArgs.  Returns (args, keepalive) -- keep `keepalive` until the call."""
    keep = []
    if q.dim() == 4:
        B, T, H, dk = q.shape
        num_seqs, total = B, B * T
        cu_ptr = None
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens is for packed [T_tot, H, d] inputs")
    else:
        total, H, dk = q.shape
        if cu_seqlens is None:
            num_seqs, cu_ptr = 1, None
        else:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
            keep.append(cu)
            num_seqs = cu.shape[0] - 1
            cu_ptr = cu.ctypes.data
    dv = v.shape[-1]
    a = KdaChunkArgs()
    a.num_seqs, a.total_tokens, a.cu_seqlens = num_seqs, total, cu_ptr
    a.H, a.dk, a.dv = H, dk, dv
    a.dtype = _dtype_code(q)
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.gate, a.norm_weight, a.initial_state = map(_ptr, (gate, norm_weight, initial_state))
    a.out, a.final_state = _ptr(out), _ptr(final_state)
    a.scale, a.eps, a.flags, a.split_segments = float(scale), float(eps), int(flags), int(split_segments)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    a.snapshots, a.snapshot_interval = _ptr(snapshots), int(snapshot_interval)
    return a, keep


def kda_chunk_fwd_snapshot_count(args: KdaChunkArgs) -> int:
    n = ctypes.c_int64(0)
    rc = lib().kda_chunk_fwd_snapshot_count(ctypes.byref(args), ctypes.byref(n))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_snapshot_count")
    return int(n.value)


def snapshot_count(q, v, snapshot_interval, *, cu_seqlens=None) -> int:
    """Rows of the snapshot buffer for these inputs (sum over sequences of len // interval)."""
    if isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = cu_seqlens.cpu().numpy()
    a, keep = make_chunk_args(q, q, v, q, q, cu_seqlens=cu_seqlens, snapshot_interval=snapshot_interval)
    # (the count reads the sequence layout and the interval only)
    n = kda_chunk_fwd_snapshot_count(a)
    del keep
    return n


def kda_chunk_fwd_workspace_size(args: KdaChunkArgs) -> int:
    n = ctypes.c_size_t(0)
    rc = lib().kda_chunk_fwd_workspace_size(ctypes.byref(args), ctypes.byref(n))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_workspace_size")
    return int(n.value)


def kda_chunk_fwd(q, k, v, g, beta, *, gate=None, cu_seqlens=None, initial_state=None,
                  norm_weight=None, output_final_state=True, scale=0.0, eps=1e-6, flags=0,
                  split_segments=0, out=None, final_state=None, workspace=None, stream=None,
                  snapshots=None, snapshot_interval=0):
    """Chunkwise KDA prefill through the C ABI.

    q, k, g [T_tot, H, dk] (or [B, T, H, dk]); v, gate [.., H, dv]; beta [.., H];
    cu_seqlens: host sequence offsets (list / numpy / CPU tensor) for packed varlen input.
    snapshots: optional fp32 [snapshot_count(...), H, dk, dv] buffer that receives the state after
    every multiple of snapshot_interval tokens of every sequence (include/kda.h gives the rows).
    Returns (out, final_state, workspace).  Asynchronous on the current stream.
    """
    _check_cuda(q, k, v, g, beta, gate, initial_state, norm_weight)
    if isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = cu_seqlens.cpu().numpy()
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if final_state is None and output_final_state:
        num_seqs = q.shape[0] if q.dim() == 4 else (1 if cu_seqlens is None else len(cu_seqlens) - 1)
        final_state = torch.empty((num_seqs, q.shape[-2], q.shape[-1], v.shape[-1]),
                                  dtype=torch.float32, device=q.device)
    a, keep = make_chunk_args(q, k, v, g, beta, gate=gate, cu_seqlens=cu_seqlens,
                              initial_state=initial_state, norm_weight=norm_weight, out=out,
                              final_state=final_state, scale=scale, eps=eps, flags=flags,
                              split_segments=split_segments, workspace=workspace,
                              snapshots=snapshots, snapshot_interval=snapshot_interval)
    if snapshots is not None:
        _check_cuda(snapshots)
        need_rows = kda_chunk_fwd_snapshot_count(a)
        if (snapshots.dtype != torch.float32 or not snapshots.is_contiguous()
                or snapshots.numel() < need_rows * q.shape[-2] * q.shape[-1] * v.shape[-1]):
            raise ValueError(f"snapshots must be a contiguous fp32 tensor of at least {need_rows} "
                             f"x [H, dk, dv]")
    if workspace is None:
        need = kda_chunk_fwd_workspace_size(a)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), need
    rc = lib().kda_chunk_fwd(ctypes.byref(a), _stream(stream))
    del keep
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd")
    return out, final_state, workspace


def kda_chunk_fwd_noalloc(q, k, v, g, beta, *, gate=None, cu_seqlens=None, initial_state=None,
                          norm_weight=None, output_final_state=True, scale=0.0, eps=1e-6, flags=0,
                          split_segments=0, out=None, final_state=None, stream=None):
    """kda_chunk_fwd through the entry point that needs no workspace: for callers that cannot
    allocate device memory, the library's static scratch array is used (see include/kda.h).
    Returns (out, final_state, error_word_address)."""
    _check_cuda(q, k, v, g, beta, gate, initial_state, norm_weight)
    if isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = cu_seqlens.cpu().numpy()
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if final_state is None and output_final_state:
        num_seqs = q.shape[0] if q.dim() == 4 else (1 if cu_seqlens is None else len(cu_seqlens) - 1)
        final_state = torch.empty((num_seqs, q.shape[-2], q.shape[-1], v.shape[-1]),
                                  dtype=torch.float32, device=q.device)
    a, keep = make_chunk_args(q, k, v, g, beta, gate=gate, cu_seqlens=cu_seqlens,
                              initial_state=initial_state, norm_weight=norm_weight, out=out,
                              final_state=final_state, scale=scale, eps=eps, flags=flags,
                              split_segments=split_segments)
    err = ctypes.c_void_p(0)
    rc = lib().kda_chunk_fwd_noalloc(ctypes.byref(a), _stream(stream), ctypes.byref(err))
    del keep
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_noalloc")
    return out, final_state, int(err.value or 0)


def kda_decode_step(q, k, v, g, beta, state, *, gate=None, state_indices=None, norm_weight=None,
                    out=None, scale=0.0, eps=1e-6, flags=0, error_word=None, stream=None,
                    position_states=None):
    """Decode through the C ABI; `state` [slots, H, dk, dv] fp32 is updated in place (unless
    KDA_FLAG_DECODE_NO_COMMIT).  q [N, H, dk] is one token per sequence; q [N, K, H, dk] is the
    next K tokens of each sequence, with outputs for every position and, if position_states
    [N, K, H, dk, dv] fp32 is given, the state after each position.  Returns out."""
    _check_cuda(q, k, v, g, beta, state, gate, state_indices, norm_weight, position_states)
    if q.dim() == 4:
        N, K, H, dk = q.shape
    else:
        (N, H, dk), K = q.shape, 1
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(tuple(q.shape[:-1]) + (dv,), dtype=v.dtype, device=v.device)
    a = KdaDecodeArgs()
    a.N, a.H, a.dk, a.dv = N, H, dk, dv
    a.dtype = _dtype_code(q)
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.gate, a.norm_weight, a.state = _ptr(gate), _ptr(norm_weight), _ptr(state)
    a.num_slots = state.shape[0]
    a.state_indices = _ptr(state_indices)
    a.out = _ptr(out)
    a.scale, a.eps, a.flags = float(scale), float(eps), int(flags)
    a.error_word = _ptr(error_word)
    a.tokens, a.position_states = K, _ptr(position_states)
    rc = lib().kda_decode_step(ctypes.byref(a), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step")
    return out


def kda_read_device_error(error_word, stream=None) -> int:
    """Synchronise, read and clear a device error word (a workspace or decode error_word)."""
    return int(lib().kda_read_device_error(_ptr(error_word), _stream(stream)))
