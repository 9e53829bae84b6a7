"""B200 (sm_100a) Kimi Delta Attention core: chunkwise prefill and decode step.

The compute lives in libkda.so (hand-written CUDA for sm_100a, C ABI declared in
include/kda.h).  This package holds its sources (csrc/), the in-tree build (build.py),
a thin ctypes binding with the C entry points' names (binding.py) and the seeded
synthetic-input generator (synth.py).
"""
from .binding import (  # noqa: F401
    KDA_BF16, KDA_F32, KDA_FLAG_CHECK_DECAY, KDA_FLAG_FORCE_SIMT, KDA_FLAG_TEST_FORCE_TIMEOUT,
    KDA_FLAG_G_LOGITS, KDA_FLAG_BETA_LOGITS, KDA_FLAG_QK_L2NORM, KDA_FLAG_DECODE_NO_COMMIT,
    KDA_FLAG_UNBOUNDED_DECAY,
    KDA_OK, KdaError, kda_chunk_fwd, kda_chunk_fwd_workspace_size, kda_decode_step,
    kda_read_device_error, kda_status_string, lib, lib_path, make_chunk_args, kda_chunk_fwd_noalloc,
    kda_chunk_fwd_snapshot_count, snapshot_count)
from .build import build as build_library  # noqa: F401
