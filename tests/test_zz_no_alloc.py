"""The entry point that allocates nothing: kda_chunk_fwd_noalloc.

Some callers cannot allocate device memory when they run the layer (code being captured into a
CUDA graph, runtimes with a fixed memory pool).  kda_chunk_fwd_noalloc serves them with a static
scratch array inside the library instead of a caller-provided workspace.  This test runs it twice
in a row through the C ABI on a batch whose sequences are split across SMs (so the scratch holds
real per-segment state, not only the error word) and checks both results against kda_chunk_fwd
with an ordinary workspace.  The two entry points launch the same deterministic kernels on the
same inputs, so the results must be identical bit for bit.  The file name makes pytest collect it
last.
"""
import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
from linear_attention_serving_rule_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def test_noalloc_matches_workspace_entry_point():
    inp = synth.make_prefill(H=4, dk=128, dv=128, dtype="bf16", seed=51, device="cuda",
                             lengths=np.array([900, 130, 1500]), gate=True, init_state=True,
                             decay_shift=-6.0)
    args = dict(gate=inp.gate, cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                split_segments=4)
    o_ref, f_ref, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, **args)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    for _ in range(2):
        out, fin, err = kda.kda_chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.g, inp.beta, **args)
        assert err != 0
        assert kda.kda_read_device_error(err) == kda.KDA_OK
        assert torch.equal(out, o_ref)
        assert torch.equal(fin, f_ref)


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 2 sequences x 4 heads x 65,536 tokens split 64 ways need 128 segment slots of per-head state
    # (about 96 MB), more than the static scratch; the check runs on the host before any launch.
    T = 1 << 16
    e = torch.empty((2 * T, 4, 128), dtype=torch.bfloat16, device="cuda")
    b = torch.empty((2 * T, 4), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kda.KdaError) as ei:
        kda.kda_chunk_fwd_noalloc(e, e, e, e, b, cu_seqlens=np.array([0, T, 2 * T]), split_segments=64)
    assert ei.value.status == kda.binding.KDA_ERR_WORKSPACE_TOO_SMALL
