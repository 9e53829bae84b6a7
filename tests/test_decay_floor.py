"""GPU parity at the edges of the decay range and of beta, through the C ABI.

The log-decay floor g >= -5 is what lets every causal tile be a dense tensor-core product: a
16-token sub-tile's cumulative log-decay stays in (-80, 0], so its reciprocal factors (at most
e^80) and direct factors (at least e^-80) fit bf16 ("Kimi K3: Engineering a 2.8 Trillion
Parameter Frontier", section "Dimension 1: Sequence Length via Hybrid KDA-Gated MLA").  These
tests sit exactly on that floor, where the tensor-core kernel's column factors reach e^80 and its
row factors e^-80, and on the other cases the recurrence fixes:

  g = -5 on every channel            (cumulative decay of a sub-tile exactly -80)
  g alternating -5 / 0 over channels (half the channels forget at the floor, half never)
  g = 0                              (no forgetting)
  beta = 1 with exactly unit keys    (the delta write is a Householder projection, so the
                                      state recalls the last value exactly: S^T k_t = v_t;
                                      "Kimi K3 from Moonshot AI", section "Kimi Delta Attention")
  beta = 0                           (no write at all: pure decay of the initial state)

Each case runs the tensor-core path, the fp32 CUDA-core path and the sequence split (3
segments), with lengths that cross sub-tile and chunk boundaries plus one full 4096-token unit,
and the decode step; every element is compared with the fp64 oracle at the usual tolerances.
"""
import math

import numpy as np
import pytest
import torch

import linear_attention_serving_rule_b200 as kda
import oracle
from linear_attention_serving_rule_b200 import synth
from tests.gpu_helpers import TOL_OUT_BF16, TOL_STATE_BF16, host, oracle_full, rel_l2

pytestmark = pytest.mark.gpu

LENGTHS = np.array([17, 64, 65, 200, 4096])
CASES = ["g_floor", "g_alternating", "g_zero", "beta_one_unit_keys", "beta_zero"]
PATHS = {"tc": (0, 0), "simt": (kda.KDA_FLAG_FORCE_SIMT, 0), "split3": (0, 3)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.build_library()
    kda.lib()


def _unit_keys(gen, n, d, nnz=16):
    """Rows with nnz entries of +-1/sqrt(nnz) on random channels: unit norm exactly in bf16."""
    x = torch.zeros((n, d), dtype=torch.float32)
    idx = torch.argsort(torch.rand((n, d), generator=gen), dim=1)[:, :nnz]
    sgn = torch.where(torch.rand((n, nnz), generator=gen) < 0.5, -1.0, 1.0)
    x.scatter_(1, idx, sgn / math.sqrt(nnz))
    return x


def _edit(inp, case, seed):
    """Overwrite g / beta / k of a bf16 PrefillInputs (tokens-first tensors) for one case."""
    T, H, dk = inp.k.shape
    gen = torch.Generator().manual_seed(seed)
    dev, dt = inp.k.device, inp.k.dtype
    if case == "g_floor":
        inp.g.fill_(-5.0)
    elif case == "g_alternating":
        pat = torch.tensor([-5.0, 0.0], device=dev).repeat(dk // 2)
        inp.g.copy_(pat.expand(T, H, dk).to(dt))
    elif case == "g_zero":
        inp.g.zero_()
    elif case == "beta_one_unit_keys":
        inp.beta.fill_(1.0)
        inp.k.copy_(_unit_keys(gen, T * H, dk).reshape(T, H, dk).to(device=dev, dtype=dt))
    elif case == "beta_zero":
        inp.beta.zero_()
    return inp


def _make(case, lengths=LENGTHS, H=2, seed=60):
    # beta = 0 keeps only the decayed initial state: use the slow-decay draw so that it stays far
    # from fp32 underflow over 4096 tokens
    shift = -6.0 if case == "beta_zero" else 0.0
    inp = synth.make_prefill(H=H, dk=128, dv=128, dtype="bf16", seed=seed, device="cuda",
                             lengths=lengths, gate=True, init_state=True, decay_shift=shift)
    return _edit(inp, case, seed)


_REF = {}


def _oracle(case, inp):
    if case not in _REF:  # the same inputs for every path
        _REF[case] = oracle_full(inp)
    return _REF[case]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("case", CASES)
def test_prefill_edge_cases(case, path):
    flags, split = PATHS[path]
    inp = _make(case)
    assert float(inp.g.float().min()) >= -5.0
    out, fin, ws = kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                     cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                     flags=flags | kda.KDA_FLAG_CHECK_DECAY, split_segments=split)
    assert kda.kda_read_device_error(ws) == kda.KDA_OK
    o_ref, f_ref = _oracle(case, inp)
    cu = inp.cu_seqlens
    for n in range(len(cu) - 1):
        sl = slice(cu[n], cu[n + 1])
        assert rel_l2(host(out[sl]), o_ref[sl]) <= TOL_OUT_BF16, (case, path, n)
        assert rel_l2(host(fin[n]), f_ref[n]) <= TOL_STATE_BF16, (case, path, n)
    if case == "beta_one_unit_keys":
        # the last write is recalled: S^T k_last = v_last (exact in the oracle; the GPU state
        # is within the state tolerance of it)
        for n in range(len(cu) - 1):
            t = cu[n + 1] - 1
            for h in range(inp.k.shape[1]):
                kl = inp.k[t, h].double().cpu().numpy()
                rec = host(fin[n, h]).astype(np.float64).T @ kl
                assert rel_l2(rec, host(inp.v[t, h])) <= TOL_OUT_BF16, (path, n, h)


@pytest.mark.parametrize("case", CASES)
def test_decode_edge_cases(case):
    N, H, steps = 8, 4, 4
    state = synth.make_states(slots=N, H=H, dk=128, dv=128, seed=61, device="cuda")
    s64 = state.double().cpu().numpy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i in range(steps):
        p = _make(case, lengths=np.ones(N, dtype=np.int64), H=H, seed=62 + i)
        out = kda.kda_decode_step(p.q, p.k, p.v, p.g, p.beta, state, gate=p.gate,
                                  flags=kda.KDA_FLAG_CHECK_DECAY, error_word=err)
        o_ref = oracle.decode_step(host(p.q), host(p.k), host(p.v), host(p.g), host(p.beta), s64,
                                   gate=host(p.gate))
        assert rel_l2(host(out), o_ref) <= TOL_OUT_BF16, (case, i)
        assert rel_l2(state.cpu().numpy(), s64) <= TOL_STATE_BF16, (case, i)
        if case == "beta_one_unit_keys":
            rec = np.einsum("nhij,nhi->nhj", state.double().cpu().numpy(), p.k.double().cpu().numpy())
            assert rel_l2(rec, host(p.v)) <= TOL_OUT_BF16
    assert kda.kda_read_device_error(err) == kda.KDA_OK
