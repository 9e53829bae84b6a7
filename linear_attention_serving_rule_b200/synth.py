"""Seeded synthetic inputs for the KDA core (shared by tests, smoke check and bench).

This module only draws random tensors with the distributions of the five
workloads; it holds none of the recurrence's arithmetic.  The recipe
(per unit = (token, head)):

  q, k    ~ N(0, 1), then L2-normalised over the key channels in fp32
  v       ~ N(0, 1)
  beta    = sigmoid(N(0, 1))
  g       = g_min * sigmoid(N(0, 1) + decay_shift), g_min = -5 (decay_shift = 0
            for every workload; a negative shift gives the slow-decay test variant)
  gate    ~ N(0, 1) (gate logits of the output gate), or absent
  S0      ~ 0.02 * N(0, 1) fp32 when a workload has initial states
  lengths ~ uniform integers in [lo, hi] (numpy PCG64), for packed varlen batches

Draw order: q, k, v, beta logits, g logits, gate, initial state.  Tensors are
drawn with a torch.Generator seeded with `seed` on the target device, in fp32,
then cast to the workload dtype.  The same (seed, device) always gives the same
tensors.  The g_min = -5 floor is the lower-bounded decay of
"Kimi K3: Engineering a 2.8 Trillion Parameter Frontier", section
"Dimension 1: Sequence Length via Hybrid KDA-Gated MLA".
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

G_MIN = -5.0

# The five workloads (sizes and distributions of the KDA configurations).
WORKLOADS = {
    "tiny_fp32": dict(B=1, H=2, T=256, dk=64, dv=64, dtype="f32", gate=False,
                      init_state=False, seed=0),
    "prefill_bf16": dict(B=4, H=32, T=4096, dk=128, dv=128, dtype="bf16", gate=True,
                         init_state=False, seed=1),
    "varlen_bf16": dict(num_seqs=64, len_lo=128, len_hi=8192, H=32, dk=128, dv=128,
                        dtype="bf16", gate=True, init_state=True, seed=2),
    "long_bf16": dict(B=1, H=16, T=1 << 20, dk=128, dv=128, dtype="bf16", gate=True,
                      init_state=False, seed=3),
    "decode_bf16": dict(N=512, H=32, dk=128, dv=128, dtype="bf16", gate=True, steps=1000,
                        ring=16, seed=4),
}

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name):
    if isinstance(name, torch.dtype):
        return name
    return _DT[name]


def sample_lengths(num_seqs: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Integer sequence lengths uniform on [lo, hi] inclusive (numpy PCG64)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, size=num_seqs, dtype=np.int64)


def cu_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@dataclass
class PrefillInputs:
    q: torch.Tensor          # [T_tot, H, dk]
    k: torch.Tensor          # [T_tot, H, dk]
    v: torch.Tensor          # [T_tot, H, dv]
    g: torch.Tensor          # [T_tot, H, dk]
    beta: torch.Tensor       # [T_tot, H]
    gate: torch.Tensor | None  # [T_tot, H, dv]
    initial_state: torch.Tensor | None  # [N, H, dk, dv] fp32
    cu_seqlens: np.ndarray   # [N+1] int64 (host)
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self):
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def total_tokens(self):
        return int(self.cu_seqlens[-1])


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt((x * x).sum(-1, keepdim=True))


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def make_prefill(*, H: int, dk: int, dv: int, dtype="bf16", seed: int = 0,
                 device="cpu", lengths=None, B: int | None = None, T: int | None = None,
                 gate: bool = True, init_state: bool = False, decay_shift: float = 0.0,
                 state_std: float = 0.02, raw: bool = False, decay: str = "sigmoid") -> PrefillInputs:
    """Packed prefill inputs.  Give either `lengths` (varlen) or B and T (B equal
    sequences of T tokens, stored packed as [B*T, H, d]).

    raw=True returns the same draws before their last step: q and k not L2-normalised, beta
    and g as the logits b and a of beta = sigmoid(b), g = -5 sigmoid(a) (the inputs of the
    library's pre-processing flags).  decay="softplus" draws g = -softplus(a) instead of
    -5 sigmoid(a): the unbounded negative-softplus decay (no lower bound)."""
    if lengths is None:
        lengths = np.full(B, T, dtype=np.int64)
    cu = cu_from_lengths(lengths)
    T_tot = int(cu[-1])
    N = len(lengths)
    dt = torch_dtype(dtype)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    nrm = (lambda x: x) if raw else _l2norm
    q = nrm(_randn((T_tot, H, dk), gen, device)).to(dt)
    k = nrm(_randn((T_tot, H, dk), gen, device)).to(dt)
    v = _randn((T_tot, H, dv), gen, device).to(dt)
    b_logit = _randn((T_tot, H), gen, device)
    beta = (b_logit if raw else torch.sigmoid(b_logit)).to(dt)
    a_logit = _randn((T_tot, H, dk), gen, device) + decay_shift
    if raw:
        g = a_logit.to(dt)
    elif decay == "softplus":
        g = (-torch.nn.functional.softplus(a_logit)).to(dt)
    else:
        g = (G_MIN * torch.sigmoid(a_logit)).to(dt)
    gt = _randn((T_tot, H, dv), gen, device).to(dt) if gate else None
    s0 = (state_std * _randn((N, H, dk, dv), gen, device)) if init_state else None
    return PrefillInputs(q, k, v, g, beta, gt, s0, cu)


def make_workload(name: str, device="cpu", **overrides) -> PrefillInputs:
    """Prefill inputs of one named workload (overrides may shrink it for tests)."""
    w = dict(WORKLOADS[name])
    w.update(overrides)
    lengths = None
    if "num_seqs" in w:
        lengths = sample_lengths(w["num_seqs"], w["len_lo"], w["len_hi"], w["seed"])
    return make_prefill(H=w["H"], dk=w["dk"], dv=w["dv"], dtype=w["dtype"], seed=w["seed"],
                        device=device, lengths=lengths, B=w.get("B"), T=w.get("T"),
                        gate=w["gate"], init_state=w["init_state"],
                        decay_shift=w.get("decay_shift", 0.0), raw=w.get("raw", False),
                        decay=w.get("decay", "sigmoid"))


@dataclass
class DecodeInputs:
    q: torch.Tensor      # [N, H, dk]
    k: torch.Tensor
    v: torch.Tensor      # [N, H, dv]
    g: torch.Tensor      # [N, H, dk]
    beta: torch.Tensor   # [N, H]
    gate: torch.Tensor | None


def make_decode_token(*, N: int, H: int, dk: int, dv: int, dtype="bf16", seed: int = 0,
                      device="cpu", gate: bool = True, decay_shift: float = 0.0,
                      raw: bool = False) -> DecodeInputs:
    """Inputs of one decode step (one token per sequence)."""
    p = make_prefill(H=H, dk=dk, dv=dv, dtype=dtype, seed=seed, device=device,
                     lengths=np.ones(N, dtype=np.int64), gate=gate, decay_shift=decay_shift, raw=raw)
    return DecodeInputs(p.q, p.k, p.v, p.g, p.beta, p.gate)


def make_states(*, slots: int, H: int, dk: int, dv: int, seed: int, device="cpu",
                std: float = 0.02) -> torch.Tensor:
    """fp32 recurrent states ~ std * N(0, 1), [slots, H, dk, dv]."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return std * _randn((slots, H, dk, dv), gen, device)
