"""The oracle's pins reject planted mistakes.

Each case plants one plausible mistake in a copy of the oracle's C source (on the
CPU, in a temporary directory), compiles it and runs every pin of test_oracle.py
against it: at least one pin must fail.  This shows that the pins constrain each
step of the recurrence and of the epilogue, not only the code path they exercise.
"""
import pytest

import oracle
from tests import test_oracle as T

# (name, text in kda_ref.c, replacement)
MUTANTS = [
    ("decay_dropped", "row[j] *= a;", "row[j] *= 1.0 + 0.0 * a;"),
    ("decay_on_value_axis", "row[j] *= a;", "row[j] *= exp((double)g[j % dk]);"),
    ("error_sign_flipped", "u[j] = beta * ((double)v[j] - u[j]);",
     "u[j] = beta * ((double)v[j] + u[j]);"),
    ("beta_dropped", "u[j] = beta * ((double)v[j] - u[j]);", "u[j] = ((double)v[j] - u[j]);"),
    ("write_dropped", "row[j] += ki * u[j];", "row[j] += 0.0 * ki * u[j];"),
    ("erase_reads_q", "const double ki = (double)k[i];\n      const double* row = S + (size_t)i * dv;\n      for (int32_t j = 0; j < dv; ++j) u[j] += row[j] * ki;",
     "const double ki = (double)q[i];\n      const double* row = S + (size_t)i * dv;\n      for (int32_t j = 0; j < dv; ++j) u[j] += row[j] * ki;"),
    ("scale_dropped", "o[j] *= scale;", "o[j] *= 1.0;"),
    ("eps_outside_sqrt", "sqrt(ss / (double)dv + eps)", "(sqrt(ss / (double)dv) + eps)"),
    ("sum_instead_of_mean", "sqrt(ss / (double)dv + eps)", "sqrt(ss + eps)"),
    ("gate_sigmoid_sign", "1.0 / (1.0 + exp(-x))", "1.0 / (1.0 + exp(x))"),
    ("norm_weight_ignored", "const double wj = w ? (double)w[j] : 1.0;", "const double wj = 1.0;"),
    ("decay_after_write", None, None),      # built below: the forget step moved after the write
    ("readout_before_write", None, None),   # built below: the read-out moved before the write
    ("decode_ignores_slot_map", "const int64_t slot = state_indices ? state_indices[n] : n;",
     "const int64_t slot = n;"),
    ("snapshot_wrong_head", "memcpy(snapshots + ((size_t)srow * H + h) * state_elems, S,",
     "memcpy(snapshots + ((size_t)srow * H + 0) * state_elems, S,"),
    ("snapshot_one_token_early", None, None),  # built below: the copy moved before the token's update
    ("decay_logit_sign", "KDA_REF_G_MIN * sigmoid((double)g[i])", "KDA_REF_G_MIN * sigmoid(-(double)g[i])"),
    ("beta_logit_ignored", "sigmoid((double)beta) : (double)beta", "(double)beta : (double)beta"),
    ("l2norm_q_only", "kd[i] *= rk;", "kd[i] *= 1.0;"),
    ("l2norm_eps_outside", "1.0 / sqrt(sk + KDA_REF_L2NORM_EPS)", "1.0 / (sqrt(sk) + 0.3)"),
]


def _block(src, start_marker, end_marker):
    i = src.index(start_marker)
    j = src.index(end_marker, i) + len(end_marker)
    return i, j


def _mutant_source(name, old, new):
    src = oracle.source_text()
    if name == "decay_after_write":
        i, j = _block(src, "  for (int32_t i = 0; i < dk; ++i) {\n    const double a = exp",
                      "for (int32_t j = 0; j < dv; ++j) row[j] *= a;\n  }\n")
        decay = src[i:j]
        src = src[:i] + src[j:]
        k = src.index("  for (int32_t j = 0; j < dv; ++j) o[j] = 0.0;")
        return src[:k] + decay + src[k:]
    if name == "readout_before_write":
        i, j = _block(src, "  for (int32_t j = 0; j < dv; ++j) o[j] = 0.0;",
                      "for (int32_t j = 0; j < dv; ++j) o[j] *= scale;\n")
        readout = src[i:j]
        src = src[:i] + src[j:]
        k = src.index("  for (int32_t i = 0; i < dk; ++i) {\n    const double ki = (double)k[i];\n    double* row")
        return src[:k] + readout + src[k:]
    if name == "snapshot_one_token_early":
        i, j = _block(src, "        const int64_t done = t - cu_seqlens[n] + 1;",
                      "sizeof(double) * state_elems);\n        }\n")
        snap = src[i:j]
        src = src[:i] + src[j:]
        k = src.index("        const double b = prep_token(dk, q + row * dk, k + row * dk, g + row * dk, beta[row],")
        return src[:k] + snap + src[k:]
    assert old in src, f"mutation anchor for {name} not found"
    return src.replace(old, new, 1)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    lib = oracle.compile_variant(_mutant_source(name, old, new), str(tmp_path / f"lib_{name}.so"))
    ref = oracle.Oracle(lib)
    failed = []
    for pin in T.PINS:
        try:
            pin(ref)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin rejects the planted mistake '{name}'"
