"""The Python binding restates the C header's status codes, dtypes, flags and sizes; a drift
between the two would silently change what the product path asks the kernels to do.  This
parses include/kda.h and compares every such constant with the binding's."""
import os
import re

from linear_attention_serving_rule_b200 import binding as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "kda.h")


def _header_constants():
    text = open(HEADER).read()
    consts = {}
    for name, val in re.findall(r"#define\s+(KDA_FLAG_\w+)\s+(0x[0-9a-fA-F]+)u", text):
        consts[name] = int(val, 16)
    for name, val in re.findall(r"\b(KDA_(?:OK|ERR_\w+|BF16|F32))\s*=\s*(\d+)", text):
        consts[name] = int(val)
    m = re.search(r"#define\s+KDA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "KDA_NOALLOC_SCRATCH_BYTES not found"
    consts["KDA_NOALLOC_SCRATCH_BYTES"] = int(m.group(1)) << int(m.group(2))
    return consts


def test_every_header_constant_matches_the_binding():
    consts = _header_constants()
    assert len([n for n in consts if n.startswith("KDA_FLAG_")]) >= 8
    assert len([n for n in consts if n.startswith("KDA_ERR_")]) >= 7
    for name, val in consts.items():
        assert hasattr(B, name), f"binding lacks {name}"
        assert getattr(B, name) == val, (name, getattr(B, name), val)


def test_flags_are_distinct_single_bits():
    flags = {n: v for n, v in _header_constants().items() if n.startswith("KDA_FLAG_")}
    for n, v in flags.items():
        assert v and (v & (v - 1)) == 0, n
    assert len(set(flags.values())) == len(flags)
