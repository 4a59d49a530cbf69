"""Static checks on the CUDA sources (CPU only).

* No TMA or bulk copy carries cluster multicast.  Every CTA loads its own
  operand bytes; the only multicast in the library is the tcgen05.commit
  arrival on both CTAs of a pair.  A multicast load whose source can be
  another GPU's memory is never allowed, so the rule is kept for all loads.
* Every inline-PTX TMA instruction is a tiled load
  (`.global.tile` -> shared), never a store or reduce that could start at
  a negative coordinate.
"""
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "gram_newton_schulz_b200", "csrc")


def _sources():
    out = []
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(CSRC, name)) as fh:
                out.append((name, fh.read()))
    return out


def _template(body):
    """The instruction template of an asm body: its string literals up to
    the first ':' outside a literal (the operand lists follow it)."""
    parts, i = [], 0
    while i < len(body):
        ch = body[i]
        if ch == ":":
            break
        if ch == '"':
            j = i + 1
            while body[j] != '"':
                j += 2 if body[j] == "\\" else 1
            parts.append(body[i + 1:j])
            i = j
        i += 1
    return " ".join(parts)


def _ptx_strings(text):
    """Instruction template of every asm(...) statement."""
    for m in re.finditer(r"asm\s*(?:volatile\s*)?\((.*?)\);", text, re.S):
        yield _template(m.group(1))


def test_sources_found():
    names = [n for n, _ in _sources()]
    assert "ptx.cuh" in names and "gemm_tc.cu" in names


def test_no_multicast_bulk_copies():
    for name, text in _sources():
        for ptx in _ptx_strings(text):
            if "cp.async.bulk" in ptx:
                assert "multicast" not in ptx, (name, ptx)
            if "multicast" in ptx:
                assert ptx.lstrip().startswith("tcgen05.commit"), (name, ptx)


def test_tma_instructions_are_tiled_loads():
    seen = 0
    for name, text in _sources():
        for ptx in _ptx_strings(text):
            if "cp.async.bulk.tensor" in ptx:
                seen += 1
                assert ".global.tile" in ptx and "shared::cluster.global" in ptx, (name, ptx)
                assert "reduce" not in ptx, (name, ptx)
    assert seen >= 2


def test_scanner_joins_split_literals():
    # asm strings split over several literals and lines are joined before
    # the checks above look at them
    planted = 'asm volatile("mov.u32"\n    " %0, 1;" : "=r"(x));'
    assert list(_ptx_strings(planted)) == ["mov.u32  %0, 1;"]
    commits = [p for _, t in _sources() for p in _ptx_strings(t) if "multicast" in p]
    assert commits and all(p.startswith("tcgen05.commit") for p in commits)
