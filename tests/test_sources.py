"""Static checks of the CUDA sources.

The backward pass is deterministic because no kernel accumulates through an atomic
read-modify-write: every gradient partial has one writer and is merged by a
fixed-order reduction (the offset-based gradient sharding of "Fast and Exact
Relative-Position Attention via Structure-Aware Kernels", Abstract, technique (3)).
This test keeps it that way: no CUDA atomic intrinsic, no PTX `atom` / `red`
instruction and no bulk-copy reduction appears in the library's code (comments
are stripped first).
"""
import pathlib
import re

CSRC = pathlib.Path(__file__).resolve().parents[1] / "attention_fwd_bwd_flashattention_b200" / "csrc"

FORBIDDEN = {
    "CUDA atomic intrinsic": r"\batomic[A-Z]\w*\s*\(",
    "PTX atom": r"\batom\.",
    "PTX red": r"\bred\.(?:global|shared|gpu|cta|sys|relaxed|release|add|min|max|and|or|xor|inc|dec)",
    "bulk-copy reduction": r"\bcp\.reduce\.",
    "multimem reduction": r"\bmultimem\.red\.",
}


def strip_comments(src: str) -> str:
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    return re.sub(r"//[^\n]*", " ", src)


def library_sources():
    files = sorted(p for ext in ("*.cu", "*.cuh", "*.h") for p in CSRC.glob(ext))
    assert files, f"no sources under {CSRC}"
    return files


def test_no_atomics_in_the_library():
    hits = []
    for f in library_sources():
        code = strip_comments(f.read_text())
        for what, pat in FORBIDDEN.items():
            for m in re.finditer(pat, code):
                line = code.count("\n", 0, m.start()) + 1
                hits.append(f"{f.name}:{line}: {what}: {m.group(0)!r}")
    assert not hits, "\n".join(hits)


def test_the_checker_sees_atomics():
    """The patterns catch the forms they are meant to catch (and skip comments)."""
    samples = ["atomicAdd(&x[i], v);", 'asm volatile("atom.global.add.f32 %0, [%1], %2;")',
               'asm("red.global.add.f32 [%0], %1;")', 'asm("cp.reduce.async.bulk.tensor.2d ...")']
    for s in samples:
        assert any(re.search(p, strip_comments(s)) for p in FORBIDDEN.values()), s
    assert not any(re.search(p, strip_comments("// atomicAdd(&x, 1)\n/* red.global.add */")) for p in FORBIDDEN.values())
