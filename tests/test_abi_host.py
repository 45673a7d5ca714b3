"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/relpos_attn.h declares, the ctypes struct matches the C layout,
and argument validation returns the documented codes without touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200 import build as bld

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "relpos_attn.h")


@pytest.fixture(scope="module")
def lib():
    bld.build()
    return bd.load()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"RELPOS_API\s+[\w\s\*]*?\b(relpos_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(bd.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", bd.lib_path()], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for sym in declared_symbols():
        assert sym in exported, sym
        assert hasattr(lib, sym)
    # nothing else of ours leaks out of the library
    assert {s for s in exported if s.startswith("relpos")} == set(declared_symbols())


def test_struct_layout_matches_c(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "relpos_attn.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(relpos_params_t), offsetof(relpos_params_t,B),"
        " offsetof(relpos_params_t,scale), offsetof(relpos_params_t,t5_num_buckets), offsetof(relpos_params_t,deberta_span),"
        " offsetof(relpos_params_t,seqlens_k), offsetof(relpos_params_t,shaw_value), offsetof(relpos_params_t,mem_len));"
        "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(prog), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    S = bd.relpos_params_t
    assert got == [ctypes.sizeof(S), S.B.offset, S.scale.offset, S.t5_num_buckets.offset, S.deberta_span.offset,
                   S.seqlens_k.offset, S.shaw_value.offset, S.mem_len.offset]


def test_trace_struct_layout_matches_c(tmp_path):
    prog = tmp_path / "trace.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "relpos_attn.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %d\\n\", sizeof(relpos_trace_t), offsetof(relpos_trace_t,capacity),"
        " offsetof(relpos_trace_t,count), offsetof(relpos_trace_t,dropped), offsetof(relpos_trace_t,only),"
        " offsetof(relpos_trace_t,names), RELPOS_TRACE_MAX);"
        "return 0;}\n")
    exe = tmp_path / "trace"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(prog), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    T = bd.relpos_trace_t
    assert got == [ctypes.sizeof(T), T.capacity.offset, T.count.offset, T.dropped.offset, T.only.offset, T.names.offset,
                   bd.TRACE_MAX]


def test_trace_registration_is_validated(lib):
    t = bd.relpos_trace_t()
    assert lib.relpos_trace_begin(None) == -1
    assert lib.relpos_trace_begin(ctypes.byref(t)) == -1  # no events
    arr = (ctypes.c_void_p * 2)(None, None)
    t.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    t.capacity = 1
    assert lib.relpos_trace_begin(ctypes.byref(t)) == -1  # null event handles
    t.capacity = bd.TRACE_MAX + 1
    assert lib.relpos_trace_begin(ctypes.byref(t)) == -1
    assert lib.relpos_trace_end() == 0


def test_version_and_strerror(lib):
    assert lib.relpos_attn_version() == 10800
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert bd.strerror(code) and bd.strerror(code) != "unknown status"
    assert bd.strerror(-99) == "unknown status"


@pytest.mark.parametrize("bad", [dict(d=32), dict(mech=5), dict(L=0), dict(B=0), dict(dtype=5), dict(scale=float("nan")),
                                 dict(kernel_path=9), dict(mech=0, t5_num_buckets=1), dict(mech=0, t5_max_distance=4),
                                 dict(mech=3, deberta_span=0), dict(mech=1, shaw_clip=-1), dict(shaw_value=2),
                                 dict(mech=0, shaw_value=1), dict(mech=2, causal=True, mem_len=-1),
                                 dict(mech=2, causal=False, mem_len=64), dict(mech=1, causal=True, mem_len=64),
                                 dict(B=1 << 40, H=1 << 40), dict(B=65536, H=1), dict(B=256, H=257),
                                 dict(mech=2, causal=True, mem_len=(1 << 63) - 1), dict(mech=2, causal=True, mem_len=1 << 20),
                                 dict(L=(1 << 20) + 1), dict(causal=2)])
def test_invalid_params_rejected(lib, bad):
    kw = dict(mech=1, B=1, H=2, L=64)
    kw.update(bad)
    with pytest.raises(bd.RelposError) as e:
        bd.relpos_attn_workspace_size(bd.Params(**kw), 0)
    assert e.value.code == -1


def test_workspace_sizes(lib):
    for mech in range(5):
        for causal in (False, True):
            P = bd.Params(mech=mech, B=2, H=3, L=1000, causal=causal)
            f = bd.relpos_attn_workspace_size(P, 0)
            b = bd.relpos_attn_workspace_size(P, 1)
            assert b >= 2 * 3 * 1000 * 4  # at least D
            assert f % 256 == 0 and b % 256 == 0
            # forward scratch: T5's per-offset bias vector; on the bf16 tensor-core
            # path also Transformer-XL's u.k / v.r and DeBERTa's end-row products
            assert (f > 0) == (mech in (0, 2, 3, 4))
            f32 = bd.relpos_attn_workspace_size(bd.Params(mech=mech, B=2, H=3, L=1000, causal=causal, dtype=bd.F32), 0)
            assert (f32 > 0) == (mech in (0, 4))
    with pytest.raises(bd.RelposError):
        bd.relpos_attn_workspace_size(bd.Params(mech=1, B=1, H=1, L=8), 3)


def test_memory_adds_padded_query_buffers(lib):
    """Transformer-XL memory: the workspace grows by the query-side tensors at M + L rows."""
    for pass_ in (0, 1):
        base = bd.relpos_attn_workspace_size(bd.Params(mech=bd.TXL, B=2, H=2, L=300, causal=True), pass_)
        mem = bd.relpos_attn_workspace_size(bd.Params(mech=bd.TXL, B=2, H=2, L=300, causal=True, mem_len=100), pass_)
        assert mem >= base + 2 * 2 * 400 * (64 * 2 * (2 if pass_ == 0 else 4) + 4)


def test_smallest_backward_workspace(lib):
    """pass 2: the smallest backward workspace; it leaves out only the Transformer-XL
    tensor-core backward's stored P / dS tiles (64 KB per 128 x 128 tile)."""
    ws = bd.relpos_attn_workspace_size
    txl = bd.Params(mech=bd.TXL, B=1, H=2, L=1000, dtype=bd.BF16, causal=True)
    assert ws(txl, 1) - ws(txl, 2) == 2 * (8 * 9 // 2) * 65536
    txl_full = bd.Params(mech=bd.TXL, B=1, H=2, L=1000, dtype=bd.BF16, causal=False)
    assert ws(txl_full, 1) - ws(txl_full, 2) == 2 * 64 * 65536
    mem = bd.Params(mech=bd.TXL, B=1, H=2, L=1000, dtype=bd.BF16, causal=True, mem_len=24)
    assert ws(mem, 1) - ws(mem, 2) == 2 * (8 * 9 // 2) * 65536
    same = [bd.Params(mech=bd.TXL, B=1, H=2, L=1000, dtype=bd.F32, causal=True),
            bd.Params(mech=bd.T5, B=1, H=2, L=1000, dtype=bd.BF16),
            bd.Params(mech=bd.SHAW, B=1, H=2, L=1000, dtype=bd.BF16),
            bd.Params(mech=bd.DEBERTA, B=1, H=2, L=1000, dtype=bd.BF16),
            bd.Params(mech=bd.TXL, B=1, H=2, L=1000, dtype=bd.BF16, kernel_path=bd.PATH_SIMT)]
    for P in same:
        assert ws(P, 2) == ws(P, 1)
    for bad in (-1, 3):
        with pytest.raises(bd.RelposError):
            ws(txl, bad)


def test_backward_workspace_holds_the_stored_tiles(lib):
    """The Transformer-XL tensor-core backward keeps each 128 x 128 tile's P and dS (64 KB)
    in the workspace while they fit in 32 GiB, and recomputes them past that."""
    tile = 64 * 1024
    P = bd.Params(mech=bd.TXL, B=1, H=8, L=8192, causal=True)
    n_t = 8192 // 128
    assert bd.relpos_attn_workspace_size(P, 1) >= 8 * (n_t * (n_t + 1) // 2) * tile
    at_limit = bd.Params(mech=bd.TXL, B=1, H=8, L=32768, causal=False)  # 8 x 256^2 tiles = 32 GiB: stored
    assert bd.relpos_attn_workspace_size(at_limit, 1) >= 8 * 256 * 256 * tile
    big = bd.Params(mech=bd.TXL, B=1, H=9, L=32768, causal=False)  # 9 x 256^2 tiles = 36 GiB: not stored
    assert bd.relpos_attn_workspace_size(big, 1) < 9 * 256 * 256 * tile // 4
    f32 = bd.Params(mech=bd.TXL, B=1, H=8, L=8192, causal=True, dtype=bd.F32)  # CUDA-core path: none
    assert bd.relpos_attn_workspace_size(f32, 1) < 8 * (n_t * (n_t + 1) // 2) * tile


def test_null_pointers_rejected_before_any_device_work(lib):
    P = bd.Params(mech=1, B=1, H=1, L=64).c()
    null3 = (ctypes.c_void_p * 3)()
    rc = lib.relpos_attn_fwd(ctypes.byref(P), None, None, None, null3, None, None, None, 0, None, None)
    assert rc == -1
    rc = lib.relpos_attn_bwd(ctypes.byref(P), None, None, None, null3, None, None, None, None, None, None, null3, None, 0,
                             None, None)
    assert rc == -1
    # a fake non-null pointer set with a missing table is still an argument error
    fake = ctypes.c_void_p(0x1000)
    rc = lib.relpos_attn_fwd(ctypes.byref(P), fake, fake, fake, null3, fake, fake, None, 0, None, None)
    assert rc == -1


def test_workspace_checked_before_launch(lib):
    P = bd.Params(mech=0, B=1, H=1, L=64).c()  # T5 forward needs workspace
    fake = ctypes.c_void_p(0x1000)
    rel = (ctypes.c_void_p * 3)(0x1000, None, None)
    assert lib.relpos_attn_fwd(ctypes.byref(P), fake, fake, fake, rel, fake, fake, None, 0, None, None) == -2
    assert lib.relpos_attn_fwd(ctypes.byref(P), fake, fake, fake, rel, fake, fake, ctypes.c_void_p(0x1010), 1 << 20, None,
                               None) == -2  # misaligned


def test_t5_thresholds_match_oracle_buckets(lib):
    """The library's exact integer bucket thresholds (host side) against the
    oracle's bucket function, through the resolved-path query (validation only):
    checked indirectly on the GPU; here only that odd settings are accepted."""
    for nb, md, bidir in ((32, 128, True), (10, 40, True), (7, 20, False), (64, 1000, True)):
        bd.relpos_attn_workspace_size(bd.Params(mech=0, B=1, H=1, L=100, t5_num_buckets=nb, t5_max_distance=md,
                                                t5_bidirectional=bidir), 0)


def test_resolved_paths(lib):
    """Which kernel family each pass runs (host-side dispatch, no device work): bf16
    runs on the tensor cores except Shaw's value-side table with c > 64 (Shaw with c > 64
    and no value table runs on the Transformer-XL tensor-core kernels); float32 and an
    explicit CUDA-core request always run the CUDA-core kernels."""
    TC, SIMT = bd.PATH_TC, bd.PATH_SIMT
    want = {  # (mech, clip) -> (forward, backward) for bf16, automatic choice
        (bd.T5, 64): (TC, TC),
        (bd.SHAW, 64): (TC, TC),
        (bd.SHAW, 65): (TC, TC),
        (bd.SHAW, 100): (TC, TC),
        (bd.SHAW, 4096): (TC, TC),
        (bd.TXL, 64): (TC, TC),
        (bd.DEBERTA, 64): (TC, TC),
        (bd.ALIBI, 64): (TC, TC),
    }
    for (mech, clip), (f, b) in want.items():
        P = bd.Params(mech=mech, B=1, H=2, L=300, shaw_clip=clip)
        assert (bd.relpos_attn_resolved_path(P, 0), bd.relpos_attn_resolved_path(P, 1)) == (f, b), (mech, clip)
        P32 = bd.Params(mech=mech, B=1, H=2, L=300, shaw_clip=clip, dtype=bd.F32)
        assert bd.relpos_attn_resolved_path(P32, 0) == SIMT and bd.relpos_attn_resolved_path(P32, 1) == SIMT
        Ps = bd.Params(mech=mech, B=1, H=2, L=300, shaw_clip=clip, kernel_path=bd.PATH_SIMT)
        assert bd.relpos_attn_resolved_path(Ps, 0) == SIMT and bd.relpos_attn_resolved_path(Ps, 1) == SIMT
    # DeBERTa: every span takes the tensor-core backward
    for span, want_b in ((256, TC), (32, TC), (96, TC), (24, TC), (288, TC), (1, TC), (4096, TC)):
        assert bd.relpos_attn_resolved_path(bd.Params(mech=bd.DEBERTA, B=1, H=2, L=300, deberta_span=span), 1) == want_b, span
    # Shaw's value-side term: tensor cores in both passes for c <= 64
    Pv = bd.Params(mech=bd.SHAW, B=1, H=2, L=300, shaw_value=True)
    assert (bd.relpos_attn_resolved_path(Pv, 0), bd.relpos_attn_resolved_path(Pv, 1)) == (TC, TC)
    Pv65 = bd.Params(mech=bd.SHAW, B=1, H=2, L=300, shaw_value=True, shaw_clip=65)
    assert (bd.relpos_attn_resolved_path(Pv65, 0), bd.relpos_attn_resolved_path(Pv65, 1)) == (SIMT, SIMT)
    with pytest.raises(bd.RelposError):
        bd.relpos_attn_resolved_path(bd.Params(mech=bd.SHAW, B=1, H=2, L=300, shaw_value=True, shaw_clip=65,
                                               kernel_path=bd.PATH_TC), 1)
    # T5: a band of tiles with more than one bias value of any width on the tensor cores
    # (all three tiles at L = 300; about 250 band tiles at L = 32768, max_distance 20000)
    wide = dict(mech=bd.T5, B=1, H=2, t5_max_distance=1000)
    assert bd.relpos_attn_resolved_path(bd.Params(L=4096, **wide), 1) == TC
    assert bd.relpos_attn_resolved_path(bd.Params(L=300, **wide), 1) == TC
    wider = dict(mech=bd.T5, B=1, H=2, t5_max_distance=20000)
    assert bd.relpos_attn_resolved_path(bd.Params(L=32768, **wider), 1) == TC
    assert bd.relpos_attn_resolved_path(bd.Params(L=32768, t5_num_buckets=64, **wider), 1) == TC
    assert bd.relpos_attn_resolved_path(bd.Params(L=4096, t5_bidirectional=False, **wide), 1) == TC  # one side flat


def test_debug_build_exports_the_same_abi():
    """The RELPOS_DEBUG build (index-checked stores) is a complete library with the same
    exported C ABI."""
    path = bld.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert {s for s in exported if s.startswith("relpos")} == set(declared_symbols())
    dlib = ctypes.CDLL(path)
    assert dlib.relpos_attn_version() == 10800
