"""The RELPOS_DEBUG build of the library on the GPU: its kernels check the indices of
their global stores (writing RELPOS_ERR_BOUNDS to the status word and skipping the access
when a check fails); on correct inputs no check fails, the status word stays 0 and every
output still matches the oracle."""
import pytest
import torch

from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200 import build as bld
from attention_fwd_bwd_flashattention_b200.inputs import DEBERTA, SHAW, T5, TXL, Workload, make_inputs

from _parity import compare_full, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_library():
    bld.build(debug=True)
    bd.use_library(bd.DEBUG_LIB)
    yield
    bd.use_library(bd.RELEASE_LIB)


CASES = [
    Workload("dbg_txl_causal", TXL, torch.bfloat16, True, 2, 2, 700),
    Workload("dbg_txl_full", TXL, torch.bfloat16, False, 1, 2, 300),
    Workload("dbg_shaw", SHAW, torch.bfloat16, False, 2, 2, 300, shaw_clip=64, rel_std=1.0),
    Workload("dbg_deberta", DEBERTA, torch.bfloat16, False, 1, 2, 300, deberta_span=64, rel_std=1.0),
    Workload("dbg_t5", T5, torch.bfloat16, True, 1, 2, 300),
]


@pytest.mark.parametrize("bwd_pass", [1, 2], ids=["stored_tiles", "smallest_workspace"])
@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_debug_build_parity(debug_library, wl, bwd_pass):
    assert bd.lib_path() == bd.DEBUG_LIB
    inp = make_inputs(wl, seed=wl.L)
    out = run_gpu(wl, inp, bd.PATH_AUTO, bwd_pass=bwd_pass)  # asserts the status word stayed 0
    compare_full(wl, inp, out)
