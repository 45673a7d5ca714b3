"""The allocation-free forward entry point (relpos_attn_fwd_noalloc).

Callers that cannot allocate device memory -- a plugin inside a framework that owns
the device-memory budget, or a latency-critical loop where cudaMalloc would
synchronise the device -- use this entry point; its scratch is a static device array
inside the library.  The GPU test checks it against the regular entry point
(relpos_attn_fwd with a caller workspace), within the parity tolerances, on two calls
in a row (the second call finds the first call's leftovers in the shared array).  The
file sorts last so a run that stops at the first failure has run everything else."""
import pytest
import torch

from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200.inputs import DEBERTA, SHAW, T5, TXL, WORKLOADS, Workload, make_inputs

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

CASES = [
    WORKLOADS["t5_L128_fp32"],
    Workload("txl_causal_small", TXL, torch.bfloat16, True, 1, 2, 700),
    Workload("txl_small", TXL, torch.bfloat16, False, 2, 2, 300),
    Workload("deberta_small", DEBERTA, torch.bfloat16, False, 1, 3, 600),
    Workload("shaw_small", SHAW, torch.bfloat16, False, 2, 2, 257),
    Workload("t5_bf16_small", T5, torch.bfloat16, True, 1, 2, 333),
]


def _params(wl):
    return bd.Params(mech=wl.mech, B=wl.B, H=wl.H, L=wl.L, dtype=bd.BF16 if wl.dtype == torch.bfloat16 else bd.F32,
                     causal=wl.causal, scale=wl.scale)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # TXL forward scratch is (B*H*L + H*(2L-1)) floats: far beyond 16 MiB here
    P = bd.Params(mech=TXL, B=64, H=64, L=4096, dtype=bd.BF16)
    assert bd.relpos_attn_workspace_size(P, 0) > bd.NOALLOC_SCRATCH_BYTES
    fake = torch.empty(0)
    null_stream = type("S", (), {"cuda_stream": 0})()  # checked on the host before any device work
    with pytest.raises(bd.RelposError) as e:
        bd.relpos_attn_fwd_noalloc(P, fake, fake, fake, [fake, fake, fake], fake, fake, stream=null_stream)
    assert e.value.code == -2


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_noalloc_matches_regular_entry_point_twice(wl):
    dev = torch.device("cuda", 0)
    inp = make_inputs(wl, seed=5)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    rel = [r.to(dev) for r in inp["rel"]]
    P = _params(wl)
    o_ref, lse_ref = bd.forward(P, q, k, v, rel)
    tol = TOL[wl.dtype]
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
        bd.relpos_attn_fwd_noalloc(P, q, k, v, rel, o, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert (o.float() - o_ref.float()).abs().max().item() <= tol
        assert (lse - lse_ref).abs().max().item() <= tol
