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


# T5, bf16, causal, B = 1, H = 64: at L = 32264 the forward scratch (per-offset bias
# vectors and buckets) is exactly the size of the built-in array, one more row is too big
AT_LIMIT = dict(mech=T5, B=1, H=64, L=32264, dtype=bd.BF16, causal=True)


def test_noalloc_size_check_at_the_limit():
    assert bd.relpos_attn_workspace_size(bd.Params(**AT_LIMIT), 0) == bd.NOALLOC_SCRATCH_BYTES
    P = bd.Params(**dict(AT_LIMIT, L=AT_LIMIT["L"] + 1))
    assert bd.relpos_attn_workspace_size(P, 0) > bd.NOALLOC_SCRATCH_BYTES
    fake = torch.empty(0)
    null_stream = type("S", (), {"cuda_stream": 0})()
    with pytest.raises(bd.RelposError) as e:
        bd.relpos_attn_fwd_noalloc(P, fake, fake, fake, [fake], fake, fake, stream=null_stream)
    assert e.value.code == -2


def _check_twice(P, q, k, v, rel, tol):
    o_ref, lse_ref = bd.forward(P, q, k, v, rel)
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
        bd.relpos_attn_fwd_noalloc(P, q, k, v, rel, o, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert (o.float() - o_ref.float()).abs().max().item() <= tol
        assert (lse - lse_ref).abs().max().item() <= tol


@pytest.mark.gpu
def test_noalloc_txl_memory_twice():
    """Transformer-XL with memory (M = 100 cached keys before a 300-query segment): the
    call that takes most from the array (padded q, O and LSE rows beside u.k and v.r)."""
    dev = torch.device("cuda", 0)
    g = torch.Generator().manual_seed(11)
    B, H, L, M, d = 2, 2, 300, 100, 64

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(dev)

    q, k, v = rn(B, H, L, d), rn(B, H, M + L, d), rn(B, H, M + L, d)
    rel = [rn(H, M + L, d, std=0.3), rn(H, d, std=0.3), rn(H, d, std=0.3)]
    P = bd.Params(mech=TXL, B=B, H=H, L=L, dtype=bd.BF16, causal=True, scale=0.125, mem_len=M)
    _check_twice(P, q, k, v, rel, TOL[torch.bfloat16])


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit_twice():
    dev = torch.device("cuda", 0)
    P = bd.Params(**AT_LIMIT)
    g = torch.Generator().manual_seed(12)
    shape = (P.B, P.H, P.L, 64)
    q, k, v = (torch.randn(*shape, generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    rel = [(torch.randn(P.H, 32, generator=g) * 0.1).to(dev)]
    _check_twice(P, q, k, v, rel, TOL[torch.bfloat16])


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_noalloc_wide_clip_shaw_twice(causal):
    """Shaw with c > 64 runs on the Transformer-XL kernels: its expanded table and zero
    u / v vector also live in the built-in array."""
    dev = torch.device("cuda", 0)
    wl = Workload("shaw_wide_noalloc", SHAW, torch.bfloat16, causal, 2, 2, 300, shaw_clip=150, rel_std=1.0)
    inp = make_inputs(wl, seed=13)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    rel = [r.to(dev) for r in inp["rel"]]
    P = bd.Params(mech=SHAW, B=2, H=2, L=300, dtype=bd.BF16, causal=causal, scale=wl.scale, shaw_clip=150)
    assert bd.relpos_attn_resolved_path(P, 0) == bd.PATH_TC
    _check_twice(P, q, k, v, rel, TOL[torch.bfloat16])


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
