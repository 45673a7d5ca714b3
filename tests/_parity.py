"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding and the fp64 oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle as orc
from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200.inputs import to_f64

# tolerances: max-abs on O (and LSE), relative L2 on every gradient
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def oracle_cfg(wl):
    return orc.RelCfg(t5_num_buckets=wl.t5_num_buckets, t5_max_distance=wl.t5_max_distance, t5_bidirectional=wl.t5_bidirectional,
                      shaw_clip=wl.shaw_clip, deberta_span=wl.deberta_span, shaw_value=wl.shaw_value)


def params_of(wl, path):
    return bd.Params(mech=wl.mech, B=wl.B, H=wl.H, L=wl.L, d=wl.d, dtype=bd.BF16 if wl.dtype == torch.bfloat16 else bd.F32,
                     causal=wl.causal, scale=wl.scale, kernel_path=path, t5_num_buckets=wl.t5_num_buckets,
                     t5_max_distance=wl.t5_max_distance, t5_bidirectional=wl.t5_bidirectional, shaw_clip=wl.shaw_clip, deberta_span=wl.deberta_span,
                     shaw_value=wl.shaw_value)


def run_gpu(wl, inp, path, dev="cuda", seqlens_k=None, bwd_pass=1):
    """Forward + backward through the C ABI; the device status word must stay 0 (a
    bounded wait that ran out inside a kernel reports RELPOS_ERR_TIMEOUT there).
    seqlens_k: optional per-batch key lengths (a sequence of B ints).
    bwd_pass: the workspace-size pass of the backward's workspace (2: the smallest)."""
    P = params_of(wl, path)
    if seqlens_k is not None:
        P.seqlens_k = torch.tensor(list(seqlens_k), dtype=torch.int32, device=dev)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    rel = [r.to(dev) for r in inp["rel"]]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    bd.relpos_attn_fwd(P, q, k, v, rel, o, lse, bd.workspace(P, 0, q.device), dev_status=status)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    drel = [torch.empty(r.shape, dtype=torch.float32, device=dev) for r in rel[: P.n_rel()]]
    bd.relpos_attn_bwd(P, q, k, v, rel, o, lse, do, dq, dk, dv, drel, bd.workspace(P, bwd_pass, q.device), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"{wl.name}: device status {int(status.item())} ({bd.strerror(int(status.item()))})"
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, drel=drel)


def maxabs(got, want):
    """Largest |got - want|; entries where both are the same infinity (LSE = -inf of
    a query without keys) count as equal, an infinity on one side only as inf."""
    if not want.size:
        return 0.0
    same_inf = np.isinf(want) & (got == want)
    with np.errstate(invalid="ignore"):  # inf - inf where same_inf; masked out below
        diff = np.abs(got - want)
    return float(np.max(np.where(same_inf, 0.0, diff)))


def rel_l2(got, want):
    """||got - want|| / ||want||.  Where the exact gradient is zero (e.g. dQ at
    L = 1) the ratio is meaningless, so the largest absolute entry of got is
    returned instead (checked against the same tolerance)."""
    den = float(np.linalg.norm(want))
    num = float(np.linalg.norm(got - want))
    if den <= 1e-6 * np.sqrt(max(want.size, 1)):
        return float(np.max(np.abs(got))) if got.size else 0.0
    return num / den


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def compare_full(wl, inp, out, heads=None, seqlens_k=None):
    """Compare every output with the oracle (optionally only some heads; table
    gradients then cover those heads, which is exact when B == 1)."""
    tol = TOL[wl.dtype]
    cfg = oracle_cfg(wl)
    q, k, v, do = (to_f64(inp[n]) for n in ("q", "k", "v", "do"))
    rel = [to_f64(r) for r in inp["rel"]]
    hs = slice(None) if heads is None else heads
    if heads is not None:
        q, k, v, do = q[:, hs], k[:, hs], v[:, hs], do[:, hs]
        rel = [r[hs] for r in rel]
    O, LSE = orc.forward(wl.mech, q, k, v, rel, wl.causal, wl.scale, cfg, seqlens_k=seqlens_k)
    dq, dk, dv, drel = orc.backward(wl.mech, q, k, v, rel, wl.causal, do, wl.scale, cfg, seqlens_k=seqlens_k)
    errs = {
        "o": maxabs(f64(out["o"][:, hs]), O),
        "lse": maxabs(f64(out["lse"][:, hs]), LSE),
        "dq": rel_l2(f64(out["dq"][:, hs]), dq),
        "dk": rel_l2(f64(out["dk"][:, hs]), dk),
        "dv": rel_l2(f64(out["dv"][:, hs]), dv),
    }
    for n, g in enumerate(drel):
        errs[f"drel{n}"] = rel_l2(f64(out["drel"][n][hs]), g)
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"{wl.name}: over tolerance {tol}: {bad} (all: {errs})"
    return errs
