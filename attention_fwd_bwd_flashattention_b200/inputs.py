"""Seeded synthetic inputs for relative-position attention.

This module only draws random numbers and lays them out: it holds none of the
attention arithmetic.  Both the CUDA path's tests/bench and the CPU oracle are
fed from it.  Every tensor is drawn on the CPU from one ``torch.Generator`` in a
fixed order, so a seed gives the same values on every machine.

Distributions (per the workload definitions): Q, K, V, dO ~ N(0, 1); T5 bias
table t[H, 32] ~ N(0, 0.1); Shaw table a[H, 129, d] ~ N(0, 0.02); DeBERTa Kr,
Qr [H, 512, d] ~ N(0, 0.02); Transformer-XL u, v [H, d] ~ N(0, 0.02) and
r = sinusoid(offset) [n_off, 512] @ W_R [512, H*d] with W_R ~ N(0, 0.02);
ALiBi slopes m[h] = 2^(-8 (h + 1) / H), the geometric sequence of the ALiBi paper
(Press et al.) for its heads (fixed, not drawn).
The sinusoid is the Transformer-XL one: [sin(delta w_k), cos(delta w_k)]
concatenated, w_k = 10000^(-2k/512), k = 0..255.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

T5, SHAW, TXL, DEBERTA, ALIBI = 0, 1, 2, 3, 4
MECH_IDS = {"t5": T5, "shaw": SHAW, "txl": TXL, "deberta": DEBERTA, "alibi": ALIBI}
MECH_NAMES = {v: k for k, v in MECH_IDS.items()}

TXL_EMB = 512  # width of the Transformer-XL sinusoid fed to W_R


@dataclass(frozen=True)
class Workload:
    name: str
    mech: int
    dtype: torch.dtype
    causal: bool
    B: int
    H: int
    L: int
    d: int = 64
    t5_num_buckets: int = 32
    t5_max_distance: int = 128
    t5_bidirectional: bool = True
    shaw_clip: int = 64
    deberta_span: int = 256
    seqlens_k: Optional[Tuple[int, ...]] = None  # per-batch key lengths (variable-length batch)
    shaw_value: bool = False  # Shaw: also the value-side table aV
    # std of the drawn Shaw (a, aV) and DeBERTa (Kr, Qr) tables instead of the workload's
    # 0.02; None keeps 0.02.  Parity tests draw them at O(1) so that the relative term
    # moves the outputs by far more than the tolerance.
    rel_std: Optional[float] = None
    # Transformer-XL (causal) memory: M cached keys / values before the segment's L
    # queries; k, v and r then have M + L rows
    mem_len: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(3 * self.d) if self.mech == DEBERTA else 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads: a small fp32 T5 case, Shaw at 2K, Transformer-XL causal
# at 8K, DeBERTa at 8K and a non-causal Transformer-XL length sweep.
WORKLOADS = {
    "t5_L128_fp32": Workload("t5_L128_fp32", T5, torch.float32, False, 1, 2, 128),
    "shaw_L2048_bf16": Workload("shaw_L2048_bf16", SHAW, torch.bfloat16, False, 2, 8, 2048),
    "txl_causal_L8192_bf16": Workload("txl_causal_L8192_bf16", TXL, torch.bfloat16, True, 1, 8, 8192),
    "deberta_L8192_bf16": Workload("deberta_L8192_bf16", DEBERTA, torch.bfloat16, False, 1, 12, 8192),
}
for _L in (4096, 8192, 16384, 32768):
    WORKLOADS[f"txl_L{_L}_bf16"] = Workload(f"txl_L{_L}_bf16", TXL, torch.bfloat16, False, 1, 8, _L)
# A variable-length batch of the speech-encoder shape (H = 8, d = 64, non-causal): four
# utterances padded to 8192 frames, key lengths fixed so that runs are comparable.
WORKLOADS["txl_varlen_B4_L8192_bf16"] = Workload("txl_varlen_B4_L8192_bf16", TXL, torch.bfloat16, False, 4, 8, 8192,
                                                 seqlens_k=(8192, 6144, 4000, 2500))
# ALiBi, causal decoder shape at 8K, and T5 at the same size for comparison.
# Shaw with its value-side table as well (CUDA-core kernels), the Shaw shape at 2K.
WORKLOADS["shaw_value_L2048_bf16"] = Workload("shaw_value_L2048_bf16", SHAW, torch.bfloat16, False, 2, 8, 2048,
                                              shaw_value=True)
WORKLOADS["alibi_causal_L8192_bf16"] = Workload("alibi_causal_L8192_bf16", ALIBI, torch.bfloat16, True, 1, 8, 8192)
# Transformer-XL with a segment memory as long as the segment (M = L = 4096): the same
# 8192 causal positions as the 8K workload, the first 4096 of them cached keys only.
WORKLOADS["txl_mem_M4096_L4096_bf16"] = Workload("txl_mem_M4096_L4096_bf16", TXL, torch.bfloat16, True, 1, 8, 4096,
                                                 mem_len=4096)
WORKLOADS["t5_causal_L8192_bf16"] = Workload("t5_causal_L8192_bf16", T5, torch.bfloat16, True, 1, 8, 8192,
                                             t5_bidirectional=False)


def txl_sinusoid(n_off: int, causal: bool, L: int) -> torch.Tensor:
    """[n_off, 512] float64 sinusoid of the offset each table row stands for
    (row = delta when causal, delta + L - 1 otherwise)."""
    rows = torch.arange(n_off, dtype=torch.float64)
    delta = rows if causal else rows - (L - 1)
    k = torch.arange(TXL_EMB // 2, dtype=torch.float64)
    w = torch.pow(torch.tensor(10000.0, dtype=torch.float64), -2.0 * k / TXL_EMB)
    ang = delta[:, None] * w[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)


def make_inputs(wl: Workload, seed: int = 0) -> dict:
    """All inputs of one workload as CPU tensors in the workload's dtype.

    Returns dict(q, k, v, do, rel) with rel the list of relative parameters:
    T5 [t (H,nb) fp32]; Shaw [a (H,2c+1,d)] (+ aV with the value term); TXL [r (H,n_off,d), u (H,d), v (H,d)];
    DeBERTa [Kr (H,2k,d), Qr (H,2k,d)]; ALiBi [m (H,) fp32].
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    B, H, L, d = wl.B, wl.H, wl.L, wl.d
    dt = wl.dtype

    def nrm(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, dtype=torch.float32) * std)

    Lk = L + wl.mem_len  # keys and values: the memory, then the segment
    q = nrm(B, H, L, d).to(dt)
    k = nrm(B, H, Lk, d).to(dt)
    v = nrm(B, H, Lk, d).to(dt)
    do = nrm(B, H, L, d).to(dt)
    if wl.mech == ALIBI:
        rel = [torch.pow(2.0, -8.0 * torch.arange(1, H + 1, dtype=torch.float32) / H)]
    elif wl.mech == T5:
        rel = [nrm(H, wl.t5_num_buckets, std=0.1)]
    elif wl.mech == SHAW:
        sd = 0.02 if wl.rel_std is None else wl.rel_std
        rel = [nrm(H, 2 * wl.shaw_clip + 1, d, std=sd).to(dt)]
        if wl.shaw_value:
            rel.append(nrm(H, 2 * wl.shaw_clip + 1, d, std=sd).to(dt))
    elif wl.mech == TXL:
        n_off = Lk if wl.causal else 2 * L - 1
        W_R = nrm(TXL_EMB, H * d, std=0.02).to(torch.float64)
        u = nrm(H, d, std=0.02).to(dt)
        vv = nrm(H, d, std=0.02).to(dt)
        r = (txl_sinusoid(n_off, wl.causal, Lk) @ W_R).reshape(n_off, H, d).permute(1, 0, 2).contiguous()
        rel = [r.to(dt), u, vv]
    else:
        sd = 0.02 if wl.rel_std is None else wl.rel_std
        rel = [nrm(H, 2 * wl.deberta_span, d, std=sd).to(dt), nrm(H, 2 * wl.deberta_span, d, std=sd).to(dt)]
    return dict(q=q, k=k, v=v, do=do, rel=rel)


def to_f64(t: torch.Tensor):
    """Exact upcast to a float64 numpy array (what the oracle consumes)."""
    return t.detach().to("cpu", torch.float64).numpy()
