"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element.

Tolerances are the workloads': max-abs 1e-4 on O for float32 inputs and 2e-2
for bfloat16, relative L2 1e-4 / 2e-2 on every gradient (dQ, dK, dV and each
relative-parameter gradient).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200.inputs import (ALIBI, DEBERTA, SHAW, T5, TXL, WORKLOADS, Workload, make_inputs,
                                                           to_f64)

from _parity import TOL, compare_full, f64, maxabs, oracle_cfg, params_of, rel_l2, run_gpu

pytestmark = pytest.mark.gpu

MECHS = {"t5": T5, "shaw": SHAW, "txl": TXL, "deberta": DEBERTA, "alibi": ALIBI}


def small_wl(mech, dtype, causal, L, B=2, H=2, **kw):
    kw.setdefault("shaw_clip", 64)
    kw.setdefault("deberta_span", 24)
    return Workload(f"small_{mech}_{L}", MECHS[mech], dtype, causal, B, H, L, **kw)


# --------------------------------------------------------------------------
# small shapes: several tiles and a ragged tail, every mechanism, both dtypes,
# causal and not, on both kernel families
# --------------------------------------------------------------------------
SMALL_L = [1, 17, 64, 130, 257, 300, 700]


@pytest.mark.parametrize("path", [bd.PATH_SIMT, bd.PATH_AUTO], ids=["simt", "auto"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("mech", list(MECHS))
@pytest.mark.parametrize("L", SMALL_L)
def test_parity_small(mech, causal, dtype, L, path):
    if path == bd.PATH_AUTO and dtype == torch.float32:
        pytest.skip("float32 always runs the CUDA-core kernels")
    wl = small_wl(mech, dtype, causal, L)
    inp = make_inputs(wl, seed=L)
    out = run_gpu(wl, inp, path)
    compare_full(wl, inp, out)


@pytest.mark.parametrize("path", [bd.PATH_SIMT, bd.PATH_AUTO], ids=["simt", "auto"])
def test_parity_deberta_span256(path):
    wl = Workload("deb600", DEBERTA, torch.bfloat16, False, 1, 2, 600)
    inp = make_inputs(wl, 3)
    compare_full(wl, inp, run_gpu(wl, inp, path))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("L", [130, 700])
def test_parity_txl_smallest_backward_workspace(L, causal):
    """Transformer-XL bf16 backward given only the smallest workspace: the kernels that
    recompute S, P and dS instead of storing the tiles; every output against the oracle."""
    wl = small_wl("txl", torch.bfloat16, causal, L)
    P = params_of(wl, bd.PATH_AUTO)
    assert bd.relpos_attn_workspace_size(P, 2) < bd.relpos_attn_workspace_size(P, 1)
    inp = make_inputs(wl, seed=L + 1)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO, bwd_pass=2))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_stored_tiles_and_smallest_workspace_agree_bitwise(causal):
    """The Transformer-XL backward with its stored P / dS tiles (streaming kernels) and
    with the smallest workspace (recomputing kernels) accumulate the same products in
    the same order: every output is bit-for-bit the same."""
    wl = small_wl("txl", torch.bfloat16, causal, 700)
    inp = make_inputs(wl, seed=21)
    a = run_gpu(wl, inp, bd.PATH_AUTO, bwd_pass=1)
    b = run_gpu(wl, inp, bd.PATH_AUTO, bwd_pass=2)
    for key in ("dq", "dk", "dv"):
        assert torch.equal(a[key], b[key]), key
    for n, (x, y) in enumerate(zip(a["drel"], b["drel"])):
        assert torch.equal(x, y), n


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("M,L", [(64, 130), (100, 300), (256, 256), (5, 1), (128, 128), (300, 200), (1000, 700)])
def test_parity_txl_memory(M, L, dtype):
    """Transformer-XL with M cached keys / values before the segment's L: every output
    against the oracle's memory formula.  Query tiles that hold only memory placeholders
    (floor(M / 128) of them on the tensor cores, floor(M / 64) on the CUDA cores) are not
    computed at all; the cases put M below, on and across those tile boundaries."""
    g = torch.Generator().manual_seed(M * 7 + L)
    B, H, d = 2, 2, 64

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(dtype)

    q, do = rn(B, H, L, d), rn(B, H, L, d)
    k, v = rn(B, H, M + L, d), rn(B, H, M + L, d)
    rel = [rn(H, M + L, d, std=0.3), rn(H, d, std=0.3), rn(H, d, std=0.3)]
    s = 1.0 / 8.0
    P = bd.Params(mech=TXL, B=B, H=H, L=L, dtype=bd.BF16 if dtype == torch.bfloat16 else bd.F32, causal=True,
                  scale=s, mem_len=M)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    reld = [r.to(dev) for r in rel]
    o, lse = bd.forward(P, qd, kd, vd, reld)
    dq, dk, dv, drel = bd.backward(P, qd, kd, vd, reld, o, lse, dod)
    torch.cuda.synchronize()
    Q, K, V, G = (to_f64(t) for t in (q, k, v, do))
    R = [to_f64(r) for r in rel]
    O, LSE = orc.txl_memory_forward(Q, K, V, R, s)
    dQ, dK, dV, dR = orc.txl_memory_backward(Q, K, V, R, G, s)
    tol = TOL[dtype]
    assert maxabs(f64(o), O) <= tol
    assert maxabs(f64(lse), LSE) <= tol
    for got, want in [(dq, dQ), (dk, dK), (dv, dV)] + list(zip(drel, dR)):
        assert rel_l2(f64(got), want) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip,L", [(3, 17), (3, 130), (64, 300), (100, 257)])
def test_parity_shaw_value_term(clip, L, causal, dtype):
    """Shaw with the value-side table aV: O, LSE, dQ, dK, dV, da and daV."""
    wl = Workload("shaw_val", SHAW, dtype, causal, 2, 2, L, shaw_clip=clip, shaw_value=True)
    inp = make_inputs(wl, clip + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


def test_parity_shaw_value_term_key_lengths_and_full_size():
    wl = Workload("shaw_val_len", SHAW, torch.bfloat16, False, 3, 2, 500, shaw_clip=20, shaw_value=True)
    lens = (500, 0, 201)
    inp = make_inputs(wl, 7)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO, seqlens_k=lens), seqlens_k=lens)
    wl = WORKLOADS["shaw_value_L2048_bf16"]
    inp = make_inputs(wl, 0)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO), heads=slice(0, 2))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("span", [32, 96, 160, 256])
@pytest.mark.parametrize("L", [130, 700, 1100])
def test_parity_deberta_tensor_core_backward(span, causal, L):
    """DeBERTa spans on the bf16 tensor-core backward (offset-ordered dS copies and
    their GEMMs), with the band of tiles narrower than, equal to and wider than the
    sequence."""
    wl = Workload("deb_tc", DEBERTA, torch.bfloat16, causal, 2, 2, L, deberta_span=span)
    assert bd.relpos_attn_resolved_path(params_of(wl, bd.PATH_AUTO), 1) == bd.PATH_TC
    inp = make_inputs(wl, span + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_parity_deberta_tensor_core_key_lengths(causal):
    wl = Workload("deb_tc_len", DEBERTA, torch.bfloat16, causal, 3, 2, 700, deberta_span=128)
    lens = (700, 0, 257)
    inp = make_inputs(wl, 5)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO, seqlens_k=lens), seqlens_k=lens)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip", [1, 7, 33, 64, 100])
@pytest.mark.parametrize("L", [300, 700])
def test_parity_shaw_clip(clip, causal, L):
    """Shaw's clip decides which tiles hold unclipped offsets (the tensor-core backward's
    band tiles: only the diagonal one for small c) and where each row's clipped pairs
    start; c > 64 runs on the Transformer-XL kernels over the table expanded by offset."""
    wl = small_wl("shaw", torch.bfloat16, causal, L, shaw_clip=clip)
    P = bd.Params(mech=SHAW, B=wl.B, H=wl.H, L=L, causal=causal, shaw_clip=clip)
    assert bd.relpos_attn_resolved_path(P, 0) == bd.PATH_TC
    assert bd.relpos_attn_resolved_path(P, 1) == bd.PATH_TC
    inp = make_inputs(wl, seed=clip + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("path", [bd.PATH_SIMT, bd.PATH_AUTO], ids=["simt", "auto"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("mech", list(MECHS))
@pytest.mark.parametrize("L,lens", [(300, (300, 171, 0)), (700, (129, 700, 384))])
def test_parity_key_lengths(mech, causal, L, lens, path):
    """Variable-length batches: per-batch key lengths inside a tile, on a tile
    boundary, the full length and an empty key set (O = 0, LSE = -inf)."""
    wl = small_wl(mech, torch.bfloat16, causal, L, B=len(lens))
    inp = make_inputs(wl, seed=L + 3)
    compare_full(wl, inp, run_gpu(wl, inp, path, seqlens_k=lens), seqlens_k=lens)


def test_key_lengths_on_the_host_are_rejected():
    wl = small_wl("txl", torch.bfloat16, False, 64, B=2)
    P = bd.Params(mech=TXL, B=2, H=2, L=64, seqlens_k=torch.tensor([64, 3], dtype=torch.int32))
    q = torch.zeros(2, 2, 64, 64, dtype=torch.bfloat16, device="cuda")
    rel = [torch.zeros(2, 127, 64, dtype=torch.bfloat16, device="cuda"), torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda"),
           torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda")]
    with pytest.raises(bd.RelposError) as ei:
        bd.forward(P, q, q, q, rel)
    assert ei.value.code == -1


@pytest.mark.parametrize("which", ["q", "a", "aV"])
def test_misaligned_tensor_core_operands_are_rejected(which):
    """The tensor-core path reads Q, K, V, dO and the bf16 tables with 16-byte loads (TMA
    and vector loads): a tensor that starts 2 bytes off a 16-byte boundary is refused on
    the host with RELPOS_ERR_INVALID_ARG, before anything is launched."""
    P = bd.Params(mech=SHAW, B=1, H=2, L=64, shaw_clip=8, shaw_value=True)
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16, device="cuda")
    a = torch.zeros(2, 17, 64, dtype=torch.bfloat16, device="cuda")
    aV = torch.zeros(2, 17, 64, dtype=torch.bfloat16, device="cuda")

    def off(t):  # same shape, one element further on: 2 bytes past the 16-byte boundary
        return torch.zeros(t.numel() + 1, dtype=t.dtype, device=t.device)[1:].view(t.shape)

    if which == "q":
        q = off(q)
    elif which == "a":
        a = off(a)
    else:
        aV = off(aV)
    o, lse = torch.empty_like(q), torch.empty(1, 2, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(bd.RelposError) as ei:
        bd.relpos_attn_fwd(P, q, q, q, [a, aV], o, lse, bd.workspace(P, 0, q.device))
    assert ei.value.code == -1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    drel = [torch.empty(2, 17, 64, dtype=torch.float32, device="cuda") for _ in range(2)]
    with pytest.raises(bd.RelposError) as ei:
        bd.relpos_attn_bwd(P, q, q, q, [a, aV], o, lse, q, dq, dk, dv, drel, bd.workspace(P, 1, q.device))
    assert ei.value.code == -1
    torch.cuda.synchronize()


def test_key_lengths_match_truncated_keys():
    """A batch whose keys stop at Lk gives the same O and LSE as the same keys with
    everything after Lk replaced (T5 and Shaw depend only on j - i)."""
    wl = small_wl("shaw", torch.bfloat16, False, 520, B=2)
    inp = make_inputs(wl, seed=9)
    lens = (333, 520)
    a = run_gpu(wl, inp, bd.PATH_AUTO, seqlens_k=lens)
    inp2 = dict(inp)
    for n in ("k", "v"):
        t = inp[n].clone()
        t[0, :, 333:] = torch.randn(t[0, :, 333:].shape, generator=torch.Generator().manual_seed(1)).to(t.dtype)
        inp2[n] = t
    b = run_gpu(wl, inp2, bd.PATH_AUTO, seqlens_k=lens)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"]) and torch.equal(a["dq"], b["dq"])
    assert torch.all(b["dk"][0, :, 333:] == 0) and torch.all(b["dv"][0, :, 333:] == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_parity_t5_unidirectional_and_odd_buckets(causal):
    for nb, md, bidir in ((32, 128, False), (10, 40, True), (7, 20, False)):
        wl = Workload("t5x", T5, torch.float32, causal, 1, 2, 300, t5_num_buckets=nb, t5_max_distance=md,
                      t5_bidirectional=bidir)
        inp = make_inputs(wl, nb)
        compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("causal", [False, True])
def test_parity_bias_family_tensor_core_backward(causal):
    """T5 bucket layouts whose band of distinct-bias tiles is narrow, wide or one-sided,
    and ALiBi slopes from nearly flat to sharply local, on the bf16 tensor-core backward."""
    for nb, md, bidir in ((32, 128, True), (10, 40, True), (7, 20, False), (32, 600, True), (64, 900, False)):
        wl = Workload("t5x", T5, torch.bfloat16, causal, 1, 2, 1100, t5_num_buckets=nb, t5_max_distance=md,
                      t5_bidirectional=bidir)
        P = params_of(wl, bd.PATH_AUTO)
        assert bd.relpos_attn_resolved_path(P, 1) == bd.PATH_TC, (nb, md, bidir)
        inp = make_inputs(wl, nb)
        compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))
    # a wide band of distinct-bias tiles (max_distance 3000: about 47 tiles)
    wl = Workload("t5_wide", T5, torch.bfloat16, causal, 1, 2, 3500, t5_num_buckets=32, t5_max_distance=3000)
    assert bd.relpos_attn_resolved_path(params_of(wl, bd.PATH_AUTO), 1) == bd.PATH_TC
    inp = make_inputs(wl, 11)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))
    wl = Workload("alibi_x", ALIBI, torch.bfloat16, causal, 2, 4, 1100)
    inp = make_inputs(wl, 3)
    inp["rel"] = [torch.tensor([1e-4, 0.02, 1.0, 8.0])]
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("causal", [False, True])
def test_parity_t5_band_of_89_tiles_L8192(causal):
    """T5 buckets that stay distinct across most of an 8K sequence (64 buckets,
    max_distance 8192: 63 buckets in use, a band of 89 distinct-bias tiles around each
    query tile) on the tensor-core backward, which folds each band tile's offset sums
    into buckets as it goes; every output of head 0 (its table gradient is exact with one
    batch) against the oracle."""
    wl = Workload("t5_band89", T5, torch.bfloat16, causal, 1, 2, 8192, t5_num_buckets=64, t5_max_distance=8192)
    assert bd.relpos_attn_resolved_path(params_of(wl, bd.PATH_AUTO), 1) == bd.PATH_TC
    inp = make_inputs(wl, 13)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO), heads=slice(0, 1))


def test_t5_small_buckets_and_fp32_config():
    # the fp32 T5 workload itself (one batch, two heads, L = 128) on its own path
    wl = WORKLOADS["t5_L128_fp32"]
    inp = make_inputs(wl, 0)
    errs = compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))
    assert errs["o"] <= 1e-4


def test_determinism():
    for name in ("shaw_L2048_bf16",):
        wl = WORKLOADS[name].with_(L=300, B=1, H=2)
        inp = make_inputs(wl, 1)
        a = run_gpu(wl, inp, bd.PATH_AUTO)
        b = run_gpu(wl, inp, bd.PATH_AUTO)
        for key in ("o", "lse", "dq", "dk", "dv"):
            assert torch.equal(a[key], b[key]), key
        for x, y in zip(a["drel"], b["drel"]):
            assert torch.equal(x, y)
    for mech in ("txl", "deberta", "t5"):
        wl = small_wl(mech, torch.bfloat16, mech == "txl", 200)
        inp = make_inputs(wl, 2)
        a = run_gpu(wl, inp, bd.PATH_AUTO)
        b = run_gpu(wl, inp, bd.PATH_AUTO)
        for x, y in zip(a["drel"] + [a["dq"], a["dk"]], b["drel"] + [b["dq"], b["dk"]]):
            assert torch.equal(x, y), mech


def test_errors_are_reported_not_raised_on_device():
    wl = small_wl("shaw", torch.bfloat16, False, 64)
    P = bd.Params(mech=SHAW, B=2, H=2, L=64, d=32)
    with pytest.raises(bd.RelposError) as e:
        bd.relpos_attn_workspace_size(P, 0)
    assert e.value.code == -1
    inp = make_inputs(wl, 0)
    P = bd.Params(mech=SHAW, B=2, H=2, L=64)
    q = inp["q"].cuda()
    o = torch.empty_like(q)
    lse = torch.empty(2, 2, 64, device="cuda")
    with pytest.raises(bd.RelposError) as e:
        bd.relpos_attn_fwd(P, q, q, q, [None], o, lse, None)
    assert e.value.code == -1


# --------------------------------------------------------------------------
# the workloads at full size
# --------------------------------------------------------------------------
def test_parity_shaw_L2048_full():
    wl = WORKLOADS["shaw_L2048_bf16"]
    inp = make_inputs(wl, 0)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("name", ["txl_causal_L8192_bf16", "deberta_L8192_bf16", "txl_L8192_bf16",
                                  "txl_varlen_B4_L8192_bf16", "alibi_causal_L8192_bf16", "t5_causal_L8192_bf16"])
def test_parity_L8192_one_head(name):
    """Every output of head 0 (table gradients of that head over the whole batch) at
    L = 8192; the variable-length batch runs with its key lengths."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, 0)
    out = run_gpu(wl, inp, bd.PATH_AUTO, seqlens_k=wl.seqlens_k)
    compare_full(wl, inp, out, heads=slice(0, 1), seqlens_k=wl.seqlens_k)


@pytest.mark.parametrize("name", ["txl_L16384_bf16", "txl_L32768_bf16"])
def test_parity_long_sampled(name):
    """Sampled query rows of O, LSE and dQ (each a function of its own row), plus
    properties that hold at any size: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0 and
    sum_rho dr_rho = 0 for Transformer-XL (each row of dS sums to zero)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, 0)
    out = run_gpu(wl, inp, bd.PATH_AUTO)
    tol = TOL[wl.dtype]
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 127, 128], np.random.default_rng(0).integers(0, wl.L, 10), [wl.L - 1]]))
    h = slice(0, 1)
    q, k, v, do = (to_f64(inp[n])[:, h] for n in ("q", "k", "v", "do"))
    rel = [to_f64(r)[h] for r in inp["rel"]]
    cfg = oracle_cfg(wl)
    O, LSE = orc.forward(wl.mech, q, k, v, rel, wl.causal, wl.scale, cfg, rows=rows)
    assert maxabs(f64(out["o"][:, h][:, :, rows]), O) <= tol
    assert maxabs(f64(out["lse"][:, h][:, :, rows]), LSE) <= tol
    dq = orc.backward_rows(wl.mech, q, k, v, rel, wl.causal, do, rows, wl.scale, cfg)
    assert rel_l2(f64(out["dq"][:, h][:, :, rows]), dq) <= tol
    dv_sum = f64(out["dv"].float().sum(dim=2))
    do_sum = to_f64(inp["do"]).sum(axis=2)
    assert rel_l2(dv_sum, do_sum) <= tol
    dk_sum = f64(out["dk"].float().sum(dim=2))
    assert np.max(np.abs(dk_sum)) <= tol * np.linalg.norm(f64(out["dk"][0, 0])) + 1e-3
    dr_sum = f64(out["drel"][0].sum(dim=1))
    assert np.max(np.abs(dr_sum)) <= tol * float(torch.linalg.norm(out["drel"][0][0])) + 1e-4


def test_bounded_wait_runs_out_and_reports():
    """Failure detection: a device wait on a barrier nothing completes gives up after its
    limit, writes RELPOS_ERR_TIMEOUT to the status word and returns; the context stays
    usable (a forward pass runs and matches the oracle afterwards)."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    limit = 50_000_000  # 50 ms
    bd.relpos_selftest_wait(limit, status, elapsed)
    torch.cuda.synchronize()
    assert int(status.item()) == -5, bd.strerror(int(status.item()))
    assert limit <= int(elapsed.item()) < limit + 20_000_000
    with pytest.raises(bd.RelposError):
        bd.relpos_selftest_wait(limit, torch.zeros(1, dtype=torch.int32), elapsed)  # host status word
    wl = small_wl("txl", torch.bfloat16, True, 130)
    inp = make_inputs(wl, seed=7)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


# --------------------------------------------------------------------------
# Shaw and DeBERTa with their tables drawn at std 1.0: at the workloads' 0.02 the
# relative term moves the outputs by about the tolerance, at 1.0 a gather one offset
# off, a flipped offset sign, a dropped term or swapped tables moves them by many
# tolerances (tests/test_parity_power.py, with the oracle alone, on these shapes)
# --------------------------------------------------------------------------
O1_L = [130, 300, 700, 1100]


@pytest.mark.parametrize("path", [bd.PATH_SIMT, bd.PATH_AUTO], ids=["simt", "auto"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip", [1, 7, 64, 100])
@pytest.mark.parametrize("L", O1_L)
def test_parity_shaw_o1_tables(L, clip, causal, path):
    wl = Workload("shaw_o1", SHAW, torch.bfloat16, causal, 2, 2, L, shaw_clip=clip, rel_std=1.0)
    inp = make_inputs(wl, seed=clip + L)
    compare_full(wl, inp, run_gpu(wl, inp, path))


@pytest.mark.parametrize("path", [bd.PATH_SIMT, bd.PATH_AUTO], ids=["simt", "auto"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("span", [32, 96, 256, 40])
@pytest.mark.parametrize("L", O1_L)
def test_parity_deberta_o1_tables(L, span, causal, path):
    wl = Workload("deb_o1", DEBERTA, torch.bfloat16, causal, 2, 2, L, deberta_span=span, rel_std=1.0)
    inp = make_inputs(wl, seed=span + L)
    compare_full(wl, inp, run_gpu(wl, inp, path))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip,L", [(3, 130), (64, 300), (100, 700)])
def test_parity_shaw_value_o1_tables(clip, L, causal):
    wl = Workload("shaw_val_o1", SHAW, torch.bfloat16, causal, 2, 2, L, shaw_clip=clip, shaw_value=True, rel_std=1.0)
    inp = make_inputs(wl, clip + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip,L", [(65, 300), (100, 1100), (257, 700), (1000, 700), (4096, 130)])
def test_parity_shaw_wide_clip(clip, L, causal):
    """Shaw with c > 64 on the Transformer-XL tensor-core kernels: the table expanded to
    one row per offset, its gradient summed back into the 2c + 1 rows.  Tables at std
    1.0; interior rows, both end rows (the clipped offsets) and c >= L (no offset
    clipped, the end rows' gradients zero)."""
    wl = Workload("shaw_wide", SHAW, torch.bfloat16, causal, 2, 2, L, shaw_clip=clip, rel_std=1.0)
    inp = make_inputs(wl, seed=clip + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_TC))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_parity_shaw_wide_clip_key_lengths_smallest_workspace(causal):
    """The wide-clip route with per-batch key lengths (an empty key set among them) and
    with the smallest backward workspace (the recomputing Transformer-XL kernels)."""
    wl = Workload("shaw_wide_len", SHAW, torch.bfloat16, causal, 3, 2, 700, shaw_clip=150, rel_std=1.0)
    lens = (700, 0, 257)
    inp = make_inputs(wl, 11)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO, seqlens_k=lens, bwd_pass=2), seqlens_k=lens)


def test_parity_shaw_L2048_o1_tables():
    """The Shaw workload's shape (B2 H8 L2048, clip 64), tables at std 1.0: every output."""
    wl = WORKLOADS["shaw_L2048_bf16"].with_(rel_std=1.0)
    inp = make_inputs(wl, 0)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("span,L", [(1, 300), (24, 700), (100, 1100), (300, 700), (700, 1100), (2000, 300)])
def test_parity_deberta_any_span(span, L, causal):
    """DeBERTa's tensor-core backward at spans whose 2k table rows are not a multiple of
    64 (rows kept Wp = 2k rounded up to 64 long, the tables read from zero-padded copies)
    or exceed 512 (the relation products in 512-column pieces, the rows kernel's K steps
    in groups); k = 1 (no interior offset) and k >= L.  Tables at std 1.0."""
    wl = Workload("deb_span", DEBERTA, torch.bfloat16, causal, 2, 2, L, deberta_span=span, rel_std=1.0)
    P = params_of(wl, bd.PATH_AUTO)
    assert bd.relpos_attn_resolved_path(P, 1) == bd.PATH_TC
    inp = make_inputs(wl, seed=span + L)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_TC))


def test_parity_deberta_L8192_o1_tables_one_head():
    """The DeBERTa workload's shape (B1 H12 L8192, span 256), tables at std 1.0: every
    output of head 0 (its table gradients included)."""
    wl = WORKLOADS["deberta_L8192_bf16"].with_(rel_std=1.0)
    inp = make_inputs(wl, 0)
    compare_full(wl, inp, run_gpu(wl, inp, bd.PATH_AUTO), heads=slice(0, 1))
