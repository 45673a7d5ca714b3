"""Host logic of bench.py: the FLOP accounting and the timing statistics.

The algorithmic FLOP totals of the workloads were worked out by hand from the
counting rule (U = 2 B H d #pairs; T5 2U / 5U, Shaw 2U + R / 5U + 3R, Transformer-XL
3U / 8U, DeBERTa 2U + 2R / 5U + 6R with R = 2 B H L rows d) and rounded to three
digits; the bench's own functions must reproduce them.
"""
import itertools
import math

import numpy as np
import pytest

import bench
from attention_fwd_bwd_flashattention_b200.inputs import WORKLOADS

HAND = {  # workload: (fwd, bwd) flop, or (None, total)
    "t5_L128_fp32": (None, 2.94e7),
    "shaw_L2048_bf16": (1.77e10, 4.46e10),
    "txl_causal_L8192_bf16": (1.03e11, 2.75e11),
    "deberta_L8192_bf16": (2.19e11, 5.54e11),
    "txl_L4096_bf16": (None, 1.89e11),
    "txl_L8192_bf16": (None, 7.56e11),
    "txl_L16384_bf16": (None, 3.02e12),
    "txl_L32768_bf16": (None, 1.21e13),
}


@pytest.mark.parametrize("name", list(HAND))
def test_algorithmic_flops_match_hand_totals(name):
    f, b = bench.algo_flops(WORKLOADS[name])
    want_f, want = HAND[name]
    if want_f is None:
        assert abs((f + b) / want - 1) < 0.01, (f + b, want)
    else:
        assert abs(f / want_f - 1) < 0.01, (f, want_f)
        assert abs(b / want - 1) < 0.01, (b, want)


def brute_pairs(L, B, causal, lens):
    n = 0
    for b in range(B):
        lk = L if lens is None else max(0, min(L, lens[b]))
        for i, j in itertools.product(range(L), range(L)):
            n += (j < lk) and (not causal or j <= i)
    return n


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lens", [None, (9, 0, 23, 40)])
def test_pairs_of_counts_unmasked_pairs(causal, lens):
    wl = WORKLOADS["txl_L4096_bf16"].with_(B=4, L=23, causal=causal, seqlens_k=lens)
    assert bench.pairs_of(wl) == brute_pairs(23, 4, causal, lens)


def test_fa_convention_flops():
    wl = WORKLOADS["txl_causal_L8192_bf16"]
    f, b = bench.fa_flops(wl)
    pairs = 8192 * 8193 // 2
    assert f == 4.0 * pairs * 64 * 8 and b == 2.5 * f


@pytest.mark.parametrize("xs", [[1.0], [2.0, 1.0], [3.0, 1.0, 2.0, 5.0, 4.0], [1.5, 2.5, 0.3, 9.0, 2.0, 2.0, 7.1]])
def test_median_iqr(xs):
    m, iqr = bench.median_iqr(xs)
    assert math.isclose(m, float(np.median(xs)))
    assert math.isclose(iqr, float(np.percentile(xs, 75) - np.percentile(xs, 25)), abs_tol=1e-12)


def test_kernel_launch_counts_of_the_default_workload():
    """Transformer-XL bf16: relation prep + forward; D, relation prep, query-tile, the
    streaming launch, dr and u / v reductions; past 32 GiB of stored tiles the three
    recomputing kernels instead (non-causal 32K at H = 8 is exactly 32 GiB)."""
    assert bench.kernel_launches(WORKLOADS["txl_causal_L8192_bf16"], "auto") == (2, 6)
    assert bench.kernel_launches(WORKLOADS["txl_L32768_bf16"], "auto") == (2, 6)
    assert bench.kernel_launches(WORKLOADS["txl_L32768_bf16"].with_(H=9), "auto") == (2, 7)


def test_kernel_launch_counts_of_the_other_routes():
    """Transformer-XL memory adds the backward's LSE fill of the placeholder rows; Shaw
    with c > 64 runs the Transformer-XL kernels with the table expansion (both passes)
    and the gradient's collapse; with its value-side table and c > 64 it runs the CUDA-core
    kernels; T5 takes the tensor cores at any band width."""
    assert bench.kernel_launches(WORKLOADS["txl_mem_M4096_L4096_bf16"], "auto") == (2, 7)
    shaw = WORKLOADS["shaw_L2048_bf16"]
    assert bench.kernel_launches(shaw, "auto") == (1, 5)
    assert bench.kernel_launches(shaw.with_(shaw_clip=100), "auto") == (3, 8)
    assert bench.kernel_launches(shaw.with_(shaw_clip=100, shaw_value=True), "auto") == (1, 5)
    assert bench.kernel_launches(shaw.with_(shaw_value=True), "auto") == (1, 7)
    t5 = WORKLOADS["t5_causal_L8192_bf16"]
    assert bench.kernel_launches(t5.with_(t5_max_distance=8192, t5_num_buckets=64), "auto") == (2, 5)


def test_txl_backward_credit_splits_8U():
    """The Transformer-XL backward's algorithmic 8U, split over the kernels of each
    variant: query-tile 5U with the streaming launch (3U) or the recomputing key-tile and
    diagonal kernels (2U + 1U)."""
    c = bench.KERNEL_CREDIT_U
    T = bench.TXL
    assert c[(T, "tc_bwd_q_kernel")] + c[(T, "tc_bwd_stream_kernel")] == 8
    assert c[(T, "tc_bwd_q_kernel")] + c[(T, "tc_bwd_kv_kernel")] + c[(T, "tc_bwd_diag_kernel")] == 8


def test_kernel_table_shares():
    k = {"a": [1.0, 1.0], "b": [0.25, 0.25, 0.25, 0.25]}
    t = bench.kernel_table(k, 2, 2.0)
    assert list(t) == ["a", "b"]
    assert t["a"] == {"launches_per_step": 1.0, "ms_per_launch": 1.0, "share_of_step": 0.5}
    assert t["b"]["launches_per_step"] == 2.0 and math.isclose(t["b"]["share_of_step"], 0.25)


def test_pairs_of_memory_workload():
    """Queries at positions M .. M + L - 1, each over every key up to its own position."""
    wl = WORKLOADS["txl_mem_M4096_L4096_bf16"].with_(H=1, L=23, mem_len=9)
    want = sum(9 + i + 1 for i in range(23))
    assert bench.pairs_of(wl) == want
