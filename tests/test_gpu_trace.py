"""Per-kernel tracing (relpos_trace_begin / relpos_trace_end) on the GPU: every kernel a
traced call launches is bracketed by the caller's events, in launch order, on the call's
stream; calls outside the traced region and from other threads are not recorded."""
import threading

import pytest
import torch

from attention_fwd_bwd_flashattention_b200 import binding as bd
from attention_fwd_bwd_flashattention_b200.inputs import TXL, Workload, make_inputs

pytestmark = pytest.mark.gpu


def _case():
    wl = Workload("txl_trace", TXL, torch.bfloat16, True, 1, 2, 512)
    inp = make_inputs(wl, 3)
    dev = torch.device("cuda")
    P = bd.Params(mech=TXL, B=1, H=2, L=512, causal=True)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    rel = [r.to(dev) for r in inp["rel"]]
    return P, q, k, v, do, rel


def test_trace_records_every_kernel_of_a_step():
    P, q, k, v, do, rel = _case()
    o, lse = bd.forward(P, q, k, v, rel)  # untraced
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with bd.Trace(16) as t:
        e0.record()
        o, lse = bd.forward(P, q, k, v, rel)
        bd.backward(P, q, k, v, rel, o, lse, do)
        e1.record()
    bd.forward(P, q, k, v, rel)  # after the trace: not recorded
    torch.cuda.synchronize()
    ks = t.kernels()
    names = [n for n, _ in ks]
    assert names[:2] == ["tc_prep_kernel", "tc_fwd_kernel"]
    assert "tc_bwd_q_kernel" in names and names.count("tc_prep_kernel") == 2
    assert t.c.dropped == 0
    assert all(ms > 0 for _, ms in ks)
    assert sum(ms for _, ms in ks) <= e0.elapsed_time(e1) * 1.01


def test_trace_is_per_thread_and_counts_overflow():
    """Also: a call from a second host thread works through the binding, which makes the
    tensors' device current for the call (the library launches on the calling thread's
    current device and keeps no state shared between threads)."""
    P, q, k, v, do, rel = _case()
    seen = []

    def other():
        try:
            bd.forward(P, q, k, v, rel)
            seen.append(True)
        except Exception as e:  # reported by the assertion below
            seen.append(repr(e))

    with bd.Trace(1) as t:
        th = threading.Thread(target=other)
        th.start()
        th.join()
        bd.forward(P, q, k, v, rel)
    torch.cuda.synchronize()
    assert seen == [True], seen
    assert t.c.count == 1 and t.c.dropped == 1
    assert t.kernels()[0][0] == "tc_prep_kernel"


def test_trace_only_one_kernel():
    P, q, k, v, do, rel = _case()
    with bd.Trace(4, only="tc_fwd_kernel") as t:
        o, lse = bd.forward(P, q, k, v, rel)
        bd.backward(P, q, k, v, rel, o, lse, do)
        bd.forward(P, q, k, v, rel)
    torch.cuda.synchronize()
    assert [n for n, _ in t.kernels()] == ["tc_fwd_kernel", "tc_fwd_kernel"] and t.c.dropped == 0
