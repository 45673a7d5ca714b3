"""The multi-rank split on CPU with two gloo ranks.

Plumbing: the relative-table gradients summed across ranks and the step time reduced
with MAX.  Decomposition: every rank runs the fp64 oracle on its shard of a workload
(its batch entries, or its block of heads with the matching table rows), the shards'
outputs are gathered and, for the batch split, the table gradients all-reduced; the
result must equal one oracle call on the whole workload.  Each (batch, head) slice is
computed on its own in both passes, so O, LSE, dQ, dK and dV agree bit for bit, and so
do the table gradients of the head split; the batch split's table gradients are the
sum of two per-batch partials, bit for bit too where the oracle forms each partial
before adding it (Shaw, Transformer-XL, DeBERTa), to 1e-12 where it scatter-adds the
pairs straight into the table (T5).
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

MECHS = ("txl", "shaw", "deberta", "t5")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _run(target, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))


def _plumbing(rank, world, port, q):
    _env(rank, world, port)
    from attention_fwd_bwd_flashattention_b200 import dist as rdist

    r, w, _ = rdist.init_from_env(backend="gloo", timeout_s=60)
    g = [torch.full((3, 4), float(r + 1)), torch.arange(5, dtype=torch.float32) * (r + 1)]
    rdist.allreduce_table_grads(g)
    t = rdist.max_over_ranks(10.0 + r)
    rdist.barrier()
    q.put((r, w, g[0].sum().item(), g[1].tolist(), t))
    rdist.shutdown()


def test_two_gloo_ranks():
    for r, w, s0, s1, t in _run(_plumbing):
        assert w == 2
        assert s0 == 12 * 3.0          # (1 + 2) summed over a 3x4 tensor
        assert s1 == [0.0, 3.0, 6.0, 9.0, 12.0]
        assert t == 11.0               # max over ranks


def _decompose(rank, world, port, q):
    _env(rank, world, port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as orc
    from attention_fwd_bwd_flashattention_b200 import dist as rdist
    from attention_fwd_bwd_flashattention_b200.inputs import MECH_IDS, Workload, make_inputs

    rdist.init_from_env(backend="gloo", timeout_s=120)
    report = []
    for name in MECHS:
        mech = MECH_IDS[name]
        for mode, B, H in (("batch", 2, 2), ("heads", 1, 4)):
            wl = Workload(f"{name}_{mode}", mech, torch.float32, name == "txl", B, H, 40, shaw_clip=5, deberta_span=8,
                          t5_num_buckets=8, t5_max_distance=20, rel_std=0.5)
            full = make_inputs(wl, seed=3)
            part = rdist.shard_inputs(full, mode, rank, world)
            cfg = orc.RelCfg(shaw_clip=5, deberta_span=8, t5_num_buckets=8, t5_max_distance=20)
            f64 = lambda t: t.double().numpy()  # noqa: E731
            args = [f64(part[n]) for n in ("q", "k", "v")], [f64(r) for r in part["rel"]]
            O, LSE = orc.forward(mech, *args[0], args[1], wl.causal, wl.scale, cfg)
            dq, dk, dv, drel = orc.backward(mech, *args[0], args[1], wl.causal, f64(part["do"]), wl.scale, cfg)
            dim = 0 if mode == "batch" else 1
            got = [rdist.gather_shards(torch.from_numpy(np.ascontiguousarray(x)), dim) for x in (O, LSE, dq, dk, dv)]
            gd = [torch.from_numpy(np.ascontiguousarray(g)) for g in drel]
            if mode == "batch":
                rdist.allreduce_table_grads(gd)
            else:
                gd = [rdist.gather_shards(g, 0) for g in gd]
            if rank == 0:
                fa = [f64(full[n]) for n in ("q", "k", "v")], [f64(r) for r in full["rel"]]
                O1, L1 = orc.forward(mech, *fa[0], fa[1], wl.causal, wl.scale, cfg)
                g1 = orc.backward(mech, *fa[0], fa[1], wl.causal, f64(full["do"]), wl.scale, cfg)
                want = [O1, L1, *g1[:3]]
                outs_equal = all(np.array_equal(a.numpy(), b) for a, b in zip(got, want))
                tab_err = max(float(np.max(np.abs(a.numpy() - b)) / max(np.max(np.abs(b)), 1e-300))
                              for a, b in zip(gd, g1[3]))
                tab_equal = all(np.array_equal(a.numpy(), b) for a, b in zip(gd, g1[3]))
                report.append((name, mode, outs_equal, tab_equal, tab_err))
    q.put((rank, report))
    rdist.shutdown()


def test_shards_reassemble_one_oracle_call_bit_for_bit():
    res = _run(_decompose)
    report = res[0][1]
    assert len(report) == 2 * len(MECHS)
    for name, mode, outs_equal, tab_equal, tab_err in report:
        assert outs_equal, (name, mode)
        if name == "t5" and mode == "batch":
            assert tab_err < 1e-12, (name, mode, tab_err)
        else:
            assert tab_equal, (name, mode, tab_err)


def test_shard_range_covers_everything_once():
    from attention_fwd_bwd_flashattention_b200 import dist as rdist

    for n in (1, 2, 7, 8, 12):
        for world in (1, 2, 3, 8):
            blocks = [rdist.shard_range(n, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(blocks, blocks[1:]))
            assert max(h - lo for lo, h in blocks) - min(h - lo for lo, h in blocks) <= 1


def test_single_process_is_a_no_op():
    from attention_fwd_bwd_flashattention_b200 import dist as rdist

    g = [torch.ones(2)]
    rdist.allreduce_table_grads(g)
    assert g[0].tolist() == [1.0, 1.0]
    assert rdist.max_over_ranks(3.5) == 3.5
    assert rdist.gather_shards(g[0], 0) is g[0]
