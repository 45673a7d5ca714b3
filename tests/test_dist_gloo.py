"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, the relative-table
gradients summed across ranks and the step time reduced with MAX."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from attention_fwd_bwd_flashattention_b200 import dist as rdist

    r, w, _ = rdist.init_from_env(backend="gloo", timeout_s=60)
    g = [torch.full((3, 4), float(r + 1)), torch.arange(5, dtype=torch.float32) * (r + 1)]
    rdist.allreduce_table_grads(g)
    t = rdist.max_over_ranks(10.0 + r)
    rdist.barrier()
    q.put((r, w, g[0].sum().item(), g[1].tolist(), t))
    rdist.shutdown()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, s0, s1, t in res:
        assert w == 2
        assert s0 == 12 * 3.0          # (1 + 2) summed over a 3x4 tensor
        assert s1 == [0.0, 3.0, 6.0, 9.0, 12.0]
        assert t == 11.0               # max over ranks


def test_single_process_is_a_no_op():
    from attention_fwd_bwd_flashattention_b200 import dist as rdist

    g = [torch.ones(2)]
    rdist.allreduce_table_grads(g)
    assert g[0].tolist() == [1.0, 1.0]
    assert rdist.max_over_ranks(3.5) == 3.5
