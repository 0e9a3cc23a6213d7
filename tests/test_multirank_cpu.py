"""The benchmark's multi-rank path on CPU (gloo, world size 2): every rank
draws its own batch of independent sequences (weak scaling, no collective on
the data path), the step time is the slowest rank's, and the whole-job value
is all ranks' tokens over that time. Each rank also runs the oracle on its own
units, which needs nothing from the other rank."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from linear_attention_recurrence_11_b200.inputs import WORKLOADS, to_f64, workload_inputs
        w = bench.rank_workload(WORKLOADS["small_f32_T256_d32"], rank)
        inp = workload_inputs(w, device="cpu")
        # this rank's units, computed locally
        o, ST = oracle.forward(*(to_f64(inp[x][0, :, 0]) for x in ("q", "k", "v", "g", "beta")))
        local_ms = 10.0 + 5.0 * rank  # stand-in for this rank's measured time
        ms_max = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.weak_scaling_value(w.total_tokens, 3, ms_max, world)
        digest = torch.tensor([float(np.abs(o).sum())], dtype=torch.float64)
        all_d = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        torch.distributed.all_gather(all_d, digest)
        q.put((rank, ms_max, value, [float(x) for x in all_d], float(np.abs(ST).sum())))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    (r0, m0, v0, d0, s0), (r1, m1, v1, d1, s1) = out
    assert m0 == m1 == 15.0                      # the slowest rank's time, on every rank
    assert v0 == v1 == 2 * 256 * 3 / 0.015       # all ranks' tokens / that time
    assert d0 == d1 and d0[0] != d0[1]           # the ranks ran different batches
    assert np.isfinite(s0) and np.isfinite(s1)
