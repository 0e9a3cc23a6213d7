"""Context parallelism on CPU (gloo, world size 2 and 3): each rank holds a
contiguous segment of every sequence, computes its segment's KCP pair, the
pairs are all-gathered, every rank scans them and replays its segment from its
incoming state. The compute steps are stood in for by the fp64 oracle (this
test checks the placement, the collective and the scan order, on the host);
the result must equal the oracle's single pass over the whole sequences."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """segment_pair / scan / forward of the context-parallel step on the fp64 oracle,
    one (sequence, head) unit at a time, in the layouts the module passes around."""

    def __init__(self, oracle, chunk):
        self.oracle, self.chunk = oracle, chunk

    def segment_pair(self, q, k, v, g, beta):
        B, T, H, dk = k.shape
        dv = v.shape[-1]
        M = torch.zeros(B, H, dk, dk, dtype=torch.float64)
        Z = torch.zeros(B, H, dv, dk, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                m, z = self.oracle.segment_pair(*(x[b, :, h].numpy() for x in (q, k, v, g, beta)), C=self.chunk)
                M[b, h], Z[b, h] = torch.from_numpy(m), torch.from_numpy(z)
        return M, Z

    def scan(self, S0, M, Z):
        B, P, H = M.shape[:3]
        dv, dk = Z.shape[3], Z.shape[4]
        S_in = torch.zeros(B, P, H, dv, dk, dtype=torch.float64)
        S_T = torch.zeros(B, H, dv, dk, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                s0 = None if S0 is None else S0[b, h].numpy()
                out = self.oracle.kcp_scan(M[b, :, h].numpy(), Z[b, :, h].numpy(), s0)
                S_in[b, :, h] = torch.from_numpy(out[:P])
                S_T[b, h] = torch.from_numpy(out[P])
        return S_in, S_T

    def forward(self, q, k, v, g, beta, S0):
        B, T, H, _ = k.shape
        dv = v.shape[-1]
        o = torch.zeros(B, T, H, dv, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                ou, _ = self.oracle.forward(*(x[b, :, h].numpy() for x in (q, k, v, g, beta)), S0=S0[b, h].numpy())
                o[b, :, h] = torch.from_numpy(ou)
        return o


def _worker(rank, world, port, seg, q_out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        _run(rank, world, seg, q_out)
    except Exception as e:  # report instead of dying silently
        import traceback
        q_out.put((rank, "error", traceback.format_exc()))
    finally:
        torch.distributed.destroy_process_group()


def _run(rank, world, seg, q_out):
    if True:
        import oracle
        from linear_attention_recurrence_11_b200.context_parallel import context_parallel_forward
        from linear_attention_recurrence_11_b200.inputs import make_inputs, to_f64
        oracle.build()
        B, H, dk, dv, chunk = 2, 2, 32, 32, 16
        T = seg * world - 5  # the last rank's segment is ragged
        inp = make_inputs(B, T, H, dk, dv, "f32", seed=77, device="cpu", s0_std=0.1)
        full = {x: torch.from_numpy(to_f64(inp[x])) for x in ("q", "k", "v", "g", "beta")}
        S0 = torch.from_numpy(to_f64(inp["S0"]))
        t0, t1 = rank * seg, min(T, (rank + 1) * seg)
        mine = {x: full[x][:, t0:t1].contiguous() for x in full}
        o, S_T = context_parallel_forward(mine["q"], mine["k"], mine["v"], mine["g"], mine["beta"], S0,
                                          ops=OracleOps(oracle, chunk))
        # the oracle's single pass over the whole sequences
        err_o, err_s = 0.0, 0.0
        for b in range(B):
            for h in range(H):
                ou, su = oracle.forward(*(full[x][b, :, h].numpy() for x in ("q", "k", "v", "g", "beta")),
                                        S0=S0[b, h].numpy())
                err_o = max(err_o, float(np.abs(o[b, :, h].numpy() - ou[t0:t1]).max()))
                err_s = max(err_s, float(np.abs(S_T[b, h].numpy() - su).max()))
        q_out.put((rank, err_o, err_s))


@pytest.mark.parametrize("world,seg", [(2, 48), (3, 32)])
def test_context_parallel_gloo(world, seg):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seg, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err_o, err_s in out:
        assert err_o != "error", err_s
        # fp64 throughout: the composed form equals the single pass to rounding
        assert err_o < 1e-12 and err_s < 1e-12, (rank, err_o, err_s)
