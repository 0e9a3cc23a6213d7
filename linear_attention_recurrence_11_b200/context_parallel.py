"""Context parallelism for long sequences: the tokens of each sequence are split
into contiguous segments, one per rank (one process per GPU), after the 4-rank
scan of the Kimi K3 pages' check script ("Exercices", Q21-Q22: a segment maps an
incoming state S to M S + S~ and pairs compose).

Per rank: (1) the KCP pair (M, S~) of its segment, from its own tokens only;
(2) an all-gather of the pairs (2 x 64 KiB per head at d = 128, the only
exchange); (3) the scan over the gathered pairs, identical on every rank, gives
the rank's incoming state and the final state S_T; (4) the prefill of its
segment from that incoming state writes its outputs. Steps 1, 3 and 4 run in
libkda.so (kda_segment_pair, kda_kcp_scan, kda_forward); the module holds only
the placement and the collective.
"""
import torch
import torch.distributed as dist


class GpuOps:
    """The compute steps, in libkda.so."""

    def __init__(self, chunk: int = 64, path: str = "auto"):
        self.chunk, self.path = chunk, path

    def segment_pair(self, q, k, v, g, beta):
        from . import kda
        return kda.kda_segment_pair(q, k, v, g, beta, chunk=self.chunk, path=self.path)

    def scan(self, S0, M, Z):
        from . import kda
        return kda.kda_kcp_scan(S0, M, Z)

    def forward(self, q, k, v, g, beta, S0):
        from . import kda
        o, _ = kda.kda_forward(q, k, v, g, beta, S0, chunk=self.chunk, return_state=False, path=self.path)
        return o


def context_parallel_forward(q, k, v, g, beta, S0=None, *, group=None, ops=None):
    """This rank's segment of B sequences: q, k, g ``[B, T_r, H, dk]``, v
    ``[B, T_r, H, dv]``, beta ``[B, T_r, H]``, where rank r holds tokens
    r T_r .. (r + 1) T_r - 1 of every sequence (equal segments; T_r a multiple of
    the chunk except possibly on the last rank). S0 ``[B, H, dv, dk]`` (the
    incoming states of the whole sequences; the same on every rank) or None.
    Returns (o of this segment ``[B, T_r, H, dv]``, S_T ``[B, H, dv, dk]``, the
    final states of the whole sequences, on every rank)."""
    ops = ops if ops is not None else GpuOps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    M, Z = ops.segment_pair(q, k, v, g, beta)              # [B, H, dk, dk], [B, H, dv, dk]
    # gathered along the first dimension (the form every backend accepts), then viewed per rank
    M_all = torch.empty((world * M.shape[0],) + tuple(M.shape[1:]), dtype=M.dtype, device=M.device)
    Z_all = torch.empty((world * Z.shape[0],) + tuple(Z.shape[1:]), dtype=Z.dtype, device=Z.device)
    dist.all_gather_into_tensor(M_all, M.contiguous(), group=group)
    dist.all_gather_into_tensor(Z_all, Z.contiguous(), group=group)
    M_all = M_all.view((world,) + tuple(M.shape))
    Z_all = Z_all.view((world,) + tuple(Z.shape))
    # [P, B, H, ...] -> [B, P, H, ...]: segment p of every sequence is rank p's
    S_in, S_T = ops.scan(S0, M_all.transpose(0, 1).contiguous(), Z_all.transpose(0, 1).contiguous())
    o = ops.forward(q, k, v, g, beta, S_in[:, rank].contiguous())
    return o, S_T
