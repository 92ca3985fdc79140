"""Context parallelism: one long sequence split across ranks (one process per GPU).

The KDA step is linear in the state, so a run of tokens maps any entry state S
to M S + B (M: dk x dk, B: dk x dv).  Rank r holds the r-th consecutive piece
of the same sequences.  Then:

1. local:    (M_r, B_r) of its piece             -- ``chunk_fwd_segmap``
2. exchange: all-gather of every rank's (M, B)   -- one collective (NCCL over
             NVLink on GPUs; 2 x 64 KiB per (sequence, head) at d = 128)
3. local:    entry state X_r = M_{r-1}(...(M_0 h0 + B_0)...) + B_{r-1}
                                                 -- ``affine_prefix``
4. local:    out_r, S_r = chunk_fwd(piece r, h0 = X_r)

and the last rank's S_r is the final state of the whole sequence.  The pages
run the method at contexts of about a million tokens ("Kimi Linear acaba de
superar a la atencion completa en sus propios terminos", sections on decode
timing and the open release); the split is derived from the linearity of the
step.  Every rank must pass the same h0 (or None).

The per-rank compute goes through ``ops`` (default: the CUDA library); the
exchange is the only collective.
"""
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def token_range(T: int, world: int, rank: int, align: int = 64) -> Tuple[int, int]:
    """Consecutive split of T tokens into `world` pieces whose boundaries fall
    on multiples of `align` (so every piece but the last is whole chunks):
    rank gets [start, stop)."""
    if world < 1 or not 0 <= rank < world or align < 1:
        raise ValueError("bad world/rank/align")
    units = (T + align - 1) // align
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(u0 * align, T), min(u1 * align, T)


class CudaOps:
    """The per-rank compute on this process's GPU (the library's C ABI)."""

    def segmap(self, q, k, v, log_alpha, beta):
        from . import chunk_fwd_segmap
        return chunk_fwd_segmap(q, k, v, log_alpha, beta)

    def prefix(self, maps, offs, h0):
        from . import affine_prefix
        return affine_prefix(maps, offs, h0)

    def forward(self, q, k, v, log_alpha, beta, scale, h0):
        from . import chunk_fwd
        return chunk_fwd(q, k, v, log_alpha, beta, scale, h0=h0)


def chunk_fwd_context_parallel(q, k, v, log_alpha, beta, scale, h0=None, group=None,
                               ops: Optional[object] = None):
    """Prefill of this rank's piece [B, T_r, H, .] of B sequences whose pieces
    are held by the ranks of `group` in rank order.  Returns (out_r, S_r):
    this piece's outputs and the state at its end (the final state of the
    whole sequences on the last rank)."""
    ops = ops if ops is not None else CudaOps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    maps, offs = ops.segmap(q, k, v, log_alpha, beta)
    # one all-gather of [M | B] per rank
    flat = torch.cat([maps.reshape(-1), offs.reshape(-1)])
    bufs = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(bufs, flat, group=group)
    nm = maps.numel()
    if rank == 0:
        start = h0
    else:
        ms = torch.stack([b[:nm].view_as(maps) for b in bufs[:rank]])
        bs = torch.stack([b[nm:].view_as(offs) for b in bufs[:rank]])
        start = ops.prefix(ms, bs, h0)
    return ops.forward(q, k, v, log_alpha, beta, scale, start)
