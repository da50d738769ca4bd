"""One sequence split across ranks: the prefill of each rank's stretch, with the
entry states passed on through the affine chunk maps.

"KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解" (Figure 1, Figure 3):
the prefill maps its entry state affinely, final = M S0 + B.  Rank r holds
tokens [a_r, a_{r+1}) of one sequence (ranks in sequence order, every stretch
non-empty).  Each rank computes its stretch's (M_r, B_r) on its own device,
the maps are all-gathered (the one exchange of the path, 192 KiB per head and
rank), each rank composes its entry state E_r = M_{r-1}(... (M_0 S0 + B_0) ...)
+ B_{r-1} locally, runs its stretch from E_r, and the last rank's final state
is broadcast.  The arithmetic runs in the library's kernels (kda_chunk_map_ws,
kda_state_compose, kda_chunk_fwd); this module only orders the calls and the
collectives.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The library's kernels for the three steps (the product path)."""

    def __init__(self, workspace="auto"):
        from . import kda_chunk_fwd, kda_chunk_map, kda_state_compose
        self._fwd, self._map, self._compose = kda_chunk_fwd, kda_chunk_map, kda_state_compose
        self._ws = workspace

    def map(self, q, k, v, g, beta):
        return self._map(q, k, v, g, beta)

    def compose(self, M, B, E):
        return self._compose(M, B, E)

    def fwd(self, q, k, v, g, beta, o, scale, initial_state, final_state):
        self._fwd(q, k, v, g, beta, o, scale=scale, initial_state=initial_state,
                  final_state=final_state, workspace=self._ws)


def kda_chunk_fwd_sequence_parallel(q, k, v, g, beta, o, *, scale: float = 1.0,
                                    initial_state=None, final_state=None, group=None, ops=None):
    """Prefill of this rank's stretch of one sequence split across the ranks of
    ``group`` (the default group when None; a single process when
    torch.distributed is not initialised).  q, k, v, g, beta, o: this rank's
    tokens [T_r, H, D]; ``initial_state`` [1, H, D, D] the sequence's initial
    state (the same on every rank, or None).  Writes o for the stretch and
    returns the sequence's final state [1, H, D, D] on every rank (also copied
    into ``final_state`` when given).  Every rank makes the same collective
    calls in the same order: two all-gathers and one broadcast."""
    ops = LibraryOps() if ops is None else ops
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    M, B = ops.map(q, k, v, g, beta)
    if world > 1:
        Ms = [torch.empty_like(M) for _ in range(world)]
        Bs = [torch.empty_like(B) for _ in range(world)]
        dist.all_gather(Ms, M.contiguous(), group=group)
        dist.all_gather(Bs, B.contiguous(), group=group)
    else:
        Ms, Bs = [M], [B]
    E = initial_state
    for i in range(rank):
        E = ops.compose(Ms[i], Bs[i], E)
    fs = torch.empty_like(B)
    ops.fwd(q, k, v, g, beta, o, scale, E, fs)
    if world > 1:
        last = world - 1 if group is None else dist.get_global_rank(group, world - 1)
        dist.broadcast(fs, src=last, group=group)
    if final_state is not None:
        final_state.copy_(fs)
    return fs
