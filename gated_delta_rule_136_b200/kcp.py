"""Context-parallel KDA prefill across GPUs (KCP).

Kimi K3 report digest (fupanwang.com), section 基础设施: a sequence too long
for one GPU is cut into contiguous pieces, one per rank.  Every piece maps the
state affinely, S_end = M S_start + S_loc, so each rank

1. summarises its piece on its own GPU (``kda_segment_summary``): S_loc from
   zero (from S0 on rank 0) and the transition product M;
2. all-gathers the fixed-size summaries (2 x dk x dv fp32 per sequence and
   head, whatever the piece length): the one exchange step of the method;
3. folds the summaries of the ranks before it into its start state
   (``kda_state_combine``): S = S_loc(0), S = M(p) S + S_loc(p);
4. reruns its piece from that state with outputs (``kda_chunk_fwd``).

Every rank holds the same N sequences, each as its own piece, packed as a
variable-length batch with its own ``cu_seqlens``; pieces may differ in length
between ranks and may be empty.  The last rank's summary is never read (no
rank comes after it), so it skips step 1 and contributes zeros.  Returns the
rank's outputs and the state after its pieces, which on the last rank is the
final state of every sequence.

The compute steps are methods of an ``ops`` object (``DeviceOps`` by
default: the C-ABI kernels), so the collective logic is the same whatever
computes the pieces.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kda


class DeviceOps:
    """The GPU steps, through the C ABI."""

    summary_dtype = torch.float32

    def summary(self, q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0, with_M, scale, g_floor):
        return kda.segment_summary(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0=S0,
                                   with_M=with_M, scale=scale, g_floor=g_floor)

    def combine(self, summaries):
        return kda.state_combine(summaries)

    def prefill(self, q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0, gate, scale, g_floor):
        return kda.chunk_fwd(q, k, v, g, beta, S0=S0, cu_seqlens=cu_seqlens, scale=scale, gate=gate,
                             g_floor=g_floor, cu_seqlens_host=cu_seqlens_host)


def _all_gather(summ: torch.Tensor, world: int, group) -> torch.Tensor:
    """[world, *summ.shape]: every rank's summary in rank order."""
    out = torch.empty((world, *summ.shape), dtype=summ.dtype, device=summ.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, summ.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), summ.contiguous(), group=group)
    return out


def kcp_chunk_fwd(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0=None, gate=None, scale=None,
                  g_floor: float = -5.0, group=None, ops=None):
    """This rank's piece of a context-parallel prefill.

    q, k, g [T,H,dk]; v, gate [T,H,dv]; beta [T,H]: the rank's pieces of N
    sequences, packed with ``cu_seqlens`` (int32 [N+1], on the inputs' device)
    and its host copy ``cu_seqlens_host``.  ``S0`` fp32 [N,H,dk,dv], the
    sequences' initial states, is read on rank 0 only (pass the same on every
    rank, or None).  All ranks of ``group`` must call this with the same N,
    H, dk, dv.  Returns ``(o, S_end)``: outputs [T,H,dv] of the rank's tokens
    and the state after its pieces.
    """
    ops = ops if ops is not None else DeviceOps()
    if not dist.is_available() or not dist.is_initialized():
        world, rank = 1, 0
    else:
        world, rank = dist.get_world_size(group), dist.get_rank(group)
    if world == 1:
        return ops.prefill(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0, gate, scale, g_floor)

    N = len(cu_seqlens_host) - 1
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    if rank < world - 1:
        summ = ops.summary(q, k, v, g, beta, cu_seqlens, cu_seqlens_host,
                           S0 if rank == 0 else None, rank > 0, scale, g_floor)
    else:
        summ = torch.zeros((2, N, H, dk, dv), dtype=getattr(ops, "summary_dtype", torch.float32),
                           device=q.device)
    gathered = _all_gather(summ, world, group)
    if rank == 0:
        S_in = S0
    else:
        S_in = ops.combine(gathered[:rank].contiguous())
    return ops.prefill(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S_in, gate, scale, g_floor)


def split_pieces(lengths, world: int, granule: int = 64):
    """Cut each sequence length into ``world`` contiguous pieces of nearly
    equal length, rounded to ``granule`` tokens (the chunk size) except the
    last: returns per-rank lists of (start, end) token offsets within each
    sequence."""
    out = [[] for _ in range(world)]
    for L in lengths:
        L = int(L)
        base = -(-L // world)
        base = -(-base // granule) * granule
        for r in range(world):
            a = min(L, r * base)
            b = min(L, a + base) if r < world - 1 else L
            out[r].append((a, b))
    return out
