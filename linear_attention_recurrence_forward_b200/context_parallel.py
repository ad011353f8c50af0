"""KDA context parallelism: one batch of long sequences split along T over ranks.

Over a segment of tokens the recurrence is affine in the state it starts from,

    S_end = M S_start + N,   M = prod_t (I - beta_t k_t k_t^T) Diag(exp g_t)  (dk x dk),

with N the segment's final state from a zero start.  So ranks only need to exchange this
fixed-size pair, never the activations (channel post on the K3 report (t.iss.one),
infrastructure paragraph: KDA context parallelism splits long sequences across devices and
exchanges only the fixed-size recurrent state).  The steps, all on the library's kernels:

1. every rank but the last forms its segment's map: N = forward(x, S0 = 0).S_T and
   M = forward(q, k, v = 0, g, beta, S0 = I).S_T (the homogeneous recurrence from the
   identity; dv = dk).  Rank 0 knows its true start S0, so it runs its segment once for real
   and publishes (M = 0, N = its final state);
2. all ranks all-gather the maps (one collective over NCCL);
3. rank r composes its incoming state S_r = M_{r-1}(... (M_0 S + N_0) ...) + N_{r-1} with
   kda_state_compose;
4. rank r > 0 runs its segment from S_r (its outputs are then exact); the last rank's final
   state, the whole sequence's, is broadcast.

Ranks 1 .. R-2 run three segment passes and rank 0 and the last rank one each, all ranks in
parallel, plus r small compositions on rank r.  The pages' own scheme corrects
the outputs of a zero-start pass instead of re-running the segment; that needs per-chunk
quantities kept from the first pass, which this version trades for one more pass.

`ops` supplies the per-segment computations; the default is the CUDA library.  Tests pass
their own (an fp64 CPU stand-in) to check the orchestration and the exchange with gloo ranks.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import torch

from . import kda_forward_chunked, kda_state_compose

__all__ = ["CudaOps", "segment_map", "rank_first_step", "incoming_state", "rank_finish",
           "context_parallel_forward"]


class CudaOps:
    """Per-segment computations on the library's kernels (fp32 states)."""

    state_dtype = torch.float32

    def forward(self, q, k, v, g, beta, S0):
        return kda_forward_chunked(q, k, v, g, beta, S0)

    def compose(self, M, S, N):
        return kda_state_compose(M, S, N)


def segment_map(q, k, v, g, beta, ops=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(M [B,H,dk,dk], N [B,H,dk,dv]) of one segment: S_end = M S_start + N."""
    ops = ops or CudaOps()
    B, T, H, dk = q.shape
    _, N = ops.forward(q, k, v, g, beta, None)
    zero_v = torch.zeros((B, T, H, dk), dtype=v.dtype, device=v.device)
    eye = torch.eye(dk, dtype=ops.state_dtype, device=q.device).expand(B, H, dk, dk).contiguous()
    _, M = ops.forward(q, k, zero_v, g, beta, eye)
    return M, N


def rank_first_step(rank: int, world: int, q, k, v, g, beta, S0=None, ops=None):
    """Step 1 on one rank: returns (M, N, o, S_end); o and S_end are final on rank 0, else None."""
    ops = ops or CudaOps()
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    if rank == 0:
        o, S_end = ops.forward(q, k, v, g, beta, S0)
        M = torch.zeros((B, H, dk, dk), dtype=ops.state_dtype, device=q.device)
        return M, S_end, o, S_end
    if rank == world - 1:
        # nobody composes the last rank's map
        M = torch.zeros((B, H, dk, dk), dtype=ops.state_dtype, device=q.device)
        N = torch.zeros((B, H, dk, dv), dtype=ops.state_dtype, device=q.device)
        return M, N, None, None
    M, N = segment_map(q, k, v, g, beta, ops)
    return M, N, None, None


def incoming_state(Ms: Sequence[torch.Tensor], Ns: Sequence[torch.Tensor], rank: int, ops=None):
    """Step 3: the state entering segment `rank`, composed from the maps of the ranks before it.

    Rank 0 publishes (0, its final state), so the composition needs no S0 here.
    """
    ops = ops or CudaOps()
    S = torch.zeros_like(Ns[0])
    for j in range(rank):
        S = ops.compose(Ms[j], S, Ns[j])
    return S


def rank_finish(S_in, q, k, v, g, beta, ops=None):
    """Step 4 on rank > 0: the segment from its true start; returns (o, S_end)."""
    ops = ops or CudaOps()
    return ops.forward(q, k, v, g, beta, S_in)


def context_parallel_forward(q, k, v, g, beta, S0=None, *, group=None, ops=None):
    """This rank's contiguous segment of the batch's sequences (same B, H on every rank; segment
    lengths may differ).  Returns (o of this segment, the whole sequence's final state), the
    latter on every rank.  Collective: every rank of `group` must call it."""
    import torch.distributed as dist

    ops = ops or CudaOps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    M, N, o, S_end = rank_first_step(rank, world, q, k, v, g, beta, S0, ops)
    Ms = [torch.empty_like(M) for _ in range(world)]
    Ns = [torch.empty_like(N) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    if rank > 0:
        S_in = incoming_state(Ms, Ns, rank, ops)
        o, S_end = rank_finish(S_in, q, k, v, g, beta, ops)
    final = S_end.contiguous() if rank == world - 1 else torch.empty_like(N)
    src = world - 1 if group is None else dist.get_global_rank(group, world - 1)
    dist.broadcast(final, src=src, group=group)
    return o, final
