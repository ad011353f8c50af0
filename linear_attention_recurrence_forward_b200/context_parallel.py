"""KDA context parallelism: one batch of long sequences split along T over ranks.

Over a segment of tokens the recurrence is affine in the state it starts from.  With
Phi_t = prod_{u<=t} (I - beta_u k_u k_u^T) Diag(exp g_u) (dk x dk),

    S_t = Phi_t S_start + S_t^0,      o_t = o_t^0 + S_start^T (Phi_t^T q_t),

where S_t^0 and o_t^0 are the state and the outputs from a zero start.  At the segment's end
this is S_end = M S_start + N, with M = Phi_T and N = S_T^0.  So the ranks only need to exchange
the fixed-size pair (M, N), never the activations (channel post on the K3 report (t.iss.one),
infrastructure paragraph: KDA context parallelism splits long sequences across devices and
exchanges only the fixed-size recurrent state).

The steps, all on the library's kernels:

1. Rank 0 knows its true start S0.  It runs its segment once for real and publishes
   (M = 0, N = its final state).  Every other rank runs its segment twice, before its start
   state is known:
   - with S0 = 0, for the zero-start outputs o^0 and N;
   - with v = 0 and S0 = I (dv = dk), whose state is Phi_t.  So its outputs are the correction
     operands C_t = Phi_t^T q_t, and its final state is M.
   The two runs are independent of each other and of the other ranks.
2. All ranks all-gather the maps (one collective over NCCL).
3. Rank r composes its incoming state S_r = M_{r-1}(... (M_0 S + N_0) ...) + N_{r-1} with
   kda_state_compose.
4. Rank r > 0 corrects its outputs with kda_output_correct, o_t = o^0_t + S_r^T C_t, a light
   tensor-core pass.  Its final state is M S_r + N.  The last rank's final state, the whole
   sequence's, is broadcast.

Work per rank: rank 0 runs one pass over its segment.  Every other rank runs two passes, one
correction and r compositions of 128 x 128 maps.

`ops` supplies the per-segment computations; the default is the CUDA library.  Tests pass
their own (an fp64 CPU stand-in) to check the orchestration and the exchange with gloo ranks.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import torch

from . import kda_forward_chunked, kda_output_correct, kda_state_compose

__all__ = ["CudaOps", "segment_pass", "segment_map", "rank_first_step", "incoming_state", "rank_finish",
           "context_parallel_forward"]


class CudaOps:
    """Per-segment computations on the library's kernels (fp32 states)."""

    state_dtype = torch.float32

    def forward(self, q, k, v, g, beta, S0):
        return kda_forward_chunked(q, k, v, g, beta, S0)

    def compose(self, M, S, N):
        return kda_state_compose(M, S, N)

    def correct(self, C, S, o0):
        return kda_output_correct(C, S, o0)


def segment_pass(q, k, v, g, beta, ops=None):
    """The two zero-start runs of one segment: (o0, N, C, M).

    o0 [B,T,H,dv] and N [B,H,dk,dv] from S0 = 0.  C [B,T,H,dk] (C_t = Phi_t^T q_t) and
    M [B,H,dk,dk] from v = 0 and S0 = I.
    """
    ops = ops or CudaOps()
    B, T, H, dk = q.shape
    o0, N = ops.forward(q, k, v, g, beta, None)
    zero_v = torch.zeros((B, T, H, dk), dtype=v.dtype, device=v.device)
    eye = torch.eye(dk, dtype=ops.state_dtype, device=q.device).expand(B, H, dk, dk).contiguous()
    C, M = ops.forward(q, k, zero_v, g, beta, eye)
    return o0, N, C, M


def segment_map(q, k, v, g, beta, ops=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(M [B,H,dk,dk], N [B,H,dk,dv]) of one segment: S_end = M S_start + N."""
    _, N, _, M = segment_pass(q, k, v, g, beta, ops)
    return M, N


def rank_first_step(rank: int, world: int, q, k, v, g, beta, S0=None, ops=None):
    """Step 1 on one rank.

    Returns (M, N, o, S_end, C).  On rank 0, o and S_end are final and C is None.  On the other
    ranks, o is the zero-start output, S_end is None and C is the correction operand.
    """
    ops = ops or CudaOps()
    B, _, H, dk = q.shape
    if rank == 0:
        o, S_end = ops.forward(q, k, v, g, beta, S0)
        M = torch.zeros((B, H, dk, dk), dtype=ops.state_dtype, device=q.device)
        return M, S_end, o, S_end, None
    o0, N, C, M = segment_pass(q, k, v, g, beta, ops)
    return M, N, o0, None, C


def incoming_state(Ms: Sequence[torch.Tensor], Ns: Sequence[torch.Tensor], rank: int, ops=None):
    """Step 3: the state entering segment `rank`, composed from the maps of the ranks before it.

    Rank 0 publishes (0, its final state), so the composition needs no S0 here.
    """
    ops = ops or CudaOps()
    S = torch.zeros_like(Ns[0])
    for j in range(rank):
        S = ops.compose(Ms[j], S, Ns[j])
    return S


def rank_finish(S_in, o0, C, M, N, ops=None):
    """Step 4 on rank > 0: the corrected outputs and the segment's final state (o, S_end)."""
    ops = ops or CudaOps()
    return ops.correct(C, S_in, o0), ops.compose(M, S_in, N)


def context_parallel_forward(q, k, v, g, beta, S0=None, *, group=None, ops=None):
    """This rank's contiguous segment of the batch's sequences (same B, H on every rank; segment
    lengths may differ).  Returns (o of this segment, the whole sequence's final state), the
    latter on every rank.  Collective: every rank of `group` must call it."""
    import torch.distributed as dist

    ops = ops or CudaOps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    M, N, o, S_end, C = rank_first_step(rank, world, q, k, v, g, beta, S0, ops)
    Ms = [torch.empty_like(M) for _ in range(world)]
    Ns = [torch.empty_like(N) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    if rank > 0:
        S_in = incoming_state(Ms, Ns, rank, ops)
        o, S_end = rank_finish(S_in, o, C, M, N, ops)
    final = S_end.contiguous() if rank == world - 1 else torch.empty_like(N)
    src = world - 1 if group is None else dist.get_global_rank(group, world - 1)
    dist.broadcast(final, src=src, group=group)
    return o, final
