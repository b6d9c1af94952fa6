"""The rows s of one attention problem split over the ranks of a process group.

The rows are independent problems that share one additive pair bias,
broadcast over them (MegaFold summary, section "EvoFlash-3D"), so a
sequence-parallel group that partitions the pair tensor (same page, section
"EvoSP-3D") can give each rank a contiguous block of rows:

* forward: each rank runs evo_attn_fwd on its own rows, with no
  communication;
* backward: dq, dk, dv and dg of a row stay with its rank, and d_pair_bias --
  the sum over every row -- is the one exchange.  Each rank's evo_attn_bwd
  returns the sum over its own rows; the ranks all-gather these partials
  (NCCL over NVLink on GPUs) and each adds them in rank order with
  evo_sum_partials, so that every rank holds the same bits.

The all-gather moves (world - 1) partials of B*H*N*N fp32 into every rank,
where a reduce would move fewer bytes; it is chosen because the sum is then
taken in one fixed order, independent of the collective's algorithm.
Ranks whose block is empty (S smaller than the group) contribute zeros.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import attention as A


def row_range(S: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [s0, s1) that rank ``rank`` of ``world`` holds.

    Contiguous blocks in rank order whose sizes differ by at most one, the
    larger blocks first; together they cover [0, S) once.
    """
    if S < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"no row block for S={S}, world={world}, rank={rank}")
    base, extra = divmod(S, world)
    s0 = rank * base + min(rank, extra)
    return s0, s0 + base + (1 if rank < extra else 0)


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather one partial per rank: a [world, *partial.shape] tensor, rank r's at index r.

    Every rank takes part, in the same order as the others' calls.
    """
    world = _world(group)
    flat = partial.contiguous().reshape(-1)
    buf = torch.empty(world * flat.numel(), dtype=partial.dtype, device=partial.device)
    dist.all_gather_into_tensor(buf, flat, group=group)
    return buf.view(world, *partial.shape)


def attn_fwd(q, k, v, g, mask_bias=None, pair_bias=None, out=None, lse=None):
    """Forward of this rank's rows: evo_attn_fwd on them, no communication.

    q, k, v, g (and mask_bias, if any) hold this rank's rows only; pair_bias
    is the full bias every rank shares.
    """
    return A.evo_attn_fwd(q, k, v, g, mask_bias, pair_bias, out, lse)


def attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, group=None, grads=None, workspace=None):
    """Backward of this rank's rows, with d_pair_bias summed over every rank's rows.

    Arguments as for evo_attn_bwd, restricted to this rank's rows (pair_bias
    in full).  Returns its dict of gradients, in which d_pair_bias is the sum
    over all ranks, added in rank order.  Every rank of ``group`` must call it
    (a collective).  With one rank, no collective runs.
    """
    grads = A.evo_attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, grads, workspace)
    if _world(group) > 1:
        parts = gather_partials(grads["d_pair_bias"], group)
        A.sum_partials(parts, out=grads["d_pair_bias"])
    return grads
