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


def start_gather(partial: torch.Tensor, group=None):
    """Start the all-gather of one partial per rank; returns (parts, work).

    ``parts`` is a [world, *partial.shape] view of the gathered buffer, rank
    r's partial at index r, valid once ``work.wait()`` has returned (with
    NCCL: once the caller's current stream has been made to wait).  Until
    then ``partial`` is being read and must not change.  Every rank takes
    part, in the same order as the others' calls.
    """
    world = _world(group)
    flat = partial.contiguous().reshape(-1)
    buf = torch.empty(world * flat.numel(), dtype=partial.dtype, device=partial.device)
    work = dist.all_gather_into_tensor(buf, flat, group=group, async_op=True)
    return buf.view(world, *partial.shape), work


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather one partial per rank: a [world, *partial.shape] tensor, rank r's at index r."""
    parts, work = start_gather(partial, group)
    work.wait()
    return parts


class PendingPairBiasGrad:
    """The d_pair_bias exchange of one row-split backward, started but not finished.

    wait() waits for the all-gather and adds the gathered partials, in rank
    order, into the tensor that held this rank's partial; it returns that
    tensor.  Between attn_bwd(..., async_op=True) and wait() the caller can
    enqueue work that needs only dq, dk, dv, dg (their projections'
    backward, say), which then overlaps the transfer.
    """

    def __init__(self, parts=None, work=None, out=None, summer=None):
        self._parts, self._work, self._out = parts, work, out
        self._sum = summer or A.sum_partials

    def wait(self) -> torch.Tensor:
        if self._work is not None:
            self._work.wait()
            self._sum(self._parts, out=self._out)
            self._work = self._parts = None
        return self._out


def attn_fwd(q, k, v, g, mask_bias=None, pair_bias=None, out=None, lse=None, out_lo=None):
    """Forward of this rank's rows: evo_attn_fwd on them, no communication.

    q, k, v, g (and mask_bias, if any) hold this rank's rows only; pair_bias
    is the full bias every rank shares.  out_lo as for evo_attn_fwd.
    """
    return A.evo_attn_fwd(q, k, v, g, mask_bias, pair_bias, out, lse, out_lo)


def attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, group=None, grads=None, workspace=None,
             async_op: bool = False, backward=None, summer=None, out_lo=None):
    """Backward of this rank's rows, with d_pair_bias summed over every rank's rows.

    Arguments as for evo_attn_bwd, restricted to this rank's rows (pair_bias
    in full).  Returns its dict of gradients, in which d_pair_bias is the sum
    over all ranks, added in rank order.  Every rank of ``group`` must call it
    (a collective).  With one rank, no collective runs.  With
    ``async_op=True`` it returns (grads, pending) instead: grads["d_pair_bias"]
    holds this rank's partial until pending.wait() turns it into the sum.

    ``backward`` and ``summer`` replace the library's evo_attn_bwd and
    sum_partials (same signatures); they exist so that the exchange can be
    exercised on CPU ranks with another implementation of the two.
    """
    world = _world(group)
    if world > A.MAX_PARTIALS:
        # refused before any kernel or collective runs, on every rank alike
        raise ValueError(f"a row split over {world} ranks exceeds the {A.MAX_PARTIALS} partials "
                         "evo_sum_partials adds in one call")
    if out_lo is None:
        grads = (backward or A.evo_attn_bwd)(q, k, v, g, mask_bias, pair_bias, out, lse, dout, grads, workspace)
    else:
        grads = (backward or A.evo_attn_bwd)(q, k, v, g, mask_bias, pair_bias, out, lse, dout, grads, workspace,
                                             out_lo=out_lo)
    pending = PendingPairBiasGrad(out=grads["d_pair_bias"])
    if world > 1:
        parts, work = start_gather(grads["d_pair_bias"], group)
        pending = PendingPairBiasGrad(parts, work, grads["d_pair_bias"], summer)
    if async_op:
        return grads, pending
    pending.wait()
    return grads
