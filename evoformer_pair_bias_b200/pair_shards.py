"""The pair representation sharded by rows over a process group, with the
triangle attentions around both nodes.

MegaFold's EvoSP-3D (MegaFold summary, section "EvoSP-3D : Partitionnement
(Sharding) Économe en Communication") splits the N x N pair tensor over a
sequence-parallel group and rotates the shard axis with all_to_all between
the row-oriented and the column-oriented operations.  Here every rank holds a
contiguous block of pair rows i (``row_range``), with every column j:

* triangle attention around the starting node attends along each pair row
  (rows s = i, keys j), so a row shard is already a set of whole problems;
  it runs on the shard in place;
* triangle attention around the ending node attends along each pair column
  (rows s = j, keys i), so its inputs are first rotated to column shards
  (``rows_to_cols``: one all_to_all), the attention runs on the transposed
  view of the column block (the strided call of the transposed pair), and
  the outputs are rotated back (``cols_to_rows``);
* the pair bias [B, 1, H, N, N] is one term shared by every row s; each rank
  projects the bias of its own pair rows and the shards are all-gathered
  (``gather_bias_rows``);
* in the backward, dq, dk, dv, dg stay (or are rotated back) with their
  rows, and d_pair_bias -- the sum over all rows s -- is the row split's
  exchange: each rank's partial is all-gathered and added in rank order
  (``row_shards``), so every rank holds the same bits.

Every collective here is a plain NCCL (or, in the tests, gloo) call issued by
every rank in the same order; no kernel reads another GPU's memory.  The
attention itself is the library's (evo_attn_fwd / evo_attn_bwd); ``fwd`` /
``bwd`` arguments replace it (same signatures), which is how the CPU tests run
the exchange with the oracle standing in.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import attention as A
from . import row_shards

row_range = row_shards.row_range


def _world_rank(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def _ranges(n: int, world: int):
    return [row_range(n, world, r) for r in range(world)]


def rows_to_cols(x: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """Row shard -> column shard of an n x n pair tensor, by one all_to_all.

    ``x`` is this rank's rows [B, i1 - i0, n, *rest] (every column); returns
    this rank's columns [B, n, j1 - j0, *rest] (every row, in order), where
    (i0, i1) and (j0, j1) are both ``row_range(n, world, rank)``.
    """
    world, rank = _world_rank(group)
    if world == 1:
        return x
    rng = _ranges(n, world)
    B, rest = x.shape[0], tuple(x.shape[3:])
    if x.shape[1] != rng[rank][1] - rng[rank][0] or x.shape[2] != n:
        raise ValueError(f"expected this rank's rows [B, {rng[rank][1] - rng[rank][0]}, {n}, ...], got {tuple(x.shape)}")
    per = 1
    for d in rest:
        per *= d
    nr = x.shape[1]
    send = torch.cat([x[:, :, j0:j1].reshape(-1) for (j0, j1) in rng])
    in_splits = [B * nr * (j1 - j0) * per for (j0, j1) in rng]
    j0, j1 = rng[rank]
    nc = j1 - j0
    out_splits = [B * (i1 - i0) * nc * per for (i0, i1) in rng]
    recv = torch.empty(sum(out_splits), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    pieces, off = [], 0
    for (i0, i1), m in zip(rng, out_splits):
        pieces.append(recv[off:off + m].view(B, i1 - i0, nc, *rest))
        off += m
    return torch.cat(pieces, dim=1)


def cols_to_rows(y: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """Column shard -> row shard, the inverse of ``rows_to_cols``.

    ``y`` is this rank's columns [B, n, j1 - j0, *rest]; returns this rank's
    rows [B, i1 - i0, n, *rest].
    """
    world, rank = _world_rank(group)
    if world == 1:
        return y
    rng = _ranges(n, world)
    B, rest = y.shape[0], tuple(y.shape[3:])
    if y.shape[1] != n or y.shape[2] != rng[rank][1] - rng[rank][0]:
        raise ValueError(f"expected this rank's columns [B, {n}, {rng[rank][1] - rng[rank][0]}, ...], "
                         f"got {tuple(y.shape)}")
    per = 1
    for d in rest:
        per *= d
    nc = y.shape[2]
    send = torch.cat([y[:, i0:i1].reshape(-1) for (i0, i1) in rng])
    in_splits = [B * (i1 - i0) * nc * per for (i0, i1) in rng]
    i0, i1 = rng[rank]
    nr = i1 - i0
    out_splits = [B * nr * (j1 - j0) * per for (j0, j1) in rng]
    recv = torch.empty(sum(out_splits), dtype=y.dtype, device=y.device)
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    pieces, off = [], 0
    for (j0, j1), m in zip(rng, out_splits):
        pieces.append(recv[off:off + m].view(B, nr, j1 - j0, *rest))
        off += m
    return torch.cat(pieces, dim=2)


def gather_bias_rows(bias_rows: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """The full pair bias [B, 1, H, n, n] from every rank's query rows [B, 1, H, i1 - i0, n] (all_gather)."""
    world, rank = _world_rank(group)
    if world == 1:
        return bias_rows.contiguous()
    rng = _ranges(n, world)
    B, _, H = bias_rows.shape[:3]
    rmax = max(i1 - i0 for (i0, i1) in rng)            # blocks padded to one size for the collective
    mine = torch.zeros((B, 1, H, rmax, n), dtype=bias_rows.dtype, device=bias_rows.device)
    mine[:, :, :, :bias_rows.shape[3]] = bias_rows
    parts = [torch.empty_like(mine) for _ in rng]
    dist.all_gather(parts, mine, group=group)
    return torch.cat([p[:, :, :, :i1 - i0] for p, (i0, i1) in zip(parts, rng)], dim=3).contiguous()


def _tri_end_view(t):
    """Column block [B, n, nc, H, C] (rows i, columns j) as the transposed pair [B, nc, n, H, C] (rows s = j)."""
    return t.permute(0, 2, 1, 3, 4)


def tri_start_fwd(q, k, v, g, mask_bias, pair_bias, fwd=None):
    """Triangle attention around the starting node on this rank's pair rows (no communication).

    q, k, v, g: [B, rows, N, H, C] (this rank's pair rows i, every column j);
    mask_bias [B, rows, 1, 1, N] or None; pair_bias the full [B, 1, H, N, N].
    Returns (out, lse) of this rank's rows.
    """
    return (fwd or A.evo_attn_fwd)(q, k, v, g, mask_bias, pair_bias)


def tri_start_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, group=None, bwd=None, summer=None):
    """Backward of ``tri_start_fwd``: this rank's rows' gradients and the summed d_pair_bias."""
    return row_shards.attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, group=group, backward=bwd,
                               summer=summer)


def tri_end_fwd(q, k, v, g, mask_bias, pair_bias, n, group=None, fwd=None):
    """Triangle attention around the ending node for a row-sharded pair representation.

    q, k, v, g: this rank's pair rows [B, rows, N, H, C].  mask_bias: the
    mask over keys i of each row s = j this rank will own after the rotation,
    [B, cols, 1, 1, N], or None; pair_bias the full [B, 1, H, N, N] in the
    orientation the op reads ([b, h, query i, key i']).  The inputs go to
    column shards with one all_to_all each; the attention runs on the
    transposed view of the column block; out goes back to row shards.
    Returns (out_rows [B, rows, N, H, C], lse [B, cols, H, N] of this rank's
    columns, and the column-shard tensors the backward reuses).
    """
    cols = [rows_to_cols(t, n, group) for t in (q, k, v, g)]
    qc, kc, vc, gc = (_tri_end_view(t) for t in cols)
    res = (fwd or A.evo_attn_fwd)(qc, kc, vc, gc, mask_bias, pair_bias)
    out_c, lse = res[0], res[1]
    out_rows = cols_to_rows(_tri_end_view(out_c), n, group)
    return out_rows, lse, {"q": qc, "k": kc, "v": vc, "g": gc, "out": out_c}


def tri_end_bwd(saved, mask_bias, pair_bias, lse, dout_rows, n, group=None, bwd=None, summer=None):
    """Backward of ``tri_end_fwd``.

    ``saved`` is the third result of tri_end_fwd; dout_rows the gradient of
    out in row shards.  dout goes to column shards, the backward runs there,
    dq, dk, dv, dg come back to row shards, and d_pair_bias is summed over
    the ranks in rank order.  Returns the gradients dict (row shards).
    """
    dout_c = _tri_end_view(rows_to_cols(dout_rows, n, group))
    out_c = saved["out"]
    if dout_c.stride() != out_c.stride():
        dout_c = A.empty_like_rows(out_c).copy_(dout_c)
    grads = row_shards.attn_bwd(saved["q"], saved["k"], saved["v"], saved["g"], mask_bias, pair_bias, out_c, lse,
                                dout_c, group=group, backward=bwd, summer=summer)
    res = {name: cols_to_rows(_tri_end_view(grads[name]), n, group) for name in ("dq", "dk", "dv", "dg")}
    res["d_pair_bias"] = grads["d_pair_bias"]
    return res
