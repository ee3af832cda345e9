"""Row-sharded triangle attention across ranks (one process per GPU).

The starting-node problems of different rows i are independent: each is a softmax
attention within row i, and only the pair bias is shared by all rows ("16张H100，训练步
提速1.73倍：TurboPairFormer为什么不是‘装个包就能加速AlphaFold3’", section "它优化了什么，
而不是只‘少存一点张量’", on the four gradients).  The partition is the 1-D row sharding of
the pair representation in "Design-CP: Context Parallelism for Design of Protein
Nanoparticles", section "方法论", item "1. 推理策略": rank r owns a contiguous block of
rows and runs the forward and the dq/dk/dv part of the backward on it alone.

The one exchange is dBias, the sum over all rows i of the score gradient: every rank
computes its block's share as FP32 partial sums (`tri_attn_bwd_rows`), the shares are
all-gathered in rank order, and every rank adds the gathered array in ascending index
order (`tri_attn_dbias_sum`), so all ranks hold the same BF16 dBias bit for bit.

The bias itself is an input replicated on every rank; the pair tensors, the mask, lse
and the gradients of a rank are views of its own rows.
"""
from __future__ import annotations

from . import _binding as Bd


def row_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """(first row, number of rows) of `rank`'s block: contiguous, sizes differ by at most
    one, larger blocks first.  Needs 1 <= world <= N."""
    if world < 1 or world > N or not 0 <= rank < world:
        raise ValueError(f"cannot split {N} rows over {world} ranks (rank {rank})")
    base, extra = divmod(N, world)
    i0 = rank * base + min(rank, extra)
    return i0, base + (1 if rank < extra else 0)


def dbias_parts(B: int, N: int, H: int, d: int, world: int) -> int:
    """Partial-sum slots per rank: the most any rank's block needs (blocks of unequal
    size may need different numbers); ranks with fewer leave the rest zero."""
    return max(Bd.tri_attn_bwd_rows_dbias_parts(B, row_range(N, r, world)[1], N, H, d) for r in range(world))


def gather_parts(local, group=None):
    """All ranks' partial sums stacked in rank order: [world * P, ...] from [P, ...]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local.contiguous(), group=group)
    else:
        dist.all_gather(list(out.chunk(world)), local.contiguous(), group=group)
    return out


def shard_fwd(q, k, v, bias, mask, o, resid, lse, scale: float = 0.0, stream=None) -> None:
    """Forward of this rank's rows: q, k, v, o, resid [B,R,N,H,d] and mask [B,R,N] are its
    block's views, bias the full [B,H,N,N], lse its own [B,H,R,N]."""
    Bd.tri_attn_fwd_rows(q, k, v, bias, mask, o, resid, lse, scale, stream)


def shard_bwd(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, dbias, workspace, parts,
              group=None, scale: float = 0.0, flags: int = 0, stream=None) -> None:
    """Backward of this rank's rows plus the dBias exchange.

    parts: contiguous float32 [P, B, H, N, N] with P = dbias_parts(B, N, H, d, world);
    dbias: BF16 [B,H,N,N], written on every rank (identical everywhere).  Collective:
    every rank of `group` must call it, in the same order as its other collectives."""
    import torch.distributed as dist
    B, R, N, H, d = q.shape
    world = dist.get_world_size(group)
    P = dbias_parts(B, N, H, d, world)
    if tuple(parts.shape) != (P, B, H, N, N):
        raise Bd.TriAttnError(Bd.TRI_ATTN_ERR_SHAPE, f"parts must be {(P, B, H, N, N)}")
    mine = Bd.tri_attn_bwd_rows_dbias_parts(B, R, N, H, d)
    if mine < P:
        parts[mine:].zero_()  # empty slots add nothing
    Bd.tri_attn_bwd_rows(q, k, v, bias, mask, o, resid, lse, dout, dq, dk, dv, parts[:mine], workspace,
                         scale, flags, stream)
    Bd.tri_attn_dbias_sum(gather_parts(parts, group), dbias, stream)
