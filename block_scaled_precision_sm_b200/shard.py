"""The block-scaled GEMM split over the ranks of a process group, one GPU per rank.

Dense (N-sharded): D = A * B^T splits along N with no exchange step.  Rank r holds all of A
and its scales, and its column shard B[n0:n1] with the matching rows of B's scales; it
computes D[:, n0:n1] with gemm_fp8_nt on its own GPU.  Where every rank needs the whole D,
one all-gather of the column shards through the process group follows (NCCL over NVLink on
GPUs).  Shard boundaries fall on multiples of 128 rows of B, so a 128 x 128 scale block of B
never straddles two ranks.

M-grouped (expert-sharded): the experts are split into contiguous ranges; rank r holds the
weights of its experts and the rows already routed to them (the routing itself, an
all-to-all dispatch, is not part of this GEMM) and runs the grouped GEMM on them with its
local expert numbers.

No kernel here reads another GPU's memory: each rank's GEMM reads only its own tensors, and
the gather is the process group's collective.
"""

from __future__ import annotations

import torch

from . import ops

SHARD_ALIGN = 128


def n_shard_bounds(n: int, world: int, align: int = SHARD_ALIGN) -> list[tuple[int, int]]:
    """Column ranges [n0, n1) of D (rows of B) per rank: whole blocks of `align` rows, as even as
    the blocks allow (earlier ranks take the extra blocks); ranks beyond the block count get
    empty ranges."""
    if n <= 0 or world <= 0 or align <= 0:
        raise ValueError("n, world and align must be positive")
    blocks = -(-n // align)
    per, extra = divmod(blocks, world)
    bounds, b0 = [], 0
    for r in range(world):
        nb = per + (1 if r < extra else 0)
        bounds.append((min(b0 * align, n), min((b0 + nb) * align, n)))
        b0 += nb
    return bounds


def expert_shard_bounds(groups: int, world: int) -> list[tuple[int, int]]:
    """Expert ranges [g0, g1) per rank, as even as possible (earlier ranks take the extra)."""
    if groups <= 0 or world <= 0:
        raise ValueError("groups and world must be positive")
    per, extra = divmod(groups, world)
    bounds, g0 = [], 0
    for r in range(world):
        g1 = g0 + per + (1 if r < extra else 0)
        bounds.append((g0, g1))
        g0 = g1
    return bounds


def shard_b(B: torch.Tensor, sfb: torch.Tensor, n: int, rank: int, world: int, sfb_gran_n: int = 128):
    """This rank's rows of B [N, K] and of its UE8M0 scales [ceil(N/g), K/128] (unpacked)."""
    n0, n1 = n_shard_bounds(n, world)[rank]
    if SHARD_ALIGN % sfb_gran_n:
        raise ValueError("sfb_gran_n must divide the shard alignment")
    return B[n0:n1], sfb[n0 // sfb_gran_n:-(-n1 // sfb_gran_n)]


def gemm_fp8_nt_n_sharded(A, sfa, B_local, sfb_local, n: int, rank: int, world: int, sfb_gran_n: int = 128,
                          D_local=None, gather: bool = False, group=None, stream=None) -> torch.Tensor:
    """D[:, n0:n1] = A * B_local^T on this rank's GPU (B_local: rows [n0, n1) of B); with
    gather=True every rank returns the whole D [M, N], all-gathered through `group`."""
    n0, n1 = n_shard_bounds(n, world)[rank]
    m = A.shape[0]
    if B_local.shape[0] != n1 - n0:
        raise ValueError(f"rank {rank} holds rows [{n0}, {n1}) of B, got {B_local.shape[0]}")
    if n1 > n0:
        D_local = ops.gemm_fp8_nt(A, sfa, B_local, sfb_local, D_local, sfb_gran_n=sfb_gran_n, stream=stream)
    elif D_local is None:
        D_local = torch.empty((m, 0), dtype=torch.bfloat16, device=A.device)
    if not gather:
        return D_local
    return all_gather_columns(D_local, n_shard_bounds(n, world), group)


def all_gather_columns(D_local: torch.Tensor, bounds: list[tuple[int, int]], group=None) -> torch.Tensor:
    """Concatenate every rank's column shard [M, n1 - n0] into [M, N] on every rank.

    The shards may differ in width: each is padded to the widest one for a single
    all-gather, and the valid columns are kept."""
    import torch.distributed as dist

    widths = [n1 - n0 for n0, n1 in bounds]
    wmax = max(widths)
    m = D_local.shape[0]
    buf = torch.zeros((m, wmax), dtype=D_local.dtype, device=D_local.device)
    buf[:, :D_local.shape[1]] = D_local
    parts = [torch.empty_like(buf) for _ in bounds]
    dist.all_gather(parts, buf, group=group)
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)


def m_grouped_gemm_fp8_nt_expert_sharded(A_local, sfa_local, B_local, sfb_local, m_indices_local, groups: int,
                                          rank: int, world: int, D=None, sfb_gran_n: int = 128,
                                          stream=None) -> torch.Tensor:
    """The contiguous grouped GEMM on this rank's experts [g0, g1): B_local [g1 - g0, N, K] and
    the rows routed here, whose expert indices are local (0 .. g1 - g0 - 1, -1 for padding).
    An index outside that range is caught on the device (BSP_ERR_DEVICE_CHECK)."""
    g0, g1 = expert_shard_bounds(groups, world)[rank]
    if B_local.shape[0] != g1 - g0:
        raise ValueError(f"rank {rank} holds experts [{g0}, {g1}), got {B_local.shape[0]}")
    return ops.m_grouped_gemm_fp8_nt_contiguous(A_local, sfa_local, B_local, sfb_local, m_indices_local, D,
                                                sfb_gran_n=sfb_gran_n, stream=stream)


def localize_expert_indices(m_indices: torch.Tensor, groups: int, rank: int, world: int) -> torch.Tensor:
    """Global expert indices of rows routed to this rank -> local ones (padding stays -1)."""
    g0, _ = expert_shard_bounds(groups, world)[rank]
    return torch.where(m_indices >= 0, m_indices - g0, m_indices).to(torch.int32)
