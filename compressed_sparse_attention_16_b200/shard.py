"""CSA prefill of one batch of sequences split across the ranks of a
torch.distributed process group (one process per GPU), by query rows.

Source: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
Attention (CSA)": every query's indexer, top-k and attention read the whole
compressed sequence but nothing of the other queries, so query rows are
independent once every rank holds the compressed cache.

Each rank

1. pools a contiguous range of the m-token blocks (:func:`block_range`) and
   stores the window entries of the same tokens (:func:`token_range`; the
   last rank also takes the partial tail block's tokens, which are window
   entries only);
2. takes part in one all-gather per buffer (entry codes and scales, window
   codes and scales, indexer keys), after which every rank holds the whole
   cache -- the only exchange of the path;
3. runs the indexer, top-k and attention for its own query rows, the
   positions t = rank, rank + world, ... (:func:`row_positions`): interleaved,
   so that every rank gets the same mix of short and long visible ranges.

Nothing here computes; the steps are the library's calls and torch's
collectives and copies.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import Dims, attend, attend_workspace, compress, index_topk, index_topk_workspace


def block_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Blocks [b0, b1) pooled by `rank`: N blocks in `world` contiguous ranges
    whose lengths differ by at most one."""
    base, rem = divmod(N, world)
    b0 = rank * base + min(rank, rem)
    return b0, b0 + base + (1 if rank < rem else 0)


def token_range(T: int, m: int, world: int, rank: int) -> tuple[int, int]:
    """Tokens [t0, t1) whose window entries `rank` stores: the tokens of its
    blocks, and for the last rank also the tokens of the partial tail."""
    b0, b1 = block_range(T // m, world, rank)
    return b0 * m, (T if rank == world - 1 else b1 * m)


def row_positions(T: int, world: int, rank: int) -> torch.Tensor:
    """Query positions handled by `rank`: rank, rank + world, ... < T."""
    return torch.arange(rank, T, world, dtype=torch.int32)


@dataclasses.dataclass
class ShardResult:
    pos: torch.Tensor        # int32 [R] positions of this rank's rows
    out: torch.Tensor        # bf16 [B, R, H, D]
    lse: torch.Tensor        # f32 [B, R, H]
    idx: torch.Tensor        # int32 [B, R, K]
    score: torch.Tensor      # f32 [B, R, K]


def _gather(local: torch.Tensor, lengths: list[int], group) -> torch.Tensor:
    """All-gather along dim 1 of [B, L_r, ...] pieces of unequal lengths L_r:
    each piece is padded to max(L_r) for the collective, then the pieces are
    concatenated in rank order."""
    L = max(lengths)
    if L == 0:   # the same on every rank: all skip the collective
        return local.contiguous()
    pad = torch.zeros((local.shape[0], L) + tuple(local.shape[2:]), dtype=local.dtype, device=local.device)
    pad[:, : local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in lengths]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :n] for p, n in zip(parts, lengths)], dim=1).contiguous()


def prefill_sharded(x_loc, z_loc, kI_loc, q_rows, qI_rows, w_rows, *, T: int, m: int, K: int, W: int,
                    group=None, softmax_scale: float = 1.0) -> ShardResult:
    """This rank's share of a CSA prefill of B sequences of T tokens.

    x_loc, z_loc: f32 [B, t1 - t0, D], tokens [t0, t1) = token_range(T, m, world, rank);
    kI_loc: u8 [B, b1 - b0, dI/2], indexer keys of blocks block_range(T // m, world, rank);
    q_rows: bf16 [B, R, H, D], qI_rows: u8 [B, R, HI, dI/2], w_rows: f32 [B, R, HI] for the
    positions row_positions(T, world, rank).
    Returns the outputs of those rows.  Every rank must call it (it takes part
    in collectives).
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, _, D = x_loc.shape
    H = q_rows.shape[2]
    HI, dI = qI_rows.shape[2], 2 * qI_rows.shape[3]
    dev = x_loc.device
    N = T // m
    b0, b1 = block_range(N, world, rank)
    t0, t1 = token_range(T, m, world, rank)
    if x_loc.shape[1] != t1 - t0 or kI_loc.shape[1] != b1 - b0:
        raise ValueError("x_loc / kI_loc do not match this rank's token and block ranges")
    # 1. this rank's entries and window entries
    codes = torch.empty((B, b1 - b0, D), dtype=torch.uint8, device=dev)
    scales = torch.empty((B, b1 - b0), dtype=torch.float32, device=dev)
    win_codes = torch.empty((B, t1 - t0, D), dtype=torch.uint8, device=dev)
    win_scales = torch.empty((B, t1 - t0), dtype=torch.float32, device=dev)
    if b1 > b0:
        compress(x_loc, z_loc, m, codes, scales, T=(b1 - b0) * m)
    if t1 > t0:
        compress(x_loc, z_loc, 1, win_codes, win_scales)
    # 2. the whole cache on every rank
    blens = [block_range(N, world, r)[1] - block_range(N, world, r)[0] for r in range(world)]
    tlens = [token_range(T, m, world, r)[1] - token_range(T, m, world, r)[0] for r in range(world)]
    codes = _gather(codes, blens, group)
    scales = _gather(scales, blens, group)
    kI = _gather(kI_loc.contiguous(), blens, group)
    win_codes = _gather(win_codes, tlens, group)
    win_scales = _gather(win_scales, tlens, group)
    # 3. this rank's query rows
    pos = row_positions(T, world, rank)
    R = pos.numel()
    if q_rows.shape[1] != R or qI_rows.shape[1] != R or w_rows.shape[1] != R:
        raise ValueError("q_rows / qI_rows / w_rows do not match this rank's rows")
    q_pos = pos.to(dev).repeat(B, 1).contiguous()
    dims = Dims(B=B, Tq=R, H=H, D=D, HI=HI, dI=dI, K=K, W=W, m=m, n_entries=N, entry_cap=N, win_cap=T,
                softmax_scale=softmax_scale)
    idx = torch.empty((B, R, K), dtype=torch.int32, device=dev)
    score = torch.empty((B, R, K), dtype=torch.float32, device=dev)
    out = torch.empty((B, R, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, R, H), dtype=torch.float32, device=dev)
    if R > 0:
        nb = index_topk_workspace(dims)
        index_topk(qI_rows, w_rows, kI, q_pos, dims, idx, score,
                   workspace=torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None)
        nb = attend_workspace(dims)
        attend(q_rows, codes, scales, idx, win_codes, win_scales, q_pos, dims, out, lse,
               workspace=torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None)
    return ShardResult(pos, out, lse, idx, score)
