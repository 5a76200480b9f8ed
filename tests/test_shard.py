"""Host logic of the sharded prefill (compressed_sparse_attention_16_b200.shard)
on CPU: the block, token and row partitions, and two and three gloo ranks
whose gathered caches and per-row calls match a single-process run.  The
library's calls are replaced by CPU stand-ins whose outputs depend on exactly
the data each call must see (the tokens of a block, the whole gathered cache,
a row's position and inputs), so a wrong range, a misplaced shard or a
missing gather changes the result."""
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressed_sparse_attention_16_b200 import shard


@pytest.mark.parametrize("N,world", [(0, 2), (1, 3), (7, 2), (8, 4), (32768, 8), (5, 5), (3, 5)])
def test_block_ranges_cover_once_and_balance(N, world):
    rs = [shard.block_range(N, world, r) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == N
    assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
    lens = [b - a for a, b in rs]
    assert max(lens) - min(lens) <= 1


@pytest.mark.parametrize("T,m,world", [(512, 4, 2), (515, 4, 3), (131072, 4, 8), (130, 128, 2), (3, 4, 2)])
def test_token_ranges_and_rows(T, m, world):
    tr = [shard.token_range(T, m, world, r) for r in range(world)]
    assert tr[0][0] == 0 and tr[-1][1] == T
    assert all(tr[i][1] == tr[i + 1][0] for i in range(world - 1))
    for r, (t0, t1) in enumerate(tr):
        b0, b1 = shard.block_range(T // m, world, r)
        assert t0 == b0 * m and (t1 == b1 * m or r == world - 1)
    rows = torch.cat([shard.row_positions(T, world, r) for r in range(world)])
    assert torch.equal(rows.sort().values, torch.arange(T, dtype=torch.int32))


# ---------------------------------------------------------------- stand-ins


def fake_compress(x, z, m, codes, scales, dst_first=0, ring_cap=0, pooled=None, T=None, first_token=0,
                  stream=None):
    B, Ttot, D = x.shape
    T = Ttot - first_token if T is None else T
    n = T // m
    blk = x[:, first_token:first_token + n * m].reshape(B, n, m, D)
    zb = z[:, first_token:first_token + n * m].reshape(B, n, m, D)
    codes[:, dst_first:dst_first + n] = (blk.sum(2) * 16).round().to(torch.int64).remainder(256).to(torch.uint8)
    scales[:, dst_first:dst_first + n] = zb.sum((2, 3)) + m


def fake_index_topk(qI, w, kI, q_pos, dims, idx, score=None, workspace=None, stream=None):
    ks = kI.to(torch.int64).sum(-1)                                   # [B, N]
    for b in range(dims.B):
        for r in range(dims.Tq):
            t = int(q_pos[b, r])
            nv = min((t + 1) // dims.m, dims.n_entries)
            h = int(ks[b, :nv].sum()) + int(qI[b, r].to(torch.int64).sum()) + int((w[b, r] * 16).sum())
            j = torch.arange(dims.K, dtype=torch.int64)
            idx[b, r] = torch.where(j < nv, (h + 7 * j) % max(nv, 1), -1).to(torch.int32)
            if score is not None:
                score[b, r] = float(h % 1000) + j.to(torch.float32)


def fake_attend(q, codes, scales, idx, wcodes, wscales, q_pos, dims, out, lse, workspace=None, stream=None):
    for b in range(dims.B):
        for r in range(dims.Tq):
            t = int(q_pos[b, r])
            sel = idx[b, r][idx[b, r] >= 0].to(torch.int64)
            lo = max(0, t - dims.W + 1)
            e = codes[b, sel].to(torch.float32).sum(0) + wcodes[b, lo:t + 1].to(torch.float32).sum(0)   # [D]
            out[b, r] = (q[b, r].to(torch.float32) + e[None] / 1024).to(out.dtype)
            lse[b, r] = scales[b, sel].sum() + wscales[b, lo:t + 1].sum() + t


def _install():
    shard.compress = fake_compress
    shard.index_topk = fake_index_topk
    shard.attend = fake_attend
    shard.index_topk_workspace = lambda d: 0
    shard.attend_workspace = lambda d: 0


def _inputs(B, T, D, H, HI, dI, m):
    g = torch.Generator().manual_seed(7)
    x = torch.randn((B, T, D), generator=g)
    z = torch.randn((B, T, D), generator=g)
    kI = torch.randint(0, 256, (B, T // m, dI // 2), generator=g, dtype=torch.uint8)
    q = torch.randn((B, T, H, D), generator=g).to(torch.bfloat16)
    qI = torch.randint(0, 256, (B, T, HI, dI // 2), generator=g, dtype=torch.uint8)
    w = torch.randint(0, 17, (B, T, HI), generator=g).to(torch.float32) / 16
    return x, z, kI, q, qI, w


SHAPE = dict(B=2, T=203, D=8, H=3, HI=2, dI=8, m=4)
KW = dict(K=6, W=5)


def _worker(rank, world, port, q_out):
    from datetime import timedelta
    _install()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        s = SHAPE
        x, z, kI, q, qI, w = _inputs(s["B"], s["T"], s["D"], s["H"], s["HI"], s["dI"], s["m"])
        t0, t1 = shard.token_range(s["T"], s["m"], world, rank)
        b0, b1 = shard.block_range(s["T"] // s["m"], world, rank)
        pos = shard.row_positions(s["T"], world, rank).to(torch.int64)
        r = shard.prefill_sharded(x[:, t0:t1].contiguous(), z[:, t0:t1].contiguous(), kI[:, b0:b1].contiguous(),
                                  q[:, pos].contiguous(), qI[:, pos].contiguous(), w[:, pos].contiguous(),
                                  T=s["T"], m=s["m"], **KW)
        q_out.put((rank, r.pos, r.out, r.lse, r.idx, r.score))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _reference():
    """The same stand-ins over the whole sequence in one process."""
    s = SHAPE
    x, z, kI, q, qI, w = _inputs(s["B"], s["T"], s["D"], s["H"], s["HI"], s["dI"], s["m"])
    B, T, D, H, m = s["B"], s["T"], s["D"], s["H"], s["m"]
    N = T // m
    codes = torch.empty((B, N, D), dtype=torch.uint8)
    scales = torch.empty((B, N))
    wc = torch.empty((B, T, D), dtype=torch.uint8)
    wsc = torch.empty((B, T))
    fake_compress(x, z, m, codes, scales)
    fake_compress(x, z, 1, wc, wsc)
    q_pos = torch.arange(T, dtype=torch.int32).repeat(B, 1)
    dims = shard.Dims(B=B, Tq=T, H=H, D=D, HI=s["HI"], dI=s["dI"], m=m, n_entries=N, entry_cap=N, win_cap=T, **KW)
    idx = torch.empty((B, T, KW["K"]), dtype=torch.int32)
    sc = torch.empty((B, T, KW["K"]))
    fake_index_topk(qI, w, kI, q_pos, dims, idx, sc)
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16)
    lse = torch.empty((B, T, H))
    fake_attend(q, codes, scales, idx, wc, wsc, q_pos, dims, out, lse)
    return out, lse, idx, sc


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_single_process(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q_out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out, lse, idx, sc = _reference()
    seen = torch.zeros(SHAPE["T"], dtype=torch.int64)
    for rank, pos, o, l, i, s in got:
        p = pos.to(torch.int64)
        seen[p] += 1
        assert torch.equal(o, out[:, p]) and torch.equal(l, lse[:, p])
        assert torch.equal(i, idx[:, p]) and torch.equal(s, sc[:, p])
    assert (seen == 1).all()
