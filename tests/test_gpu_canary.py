"""Guard bands around every output buffer (in place of compute-sanitizer,
closed on this pool): each output is a view in the middle of a larger
buffer whose 4 KiB on either side hold a fill pattern, and after the call
the pattern must be intact -- a write past either end of an output fails.

The cases run the library's paths on small ragged shapes: the fused decode
indexer, the prefill indexer, 128-head decode attention, HCA, 64-head
attention, pooling (codes, scales, pooled values) and the MXFP4 quantiser.
`test_guard_logic_on_cpu` runs the same cases with stand-ins for the calls,
which pins the guard mechanics themselves (and that a stray byte is seen)."""
import math
import types

import numpy as np
import pytest
import torch

import synth

GUARD = 4096          # bytes on each side (keeps every view 16-byte aligned)
FILL = 0x5A


def guarded(shape, dtype, device):
    n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((2 * GUARD + n,), FILL, dtype=torch.uint8, device=device)
    return buf, buf[GUARD:GUARD + n].view(dtype).view(shape)


def intact(buf):
    n = buf.numel() - 2 * GUARD
    return bool((buf[:GUARD] == FILL).all()) and bool((buf[GUARD + n:] == FILL).all())


def _indexer_case(ops, dev, B, Tq, N, K, pos, seed):
    ind = synth.indexer_inputs(B, Tq, N, 4, 64, seed=seed)
    d = ops.Dims(B=B, Tq=Tq, HI=4, dI=64, K=K, m=4, n_entries=N, entry_cap=N)
    bi, idx = guarded((B, Tq, K), torch.int32, dev)
    bs, sc = guarded((B, Tq, K), torch.float32, dev)
    nb = ops.index_topk_workspace(d)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    ops.index_topk(ind.qI.to(dev), ind.w.to(dev), ind.kI.to(dev), pos.to(dev), d, idx, sc, workspace=ws)
    return [bi, bs]


def _attend_case(ops, dev, B, Tq, H, N, K, W, win_cap, pos, m, seed, dense=False):
    D = 512
    codes, scales = synth.e4m3_cache(B, N, D, seed)
    wcodes, wscales = synth.e4m3_cache(B, win_cap, D, seed, tag="win")
    q = synth.queries(B, Tq, H, D, D ** -0.5, seed)
    d = ops.Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, entry_cap=N, win_cap=win_cap)
    bo, out = guarded((B, Tq, H, D), torch.bfloat16, dev)
    bl, lse = guarded((B, Tq, H), torch.float32, dev)
    nb = ops.attend_workspace(d, dense)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    tail = (wcodes.to(dev), wscales.to(dev), pos.to(dev), d, out, lse)
    if dense:
        ops.hca_attend(q.to(dev), codes.to(dev), scales.to(dev), *tail, workspace=ws)
    else:
        g = torch.Generator().manual_seed(seed)
        idx = torch.stack([torch.randperm(N, generator=g)[:K] for _ in range(B * Tq)]).view(B, Tq, K)
        ops.attend(q.to(dev), codes.to(dev), scales.to(dev), idx.to(torch.int32).to(dev), *tail, workspace=ws)
    return [bo, bl]


def _cases(ops, dev):
    bufs = []
    # fused decode indexer: one row per sequence at the last position
    bufs += _indexer_case(ops, dev, 4, 1, 3000, 512, torch.full((4, 1), 4 * 3000 - 1, dtype=torch.int32), 31)
    # prefill indexer: 300 rows, a ragged last tile of 128 query rows
    g = torch.Generator().manual_seed(32)
    pos = torch.randint(0, 4 * 3000 + 10, (1, 300), generator=g, dtype=torch.int32)
    bufs += _indexer_case(ops, dev, 1, 300, 3000, 100, pos, 32)
    # 128-head decode attention and HCA
    bufs += _attend_case(ops, dev, 2, 1, 128, 2000, 512, 128, 128,
                         torch.full((2, 1), 4 * 2000 - 1, dtype=torch.int32), 4, 33)
    bufs += _attend_case(ops, dev, 2, 1, 128, 300, 0, 128, 128,
                         torch.full((2, 1), 128 * 300 - 1, dtype=torch.int32), 128, 34, dense=True)
    # 64-head attention: 70 rows
    pos = torch.randint(0, 4 * 600, (1, 70), generator=g, dtype=torch.int32)
    bufs += _attend_case(ops, dev, 1, 70, 64, 600, 100, 50, 4 * 600, pos, 4, 35)
    # pooling (m = 4, with the pooled copy) and the window entries (m = 1)
    x, z = synth.tokens(2, 66, 512, 36)
    bc, codes = guarded((2, 16, 512), torch.uint8, dev)
    bsc, scales = guarded((2, 16), torch.float32, dev)
    bp, pooled = guarded((2, 16, 512), torch.float32, dev)
    ops.compress(x.to(dev), z.to(dev), 4, codes, scales, pooled=pooled)
    bwc, wcodes = guarded((2, 66, 512), torch.uint8, dev)
    bws, wscales = guarded((2, 66), torch.float32, dev)
    ops.compress(x.to(dev), z.to(dev), 1, wcodes, wscales)
    bufs += [bc, bsc, bp, bwc, bws]
    # MXFP4 quantiser
    xq = torch.randn((37, 96), generator=g)
    bq, qc = guarded((37, 48), torch.uint8, dev)
    bqs, qs = guarded((37, 3), torch.uint8, dev)
    ops.quantize_mxfp4(xq.to(dev), qc, qs)
    bufs += [bq, bqs]
    return bufs


@pytest.mark.gpu
def test_no_write_outside_outputs():
    import compressed_sparse_attention_16_b200 as csa
    bufs = _cases(csa, torch.device("cuda"))
    torch.cuda.synchronize()
    csa.sync_status()
    bad = [i for i, b in enumerate(bufs) if not intact(b)]
    assert not bad, f"guard bands overwritten around outputs {bad}"


def test_guard_logic_on_cpu():
    """The same cases with stand-ins that fill every output element: no guard
    is touched; then one stray byte on either side is detected."""
    from compressed_sparse_attention_16_b200 import Dims

    def fill(*ts):
        for t in ts:
            if t is not None:
                t.view(torch.uint8).fill_(0)

    fake = types.SimpleNamespace(
        Dims=Dims,
        index_topk_workspace=lambda d: 0,
        attend_workspace=lambda d, dense=False: 0,
        index_topk=lambda qI, w, kI, pos, d, idx, sc, workspace=None: fill(idx, sc),
        attend=lambda q, c, s, idx, wc, ws_, pos, d, out, lse, workspace=None: fill(out, lse),
        hca_attend=lambda q, c, s, wc, ws_, pos, d, out, lse, workspace=None: fill(out, lse),
        compress=lambda x, z, m, codes, scales, pooled=None: fill(codes, scales, pooled),
        quantize_mxfp4=lambda x, codes, scales: fill(codes, scales),
    )
    bufs = _cases(fake, torch.device("cpu"))
    assert len(bufs) == 17
    for b in bufs:
        assert intact(b)
        n = b.numel() - 2 * GUARD
        assert (b[GUARD:GUARD + n] == 0).all()          # the view covers the whole output
        b[GUARD - 1] = 0
        assert not intact(b)
        b[GUARD - 1] = FILL
        b[GUARD + n] = 0
        assert not intact(b)
        b[GUARD + n] = FILL
