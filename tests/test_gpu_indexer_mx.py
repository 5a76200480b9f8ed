"""GPU parity of csa_index_topk_mx (block-scaled FP4 indexer) against the
oracle's fp64 scores, with the tie-tolerant top-k check of tests/parity.py:
listed entries distinct and visible, reported scores within MX_RTOL * mag of
the exact ones and descending, and no left-out entry able to beat a listed
one.  With unit scales and weights on the 1/16 grid the path is exact and
must equal csa_index_topk bit for bit."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims
from oracle import csa as ocsa
from tests.parity import MX_RTOL, check_topk_tolerant

pytestmark = pytest.mark.gpu


def _run_mx(inp, q_pos, m, K, N):
    B, Tq, HI, half = inp.qI.shape
    d = Dims(B=B, Tq=Tq, HI=HI, dI=2 * half, K=K, m=m, n_entries=N, entry_cap=inp.kI.shape[1])
    dev = "cuda"
    idx = torch.full((B, Tq, K), -7, dtype=torch.int32, device=dev)
    sc = torch.full((B, Tq, K), -7.0, device=dev)
    ws = torch.empty(max(1, csa.index_topk_mx_workspace(d)), dtype=torch.uint8, device=dev)
    csa.index_topk_mx(inp.qI.to(dev), inp.qs.to(dev), inp.w.to(dev), inp.kI.to(dev), inp.ks.to(dev),
                      q_pos.to(dev), d, idx, sc, workspace=ws)
    csa.sync_status()
    return idx.cpu().numpy(), sc.cpu().numpy()


def _check(inp, q_pos, m, K, N):
    gi, gs = _run_mx(inp, q_pos, m, K, N)
    s, mag = ocsa.indexer_scores_mx(inp.qI.cpu().numpy(), inp.qs.cpu().numpy(), inp.w.cpu().numpy(),
                                    inp.kI[:, :N].cpu().numpy(), inp.ks[:, :N].cpu().numpy())
    nv = ocsa.n_visible(q_pos.cpu().numpy(), m, N)
    B, Tq = nv.shape
    swapped = check_topk_tolerant(gi.reshape(B * Tq, K), gs.reshape(B * Tq, K), s.reshape(B * Tq, N),
                                  mag.reshape(B * Tq, N), nv.reshape(-1), K)
    # how close the computed scores came to the exact ones, relative to the bound
    sel = gi >= 0
    if sel.any():
        ref = np.take_along_axis(s, np.maximum(gi, 0), axis=2)[sel]
        mg = np.take_along_axis(mag, np.maximum(gi, 0), axis=2)[sel]
        rel = np.abs(gs[sel].astype(np.float64) - ref) / np.maximum(mg, 1e-300)
        print(f"max |gpu - exact| / mag = {rel.max():.3g} (bound {MX_RTOL:.3g}); rows with swapped near-ties: {swapped}")
    return gi, gs


def test_decode_64k_shape():
    """16 sequences x 16,384 entries, 4 x 64 indexer, top 512: every row."""
    B, N, K = 16, 16384, 512
    inp = synth.indexer_inputs_mx(B, 1, N, 4, 64, seed=31)
    q_pos = torch.full((B, 1), 4 * N - 1, dtype=torch.int32)
    q_pos[3, 0] = 4 * 3000 + 1       # a shorter context
    q_pos[5, 0] = 4 * 512 - 1        # exactly k visible
    q_pos[7, 0] = 4 * 100            # fewer than k visible
    _check(inp, q_pos, 4, K, N)


@pytest.mark.parametrize("HI", [1, 4, 8])
def test_small_rows_ragged_positions(HI):
    B, Tq, N, m, K = 2, 9, 1300, 4, 37
    inp = synth.indexer_inputs_mx(B, Tq, N, HI, 64, seed=40 + HI)
    g = torch.Generator().manual_seed(HI)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    pos[0, :5] = torch.tensor([0, 3, 4 * K - 1, 4 * K, 4 * N - 1], dtype=torch.int32)
    _check(inp, pos, m, K, N)


def test_many_rows_several_slices_and_k_extremes():
    """64 rows over 9,000 entries (several 4,096-entry slices per row); k = 1
    and k = 2,048."""
    B, Tq, N, m = 2, 32, 9000, 4
    inp = synth.indexer_inputs_mx(B, Tq, N, 4, 64, seed=50)
    g = torch.Generator().manual_seed(50)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    for K in (1, 2048):
        _check(inp, pos, m, K, N)


def test_wide_scale_range():
    """Block scales 2^-40 .. 2^40: the two blocks of a row weigh very
    differently, so the fp32 sums round."""
    B, Tq, N, m, K = 1, 6, 3000, 4, 100
    inp = synth.indexer_inputs_mx(B, Tq, N, 4, 64, seed=60, spread=40)
    pos = torch.tensor([[4 * N - 1, 4 * N - 1, 5000, 800, 401, 4 * N - 3]], dtype=torch.int32)
    _check(inp, pos, m, K, N)


def test_unit_scales_equal_the_exact_indexer():
    """Scale codes 127 everywhere and weights on the 1/16 grid: the scores
    are exact, so indices and scores equal csa_index_topk's bit for bit."""
    B, Tq, N, m, K = 4, 3, 6000, 4, 512
    base = synth.indexer_inputs(B, Tq, N, 4, 64, seed=70)
    inp = synth.IndexerInputsMX(qI=base.qI, qs=torch.full((B, Tq, 4, 2), 127, dtype=torch.uint8), w=base.w,
                                kI=base.kI, ks=torch.full((B, N, 2), 127, dtype=torch.uint8))
    pos = torch.tensor([[4 * N - 1, 2500, 4 * 600], [4 * N - 5, 4 * N - 1, 17], [100, 4 * N - 1, 4 * 512],
                        [4 * N - 1, 4 * N - 1, 4 * N - 1]], dtype=torch.int32)
    gi, gs = _run_mx(inp, pos, m, K, N)
    d = Dims(B=B, Tq=Tq, HI=4, dI=64, K=K, m=m, n_entries=N)
    idx = torch.full((B, Tq, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Tq, K), -7.0, device="cuda")
    ws = torch.empty(max(1, csa.index_topk_workspace(d)), dtype=torch.uint8, device="cuda")
    csa.index_topk(base.qI.cuda(), base.w.cuda(), base.kI.cuda(), pos.cuda(), d, idx, sc, workspace=ws)
    csa.sync_status()
    assert np.array_equal(gi, idx.cpu().numpy())
    assert np.array_equal(gs, sc.cpu().numpy())


def test_equal_scores_take_lowest_indices():
    B, Tq, N, m, K = 1, 2, 5000, 4, 300
    inp = synth.indexer_inputs_mx(B, Tq, N, 2, 64, seed=80)
    inp.kI[:] = inp.kI[:, :1]          # every key the same: every score equal
    inp.ks[:] = inp.ks[:, :1]
    pos = torch.tensor([[4 * N - 1, 4 * 1000]], dtype=torch.int32)
    gi, _ = _run_mx(inp, pos, m, K, N)
    assert (gi[0, 0] == np.arange(K)).all() and (gi[0, 1] == np.arange(K)).all()


def test_bad_scale_and_weight_are_reported():
    B, Tq, N = 1, 1, 600
    for what in ("scale", "weight"):
        inp = synth.indexer_inputs_mx(B, Tq, N, 4, 64, seed=90)
        if what == "scale":
            inp.ks[0, 10, 1] = 0xFF
        else:
            inp.w[0, 0, 2] = -0.5
        with pytest.raises(csa.CsaError) as e:
            _run_mx(inp, torch.tensor([[4 * N - 1]], dtype=torch.int32), 4, 64, N)
        assert e.value.code == csa.CSA_ERR_INVALID


def test_unsupported_shapes_are_refused():
    d = Dims(B=1, Tq=1, HI=4, dI=32, K=64, m=4, n_entries=1000)
    assert csa.index_topk_mx_workspace(d) == 0
    big = Dims(B=1, Tq=1, HI=4, dI=64, K=2048, m=4, n_entries=60000)    # 15 slices x 2048 > 20,480
    assert csa.index_topk_mx_workspace(big) == 0
    inp = synth.indexer_inputs_mx(1, 1, 8, 4, 64, seed=91)
    with pytest.raises(csa.CsaError) as e:
        idx = torch.empty((1, 1, 2048), dtype=torch.int32, device="cuda")
        csa.index_topk_mx(inp.qI.cuda(), inp.qs.cuda(), inp.w.cuda(), inp.kI.cuda(), inp.ks.cuda(),
                          torch.zeros((1, 1), dtype=torch.int32, device="cuda"), big, idx,
                          workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == csa.CSA_ERR_UNSUPPORTED


def test_pooled_and_quantised_keys_end_to_end():
    """The f2 chain on the GPU: per-token fp32 indexer keys pooled per block of
    4 (csa_compress, fp32 pooled output), quantised to MXFP4
    (csa_quantize_mxfp4), queries quantised likewise, then csa_index_topk_mx.
    The oracle runs its own chain (pool, quantise, score).  The two chains
    round the pooled values differently, so an element may land on the
    neighbouring E2M1 code and move its key's score by more than the
    evaluation bound: the check is that at least 99 % of the oracle's top-k
    is listed per row, and that the listed entries' exact scores (on the
    oracle's codes) all reach the oracle's k-th score minus 2 % of its
    magnitude."""
    B, T, D, m, K, HI = 4, 16384, 64, 4, 512, 4
    N = T // m
    x, z = synth.tokens(B, T, D, seed=100)
    qf = torch.randn((B, 1, HI, D), generator=torch.Generator().manual_seed(101))
    w = torch.rand((B, 1, HI), generator=torch.Generator().manual_seed(102))
    dev = "cuda"
    pooled = torch.empty((B, N, D), device=dev)
    codes = torch.empty((B, N, D), dtype=torch.uint8, device=dev)
    scales = torch.empty((B, N), device=dev)
    csa.compress(x.to(dev), z.to(dev), m, codes, scales, pooled=pooled)
    kI = torch.empty((B * N, D // 2), dtype=torch.uint8, device=dev)
    ks = torch.empty((B * N, D // 32), dtype=torch.uint8, device=dev)
    csa.quantize_mxfp4(pooled.view(B * N, D), kI, ks)
    qI = torch.empty((B * HI, D // 2), dtype=torch.uint8, device=dev)
    qs = torch.empty((B * HI, D // 32), dtype=torch.uint8, device=dev)
    csa.quantize_mxfp4(qf.view(B * HI, D).to(dev), qI, qs)
    inp = synth.IndexerInputsMX(qI=qI.view(B, 1, HI, D // 2), qs=qs.view(B, 1, HI, D // 32), w=w,
                                kI=kI.view(B, N, D // 2), ks=ks.view(B, N, D // 32))
    q_pos = torch.full((B, 1), T - 1, dtype=torch.int32)
    gi, _ = _run_mx(inp, q_pos, m, K, N)
    # the oracle's chain
    p_ref = ocsa.compress(x.numpy(), z.numpy(), m)                       # [B, N, D] fp64
    from oracle.formats import mxfp4_quantize
    kc, kscl = mxfp4_quantize(p_ref.reshape(B * N, D).astype(np.float32))
    qc, qscl = mxfp4_quantize(qf.numpy().reshape(B * HI, D))
    s, mag = ocsa.indexer_scores_mx(qc.reshape(B, 1, HI, D // 2), qscl.reshape(B, 1, HI, D // 32), w.numpy(),
                                    kc.reshape(B, N, D // 2), kscl.reshape(B, N, D // 32))
    for b in range(B):
        ref = s[b, 0]
        top = np.lexsort((np.arange(N), -ref))[:K]
        got = gi[b, 0]
        assert (got >= 0).all() and np.unique(got).size == K
        recall = np.intersect1d(top, got).size / K
        assert recall >= 0.99, f"sequence {b}: recall {recall:.4f}"
        kth = ref[top[-1]]
        assert (ref[got] >= kth - 0.02 * mag[b, 0, got]).all()
