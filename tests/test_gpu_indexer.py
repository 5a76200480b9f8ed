"""GPU parity of csa_index_topk: scores and top-k indices bit-exact against
the oracle's integer indexer and stable sort, through the C ABI."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims
from oracle import csa as ocsa

pytestmark = pytest.mark.gpu


def _gpu_topk(qI, w, kI, q_pos, m, K, n_entries):
    B, Tq, HI, half = qI.shape
    d = Dims(B=B, Tq=Tq, HI=HI, dI=2 * half, K=K, m=m, n_entries=n_entries, entry_cap=kI.shape[1])
    idx = torch.full((B, Tq, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Tq, K), -7.0, device="cuda")
    nb = csa.index_topk_workspace(d)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    csa.index_topk(qI.cuda(), w.cuda(), kI.cuda(), q_pos.cuda(), d, idx, sc, workspace=ws)
    csa.sync_status()
    return idx.cpu().numpy(), sc.cpu().numpy()


def _oracle_topk(qI, w, kI, q_pos, m, K, n_entries):
    s64 = ocsa.indexer_scores64(qI.numpy(), w.numpy(), kI[:, :n_entries].numpy())
    nv = ocsa.n_visible(q_pos.numpy(), m, n_entries)
    return ocsa.topk(s64, nv, K)


def _compare(qI, w, kI, q_pos, m, K, n_entries):
    gi, gs = _gpu_topk(qI, w, kI, q_pos, m, K, n_entries)
    ri, rs = _oracle_topk(qI, w, kI, q_pos, m, K, n_entries)
    assert np.array_equal(gi, ri), f"indices differ in rows {np.argwhere((gi != ri).any(-1))[:5].tolist()}"
    assert np.array_equal(gs.astype(np.float64), rs)


@pytest.mark.parametrize("HI,dI", [(4, 64), (2, 32), (1, 64), (8, 32), (4, 32), (2, 64), (1, 32)])
def test_prefill_rows_small(HI, dI):
    B, T, m, K = 2, 700, 4, 16
    N = T // m
    inp = synth.indexer_inputs(B, T, N, HI, dI, seed=HI * 10 + dI)
    q_pos = torch.arange(T, dtype=torch.int32).repeat(B, 1)
    _compare(inp.qI, inp.w, inp.kI, q_pos, m, K, N)


def test_several_tiles_ragged_and_large_k():
    """n_entries spans several 1024-entry score tiles with a ragged tail, with
    rows below, at and above K visible entries."""
    B, Tq, N, m, K = 2, 24, 5000 + 37, 4, 512
    inp = synth.indexer_inputs(B, Tq, N + 11, 4, 64, seed=3)
    pos = np.array([0, 2, 3, 4, 2047, 2048, 2051, 4 * 511, 4 * 512 - 1, 4 * 512, 4 * 513 - 1, 5000,
                    9000, 12000, 4 * N - 1, 4 * N, 4 * N + 500, 3, 7, 11, 4095, 4096, 20000, 19999])
    q_pos = torch.from_numpy(np.stack([pos, pos[::-1]]).astype(np.int32))
    _compare(inp.qI, inp.w, inp.kI, q_pos, m, K, N)


def test_ties_resolved_by_lower_index():
    """Keys drawn from {0, 1} codes only: scores take few values, so the K-th
    place is shared by many entries."""
    B, Tq, N, m, K = 1, 6, 3000, 4, 100
    g = torch.Generator().manual_seed(1)
    codes = torch.randint(0, 2, (B, N, 64), generator=g, dtype=torch.uint8)
    kI = (codes[..., 0::2] | (codes[..., 1::2] << 4)).contiguous()
    inp = synth.indexer_inputs(B, Tq, 1, 4, 64, seed=4)
    q_pos = torch.tensor([[4 * N - 1, 4 * N - 1, 1000, 400, 401, 4 * N - 1]], dtype=torch.int32)
    _compare(inp.qI, inp.w, kI, q_pos, m, K, N)


def test_all_equal_scores_take_prefix():
    B, Tq, N, m, K = 1, 3, 9000, 4, 512      # n_eq > the tie buffer: ordered scan path
    kI = torch.zeros((B, N, 32), dtype=torch.uint8)
    inp = synth.indexer_inputs(B, Tq, 1, 4, 64, seed=5)
    q_pos = torch.tensor([[4 * N - 1, 5000, 100]], dtype=torch.int32)
    gi, gs = _gpu_topk(inp.qI, inp.w, kI, q_pos, m, K, N)
    assert (gi[0, 0] == np.arange(K)).all() and (gi[0, 1] == np.arange(K)).all()
    assert (gi[0, 2, :25] == np.arange(25)).all() and (gi[0, 2, 25:] == -1).all()
    _compare(inp.qI, inp.w, kI, q_pos, m, K, N)


def test_k_extremes_and_empty_rows():
    B, Tq, N, m = 1, 5, 1500, 4
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=6)
    q_pos = torch.tensor([[0, 1, 2, 4 * N - 1, 3000]], dtype=torch.int32)
    for K in (1, 2048):
        _compare(inp.qI, inp.w, inp.kI, q_pos, m, K, N)


def test_bad_weight_is_reported():
    B, Tq, N = 1, 1, 64
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=7)
    w = inp.w.clone()
    w[0, 0, 0] = 0.3
    with pytest.raises(csa.CsaError) as e:
        _gpu_topk(inp.qI, w, inp.kI, torch.tensor([[4 * N - 1]], dtype=torch.int32), 4, 8, N)
    assert e.value.code == csa.CSA_ERR_INVALID


@pytest.mark.parametrize("B,N", [(16, 16384), (4, 262145)])
def test_decode_full_size(B, N):
    """Decode shapes of the 64K-context (16 x 16,384 entries) and 1M-context
    (4 x 262,145 entries) workloads: every query checked."""
    inp = synth.indexer_inputs(B, 1, N, 4, 64, seed=N, device="cuda")
    q_pos = torch.full((B, 1), 4 * N - 1, dtype=torch.int32)
    _compare(inp.qI.cpu(), inp.w.cpu(), inp.kI.cpu(), q_pos, 4, 512, N)


def test_prefill_full_size_sampled_rows():
    """128K prefill (131,072 queries x up to 32,768 entries), the launch the
    bench times; 1,024 rows checked bit-exact including the block edges."""
    T, m, K, N = 131072, 4, 512, 32768
    inp = synth.indexer_inputs(1, T, N, 4, 64, seed=11, device="cuda")
    q_pos = torch.arange(T, dtype=torch.int32, device="cuda")[None].contiguous()
    d = Dims(B=1, Tq=T, HI=4, dI=64, K=K, m=m, n_entries=N)
    idx = torch.empty((1, T, K), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, T, K), device="cuda")
    ws = torch.empty(csa.index_topk_workspace(d), dtype=torch.uint8, device="cuda")
    csa.index_topk(inp.qI, inp.w, inp.kI, q_pos, d, idx, sc, workspace=ws)
    csa.sync_status()
    del ws
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 4, 127, 128, 2047, 2048, 2051, 4 * 512 - 1, 4 * 512,
                                      T - 1, T - 2], rng.choice(T, 1010, replace=False)]))
    r = torch.from_numpy(rows).cuda()
    ri, rs = _oracle_topk(inp.qI[:, r].cpu(), inp.w[:, r].cpu(), inp.kI.cpu(),
                          torch.from_numpy(rows[None].astype(np.int32)), m, K, N)
    assert np.array_equal(idx[:, r].cpu().numpy(), ri)
    assert np.array_equal(sc[:, r].cpu().numpy().astype(np.float64), rs)


def test_negative_position_is_reported():
    B, Tq, N = 1, 2, 64
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=8)
    with pytest.raises(csa.CsaError) as e:
        _gpu_topk(inp.qI, inp.w, inp.kI, torch.tensor([[-5, 10]], dtype=torch.int32), 4, 8, N)
    assert e.value.code == csa.CSA_ERR_INVALID


def test_prefill_path_ties_and_large_k():
    """Many query rows (the prefill path): keys from {0, 1} codes give massive
    ties at the threshold; K = 2048 and a partial last tile of query rows."""
    g = torch.Generator().manual_seed(2)
    B, Tq, N, m = 2, 300, 3000, 4
    codes = torch.randint(0, 2, (B, N, 64), generator=g, dtype=torch.uint8)
    kI = (codes[..., 0::2] | (codes[..., 1::2] << 4)).contiguous()
    inp = synth.indexer_inputs(B, Tq, 1, 4, 64, seed=12)
    pos = torch.randint(0, 4 * N + 40, (B, Tq), generator=g, dtype=torch.int32)
    pos[0, :5] = torch.tensor([0, 3, 4 * N - 1, 4 * 100, 4 * 2048], dtype=torch.int32)
    for K in (100, 2048):
        _compare(inp.qI, inp.w, kI, pos, m, K, N)


def test_prefill_path_random_two_sequences():
    B, Tq, N, m, K = 2, 257, 6000, 4, 512
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=13)
    g = torch.Generator().manual_seed(3)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    _compare(inp.qI, inp.w, inp.kI, pos, m, K, N)
    inp2 = synth.indexer_inputs(B, Tq, N, 2, 64, seed=14)
    _compare(inp2.qI, inp2.w, inp2.kI, pos, m, 64, N)


def test_scan_collect_path():
    """64 decode rows over 20,000 entries: more than one CTA per SM pair can
    hold (8,192 entries each), so the two-kernel tensor-core path (per-slice
    scores and histograms, then the threshold and collection) runs."""
    B, Tq, N, m, K = 1, 64, 20000, 4, 512
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=21)
    g = torch.Generator().manual_seed(21)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    pos[0, :6] = torch.tensor([0, 4 * 512 - 1, 4 * 512, 4 * N - 1, 4 * N + 9, 4 * 5000], dtype=torch.int32)
    _compare(inp.qI, inp.w, inp.kI, pos, m, K, N)


@pytest.mark.parametrize("HI,dI", [(8, 32), (2, 32)])
def test_split_merge_path(HI, dI):
    """Few rows over >= 2,048 entries with an indexer shape the tensor-core
    paths do not take: per-slice candidates, then a merge per row."""
    B, Tq, N, m, K = 1, 16, 5000, 4, 512
    inp = synth.indexer_inputs(B, Tq, N, HI, dI, seed=22 + HI)
    g = torch.Generator().manual_seed(22)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    pos[0, :4] = torch.tensor([1, 4 * 512 - 1, 4 * 512 + 3, 4 * N - 1], dtype=torch.int32)
    _compare(inp.qI, inp.w, inp.kI, pos, m, K, N)


@pytest.mark.parametrize("K", [1, 37, 1024])
def test_prefill_streaming_path_k_range(K):
    """The >64-row streaming selection at the extremes of its k range, three
    sequences of a length that is not a multiple of the 128-query block, with
    rows below, at and above k visible entries."""
    B, Tq, N, m = 3, 333, 4100, 4
    inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed=40 + K)
    g = torch.Generator().manual_seed(K)
    pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    pos[0, :6] = torch.tensor([0, 3, 4 * K - 1, 4 * K, 4 * K + 3, 4 * N - 1], dtype=torch.int32)
    _compare(inp.qI, inp.w, inp.kI, pos, m, K, N)


def test_prefill_streaming_path_crowded_bins():
    """Keys drawn from a few codes give scores with few distinct values: the
    threshold bin overflows the candidate buffer, so the finer histogram
    levels run, down to exact ties taken in index order; one sequence has
    identical keys (every score equal)."""
    g = torch.Generator().manual_seed(9)
    B, Tq, N, m, K = 2, 200, 5000, 4, 300
    codes = torch.randint(0, 3, (B, N, 64), generator=g, dtype=torch.uint8)
    codes[1] = 2
    kI = (codes[..., 0::2] | (codes[..., 1::2] << 4)).contiguous()
    inp = synth.indexer_inputs(B, Tq, 1, 4, 64, seed=41)
    pos = torch.randint(4 * K, 4 * N + 40, (B, Tq), generator=g, dtype=torch.int32)
    _compare(inp.qI, inp.w, kI, pos, m, K, N)
