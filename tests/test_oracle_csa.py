"""Pins for the CPU oracle: worked examples derived by hand (tests/golden),
closed forms, invariants, brute force on tiny inputs and independent library
routines (scipy softmax / logsumexp, torch SDPA in fp64, Python sorting,
exact rational arithmetic).  None of them re-types the oracle's own formula."""
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

from oracle import csa
from oracle.formats import e2m1_decode, e4m3_decode, e4m3_encode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(a):
    return np.asarray(a, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def _e2m1_pack(vals):
    """Encode exact E2M1 values with ml_dtypes and pack two per byte."""
    c = np.asarray(vals, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------


def test_compress_worked_example():
    g = _load("compress_worked.json")
    x = np.array(g["x"])[None]   # [1, 4, 3]
    z = np.array(g["z"])[None]
    pooled = csa.compress(x, z, g["m"])[0, 0]
    np.testing.assert_allclose(pooled, g["pooled"], rtol=1e-14, atol=0)
    codes, s = csa.quantize_entries(pooled)
    assert codes.tolist() == g["codes"]
    assert abs(float(s) - g["scale"]) <= 1e-7 * g["scale"]


def test_pool_matches_scipy_softmax():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 5, 7, 9))
    z = rng.standard_normal((2, 5, 7, 9)) * 3
    ref = (scipy.special.softmax(z, axis=-2) * x).sum(axis=-2)
    np.testing.assert_allclose(csa.pool_blocks(x, z), ref, rtol=1e-13, atol=1e-15)


def test_pool_m1_is_identity():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 33, 16)).astype(np.float32)
    z = rng.standard_normal((2, 33, 16)).astype(np.float32)
    assert np.array_equal(csa.compress(x, z, 1), x.astype(np.float64))


def test_pool_equal_logits_is_mean_and_bounds_and_permutation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 128, 8))
    zc = np.broadcast_to(rng.standard_normal((3, 1, 8)), (3, 128, 8))
    np.testing.assert_allclose(csa.pool_blocks(x, zc), x.mean(axis=1), rtol=1e-12, atol=1e-14)
    z = rng.standard_normal((3, 128, 8))
    p = csa.pool_blocks(x, z)
    assert (p <= x.max(axis=1) + 1e-12).all() and (p >= x.min(axis=1) - 1e-12).all()
    perm = rng.permutation(128)
    np.testing.assert_allclose(csa.pool_blocks(x[:, perm], z[:, perm]), p, rtol=1e-12, atol=1e-14)


def test_pool_one_hot_logit_selects_token():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 8))
    z = rng.standard_normal((4, 8))
    z[2] += 40.0
    np.testing.assert_allclose(csa.pool_blocks(x, z), x[2], rtol=1e-15, atol=1e-15)


def test_compress_drops_partial_tail_block():
    x = np.arange(2 * 10 * 3, dtype=np.float64).reshape(2, 10, 3)
    assert csa.compress(x, np.zeros_like(x), 4).shape == (2, 2, 3)


# ---------------------------------------------------------------------------
# FP8 entries
# ---------------------------------------------------------------------------


def test_quantize_codes_are_nearest_and_amax_hits_448():
    rng = np.random.default_rng(7)
    C = rng.standard_normal((50, 64)) * np.exp(rng.uniform(-8, 4, (50, 1)))
    codes, s = csa.quantize_entries(C)
    amax_ch = np.abs(C.astype(np.float32)).argmax(axis=1)
    top = codes[np.arange(50), amax_ch]
    assert set((top & 0x7F).tolist()) == {0x7E}
    # nearest-value property vs an independent search over all finite codes
    r = csa.quantize_ratio(C)
    mags = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    dist = np.abs(np.abs(r)[..., None] - mags)
    best = dist.min(axis=-1)
    got = np.abs(e4m3_decode(codes))
    assert np.all(np.abs(np.abs(r) - got) <= best + 0.0)
    # dequantisation error within half a step of E4M3 (relative 2^-4) plus fp32 rounding
    deq = csa.dequantize(codes, s)
    err = np.abs(deq - C)
    bound = np.maximum(np.abs(C) * 2.0 ** -4, s[:, None] * 2.0 ** -10) + np.abs(C) * 2e-7
    assert (err <= bound).all()


def test_quantize_zero_entry():
    codes, s = csa.quantize_entries(np.zeros((2, 8)))
    assert (codes == 0).all() and (s == 1.0).all()


def test_quantize_scale_is_fp32_amax_over_448():
    rng = np.random.default_rng(8)
    C = rng.standard_normal((20, 32))
    _, s = csa.quantize_entries(C)
    amax = np.abs(C.astype(np.float32)).max(axis=1).astype(np.float64)
    np.testing.assert_allclose(s, amax / 448.0, rtol=1e-7)
    assert s.dtype == np.float32


# ---------------------------------------------------------------------------
# visibility and window
# ---------------------------------------------------------------------------


def test_visibility_bruteforce():
    for m in (1, 4, 128):
        for t in range(0, 600):
            brute = sum(1 for b in range(700) if b * m + m - 1 <= t)
            assert csa.n_visible(t, m) == brute
    assert csa.n_visible(10 ** 6, 4, n_entries=100) == 100


def test_window_positions_bruteforce():
    for W in (1, 32, 128):
        for t in (0, 1, 31, 32, 127, 128, 500):
            brute = [p for p in range(0, t + 1) if t - W < p <= t]
            assert csa.window_positions(t, W).tolist() == brute


# ---------------------------------------------------------------------------
# indexer and top-k
# ---------------------------------------------------------------------------


def test_indexer_worked_example():
    g = _load("indexer_worked.json")
    qI = _e2m1_pack(np.array(g["q"]))[None, None]          # [1,1,H,d/2]
    w = np.array(g["w"], dtype=np.float32)[None, None]
    kI = _e2m1_pack(np.array(g["k"]))[None]                  # [1,N,d/2]
    s64 = csa.indexer_scores64(qI, w, kI)[0, 0]
    assert (s64 / 64.0).tolist() == g["scores"]
    for q in g["queries"]:
        nv = csa.n_visible(q["t"], g["m"])
        assert nv == q["n_vis"]
        idx, sc = csa.topk(s64[None, None], np.array([[nv]]), g["K"])
        assert idx[0, 0].tolist() == q["topk"]
        assert sc[0, 0].tolist() == q["topk_scores"]


def _random_indexer(rng, B, Tq, N, H, d):
    vals = e2m1_decode(np.array([0, 1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15]))
    q = rng.choice(vals, (B, Tq, H, d))
    k = rng.choice(vals, (B, N, d))
    w = rng.integers(0, 17, (B, Tq, H)) / 16.0
    return q, k, w


def test_indexer_exact_against_fractions():
    rng = np.random.default_rng(9)
    q, k, w = _random_indexer(rng, 2, 3, 11, 3, 8)
    s64 = csa.indexer_scores64(_e2m1_pack(q), w.astype(np.float32), _e2m1_pack(k))
    for b in range(2):
        for t in range(3):
            for s in range(11):
                tot = Fraction(0)
                for h in range(3):
                    dot = sum(Fraction(q[b, t, h, j]) * Fraction(k[b, s, j]) for j in range(8))
                    tot += Fraction(w[b, t, h]) * max(dot, Fraction(0))
                assert Fraction(int(s64[b, t, s]), 64) == tot


def test_indexer_matches_float_einsum():
    rng = np.random.default_rng(10)
    q, k, w = _random_indexer(rng, 1, 40, 300, 4, 64)
    s64 = csa.indexer_scores64(_e2m1_pack(q), w.astype(np.float32), _e2m1_pack(k))
    dots = np.einsum("bthj,bsj->bths", q, k)
    ref = np.einsum("bth,bths->bts", w, np.maximum(dots, 0))
    assert np.array_equal(s64 / 64.0, ref)


def test_indexer_rejects_off_grid_weights():
    with pytest.raises(ValueError):
        csa.indexer_scores64(np.zeros((1, 1, 1, 2), np.uint8), np.full((1, 1, 1), 0.3, np.float32),
                             np.zeros((1, 3, 2), np.uint8))


def test_topk_matches_python_sort_and_is_maximal():
    rng = np.random.default_rng(11)
    B, Tq, N, K = 2, 30, 50, 7
    s64 = rng.integers(0, 6, (B, Tq, N))          # many ties
    nv = rng.integers(0, N + 1, (B, Tq))
    idx, sc = csa.topk(s64, nv, K)
    for b in range(B):
        for t in range(Tq):
            n = int(nv[b, t])
            ref = sorted(range(n), key=lambda s: (-int(s64[b, t, s]), s))[:K]
            got = idx[b, t].tolist()
            assert got[: len(ref)] == ref and all(v == -1 for v in got[len(ref):])
            chosen = set(ref)
            worst = min(((int(s64[b, t, s]), -s) for s in chosen), default=None)
            for s in range(n):
                if s not in chosen:
                    assert (int(s64[b, t, s]), -s) < worst


def test_topk_all_equal_gives_prefix():
    idx, _ = csa.topk(np.zeros((1, 1, 100), np.int64), np.array([[100]]), 16)
    assert idx[0, 0].tolist() == list(range(16))


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------


def test_attention_worked_examples():
    g = _load("attention_worked.json")
    for c in g["cases"]:
        out, lse = csa.attend_one(np.array([c["q"]]), np.array(c["rows"]))
        np.testing.assert_allclose(out[0], c["out"], rtol=1e-14)
        assert abs(lse[0] - c["lse"]) < 1e-14


def test_attend_one_matches_torch_sdpa_and_logsumexp():
    rng = np.random.default_rng(12)
    q = rng.standard_normal((8, 32)) * 0.3
    U = rng.standard_normal((70, 32))
    out, lse = csa.attend_one(q, U, scale=0.7)
    tq = torch.from_numpy(q)[None, :, None, :]        # [1, H, 1, D]
    tu = torch.from_numpy(U)[None, None].expand(1, 8, 70, 32)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tu, tu, scale=0.7)[0, :, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(0.7 * q @ U.T, axis=1), rtol=1e-13)


def test_attend_special_cases():
    rng = np.random.default_rng(13)
    U = rng.standard_normal((9, 16))
    out, _ = csa.attend_one(np.zeros((2, 16)), U)
    np.testing.assert_allclose(out, np.broadcast_to(U.mean(0), (2, 16)), rtol=1e-13, atol=1e-15)
    out, lse = csa.attend_one(rng.standard_normal((3, 16)), U[:1])
    np.testing.assert_allclose(out, np.broadcast_to(U[0], (3, 16)), rtol=1e-14)
    q = 200.0 * U[4:5] / np.linalg.norm(U[4])
    out, _ = csa.attend_one(q, U / np.linalg.norm(U, axis=1, keepdims=True))
    np.testing.assert_allclose(out[0], U[4] / np.linalg.norm(U[4]), atol=1e-12)
    out, _ = csa.attend_one(rng.standard_normal((4, 16)), U)
    assert (out <= U.max(0) + 1e-12).all() and (out >= U.min(0) - 1e-12).all()


def _tiny_chain(seed, T=96, m=4, K=5, W=8, H=3, D=16, HI=2, dI=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, T, D)).astype(np.float32)
    z = rng.standard_normal((1, T, D)).astype(np.float32)
    q, k, w = _random_indexer(rng, 1, T, T // m, HI, dI)
    qb = _bf16_bits(rng.standard_normal((1, T, H, D)) * 0.25)
    codes, s = csa.quantize_entries(csa.compress(x, z, m))
    entries = csa.dequantize(codes, s)
    win = csa.window_token_values(x)
    pos = np.arange(T)[None]
    s64 = csa.indexer_scores64(_e2m1_pack(q), w.astype(np.float32), _e2m1_pack(k))
    nv = csa.n_visible(pos, m, T // m)
    return dict(x=x, qb=qb, entries=entries, win=win, pos=pos, s64=s64, nv=nv, m=m, K=K, W=W)


def test_csa_with_large_k_equals_hca():
    c = _tiny_chain(14)
    K = c["entries"].shape[1]
    idx, _ = csa.topk(c["s64"], c["nv"], K)
    wv = lambda b, p: c["win"][b, p]
    o1, l1 = csa.attend(c["qb"], c["entries"], idx, wv, c["pos"], c["W"])
    o2, l2 = csa.hca_attend(c["qb"], c["entries"], wv, c["pos"], c["m"], c["W"])
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


def test_attend_union_bruteforce_with_sdpa():
    """Every query against an explicitly assembled key set, via torch SDPA."""
    c = _tiny_chain(15)
    idx, _ = csa.topk(c["s64"], c["nv"], c["K"])
    wv = lambda b, p: c["win"][b, p]
    out, lse = csa.attend(c["qb"], c["entries"], idx, wv, c["pos"], c["W"])
    q = c["qb"].view(ml_dtypes.bfloat16).astype(np.float64)
    for t in (0, 1, 3, 4, 7, 8, 40, 95):
        rows = [c["entries"][0, s] for s in range(c["entries"].shape[1])
                if s in set(idx[0, t].tolist())]
        rows += [c["win"][0, p] for p in range(0, t + 1) if p > t - c["W"]]
        U = torch.from_numpy(np.array(rows))
        tq = torch.from_numpy(q[0, t])[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq[None], U[None, None].expand(1, tq.shape[0], -1, -1),
            U[None, None].expand(1, tq.shape[0], -1, -1), scale=1.0)[0, :, 0].numpy()
        np.testing.assert_allclose(out[0, t], ref, rtol=1e-11, atol=1e-13)


def test_early_queries_see_only_window():
    c = _tiny_chain(16)
    idx, _ = csa.topk(c["s64"], c["nv"], c["K"])
    assert (idx[0, :3] == -1).all()          # t < m - 1: nothing compressed yet
    assert (idx[0, 3, 1:] == -1).all() and idx[0, 3, 0] == 0
