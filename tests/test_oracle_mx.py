"""Pins of the block-scaled (MXFP4) indexer oracle and of the tie-tolerant
top-k check, against what the formats and the mathematics fix: the unit-
scale case is the exact integer indexer, exact rational arithmetic on tiny
inputs, an independent decode through ml_dtypes, and the invariance of a
product under moving a power of two from one factor to the other."""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from oracle import csa as ocsa
from oracle.formats import e2m1_decode, e2m1_unpack
from tests.parity import check_topk_tolerant


def _random_mx(rng, shape_rows, d, lo=100, hi=150):
    codes = rng.integers(0, 256, size=shape_rows + (d // 2,), dtype=np.uint8)
    scales = rng.integers(lo, hi, size=shape_rows + (d // 32,), dtype=np.uint8)
    return codes, scales


def test_unit_scales_reduce_to_the_exact_integer_indexer():
    rng = np.random.default_rng(0)
    B, Tq, H, N, d = 2, 5, 4, 40, 64
    qc, _ = _random_mx(rng, (B, Tq, H), d)
    kc, _ = _random_mx(rng, (B, N), d)
    w = rng.integers(0, 17, size=(B, Tq, H)).astype(np.float32) / 16
    ones_q = np.full((B, Tq, H, d // 32), 127, np.uint8)
    ones_k = np.full((B, N, d // 32), 127, np.uint8)
    s, mag = ocsa.indexer_scores_mx(qc, ones_q, w, kc, ones_k)
    assert np.array_equal(s * 64, ocsa.indexer_scores64(qc, w, kc).astype(np.float64))
    assert (mag >= s).all()


def test_scores_match_exact_fractions():
    rng = np.random.default_rng(1)
    B, Tq, H, N, d = 1, 2, 3, 6, 64
    qc, qs = _random_mx(rng, (B, Tq, H), d, lo=110, hi=140)
    kc, ks = _random_mx(rng, (B, N), d, lo=110, hi=140)
    w = rng.random((B, Tq, H)).astype(np.float32)
    s, mag = ocsa.indexer_scores_mx(qc, qs, w, kc, ks)
    qv = e2m1_decode(e2m1_unpack(qc))
    kv = e2m1_decode(e2m1_unpack(kc))
    for t in range(Tq):
        for n in range(N):
            tot = Fraction(0)
            absd = Fraction(0)
            for h in range(H):
                dot = Fraction(0)
                ad = Fraction(0)
                for j in range(d):
                    e = int(qs[0, t, h, j // 32]) + int(ks[0, n, j // 32]) - 254
                    p = Fraction(qv[0, t, h, j]) * Fraction(kv[0, n, j]) * Fraction(2) ** e
                    dot += p
                    ad += abs(p)
                wf = Fraction(float(w[0, t, h]))
                tot += wf * max(dot, Fraction(0))
                absd += wf * ad
            assert abs(Fraction(s[0, t, n]) - tot) <= abs(tot) * Fraction(1, 2 ** 50)
            assert abs(Fraction(mag[0, t, n]) - absd) <= absd * Fraction(1, 2 ** 50)


def test_values_match_ml_dtypes_decode():
    rng = np.random.default_rng(2)
    codes, scales = _random_mx(rng, (7,), 64, lo=90, hi=170)
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(7, 64)
    el = nib.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    ref = el * np.repeat(sc, 32, axis=-1)
    assert np.array_equal(ocsa.mx_values(codes, scales), ref)


def test_moving_a_power_of_two_between_factors_changes_nothing():
    rng = np.random.default_rng(3)
    B, Tq, H, N, d = 1, 3, 4, 30, 64
    qc, qs = _random_mx(rng, (B, Tq, H), d)
    kc, ks = _random_mx(rng, (B, N), d)
    w = rng.random((B, Tq, H)).astype(np.float32)
    s0, m0 = ocsa.indexer_scores_mx(qc, qs, w, kc, ks)
    a = np.array([5, -7], dtype=np.int64)     # per block
    s1, m1 = ocsa.indexer_scores_mx(qc, (qs + a).astype(np.uint8), w, kc, (ks - a).astype(np.uint8))
    assert np.array_equal(s0, s1) and np.array_equal(m0, m1)


def test_rejects_nan_scale_and_negative_weight():
    rng = np.random.default_rng(4)
    qc, qs = _random_mx(rng, (1, 1, 1), 64)
    kc, ks = _random_mx(rng, (1, 3), 64)
    w = np.ones((1, 1, 1), np.float32)
    bad = qs.copy()
    bad[..., 0] = 0xFF
    with pytest.raises(ValueError):
        ocsa.indexer_scores_mx(qc, bad, w, kc, ks)
    with pytest.raises(ValueError):
        ocsa.indexer_scores_mx(qc, qs, -w, kc, ks)


def _exact_topk(ref, nv, K):
    order = np.lexsort((np.arange(nv), -ref[:nv]))[: min(K, nv)]
    out = np.full(K, -1, np.int64)
    out[: order.size] = order
    return out


def test_tolerant_check_accepts_exact_and_near_tie_swaps():
    ref = np.array([[10.0, 9.0, 8.0, 7.9999999, 3.0, 2.0]])
    mag = np.full_like(ref, 10.0)
    nv = np.array([6])
    K = 4
    idx = _exact_topk(ref[0], 6, K)[None]
    assert check_topk_tolerant(idx, ref[:, idx[0]], ref, mag, nv, K, rtol=2 ** -12) == 0
    swap = np.array([[0, 1, 3, 4]])       # 4 (3.0) for 2 (8.0): not a near tie
    with pytest.raises(AssertionError, match="beats"):
        check_topk_tolerant(swap, None, ref, mag, nv, K, rtol=2 ** -12)
    # k = 3: entry 3 (7.9999999) listed instead of entry 2 (8.0), within the bounds
    near = np.array([[0, 1, 3]])
    assert check_topk_tolerant(near, np.array([[10.0, 9.0, 7.9999999]]), ref, mag, nv, 3) == 1


def test_tolerant_check_rejects_bad_lists():
    ref = np.array([[5.0, 4.0, 3.0, 2.0, 1.0]])
    mag = np.full_like(ref, 5.0)
    nv = np.array([3])
    with pytest.raises(AssertionError, match="padding"):
        check_topk_tolerant(np.array([[0, 1, 2, 3]]), None, ref, mag, nv, 4)
    with pytest.raises(AssertionError, match="outside"):
        check_topk_tolerant(np.array([[0, 1, 4, -1]]), None, ref, mag, nv, 4)
    with pytest.raises(AssertionError, match="repeated"):
        check_topk_tolerant(np.array([[0, 0, 1, -1]]), None, ref, mag, nv, 4)
    with pytest.raises(AssertionError, match="bound"):
        check_topk_tolerant(np.array([[0, 1, 2, -1]]), np.array([[5.0, 4.1, 3.0, 0.0]]), ref, mag, nv, 4)
    with pytest.raises(AssertionError, match="descending"):
        check_topk_tolerant(np.array([[1, 0, 2, -1]]), np.array([[4.0, 5.0, 3.0, 0.0]]), ref, mag, nv, 4)


def test_tolerant_check_on_oracle_output_with_bounded_perturbation():
    """Scores perturbed within the bound and re-ranked pass; the exact
    oracle order passes with zero swaps."""
    rng = np.random.default_rng(5)
    B, Tq, H, N, d, K = 1, 6, 4, 300, 64, 40
    qc, qs = _random_mx(rng, (B, Tq, H), d, lo=120, hi=130)
    kc, ks = _random_mx(rng, (B, N), d, lo=120, hi=130)
    w = rng.random((B, Tq, H)).astype(np.float32)
    s, mag = ocsa.indexer_scores_mx(qc, qs, w, kc, ks)
    nv = np.array([300, 250, 40, 39, 1, 120])
    ref = s[0]
    exact = np.stack([_exact_topk(ref[r], nv[r], K) for r in range(Tq)])
    ex_sc = np.where(exact >= 0, np.take_along_axis(ref, np.maximum(exact, 0), axis=1), 0.0)
    assert check_topk_tolerant(exact, ex_sc, ref, mag[0], nv, K) == 0
    noisy = ref + (rng.random(ref.shape) * 2 - 1) * 2 ** -21 * mag[0]
    pert = np.stack([_exact_topk(noisy[r], nv[r], K) for r in range(Tq)])
    pert_sc = np.where(pert >= 0, np.take_along_axis(noisy, np.maximum(pert, 0), axis=1), 0.0)
    check_topk_tolerant(pert, pert_sc, ref, mag[0], nv, K)
