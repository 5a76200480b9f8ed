"""Comparison rules shared by the GPU parity tests.

Tolerances (derived from the arithmetic; the numeric bars are the library's
contract):
* indexer scores and top-k indices: bit-exact (the scores are exact integers
  in units of 1/64 on both sides).
* pooled fp32 value of channel c: |gpu - ref| <= 1e-5 * A_c, where
  A_c = sum_i p_i |x_i| is the natural scale of a weighted sum (the fp32
  bound for m <= 128 terms is about (m + 3) * 2^-24 * A_c < 1e-5 * A_c).
* E4M3 codes: equal, except a flip to the NEIGHBOURING code where the
  oracle's fp32 ratio r = C/s lies within delta of the midpoint between the
  two codes; delta is what the pooled tolerance allows r to move:
  delta = 1e-5 * A_c / s + |r| * 1e-5 * A_amax / amax + 2^-22 |r|.
* scales: |gpu - ref| <= 1e-5 * A_amax / 448 + 2^-23 * ref.
* attention output (bf16): per query row and head, max_d |gpu - ref| <=
  1e-2 * max_d |ref|.
* log-sum-exp: |gpu - ref| <= 1e-4 (logits are exact products of bf16 and
  E4M3 values accumulated in fp32; exp2/log2 add a few ulp).
* block-scaled (MXFP4) indexer scores: |gpu - ref| <= MX_RTOL * mag with
  mag = sum_h w_h sum_j |q_hj k_j| (the oracle's second output).  The
  kernel's arithmetic: within a 32-element block the products share one
  power of two and their sum has at most 11 significant bits, exact in any
  fp32 accumulator; the tensor core adds the two scaled block sums with fp32
  accumulation (one rounding, at most 2^-24 of the magnitude), and the
  epilogue's weight-times-relu sum over at most 8 heads rounds once per
  head.  At most 9 roundings of 2^-24 * mag each: MX_RTOL = 2^-20 covers
  them with room (measured on B200: at most 1.3e-7 = 2^-22.9 of mag).
* block-scaled top-k (tie-tolerant): the k listed entries are distinct and
  visible, padded with -1, their reported scores within the score bound and
  non-increasing; and no left-out entry can beat a listed one: for every
  listed e and unlisted f, ref(e) + err(e) >= ref(f) - err(f).  Entries
  whose scores lie within the bounds of the k-th may therefore swap, and
  nothing else may.
"""
from __future__ import annotations

import numpy as np

from oracle import csa as ocsa
from oracle.formats import e4m3_decode

POOL_RTOL = 1e-5
OUT_RTOL = 1e-2
LSE_ATOL = 1e-4
MX_RTOL = 2.0 ** -20


def pooled_and_scale(x, z, m):
    """Oracle pooled values (fp64) and A = pool(|x|) for full blocks of x, z [B, T, D]."""
    ref = ocsa.compress(x, z, m)
    A = ocsa.compress(np.abs(np.asarray(x, dtype=np.float64)), z, m)
    return ref, A


def check_pooled(gpu, ref, A):
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    bad = err > POOL_RTOL * A + 1e-30
    assert not bad.any(), f"pooled mismatch at {np.argwhere(bad)[:5].tolist()}: max err/A {(err / A).max():.3g}"


def check_codes(gpu_codes, gpu_scales, ref_pooled, A):
    """Compare GPU codes/scales with the oracle's quantisation of its own pooled values."""
    ref_codes, ref_s = ocsa.quantize_entries(ref_pooled)
    r = ocsa.quantize_ratio(ref_pooled)
    gpu_codes = np.asarray(gpu_codes)
    gpu_scales = np.asarray(gpu_scales, dtype=np.float64)
    amax = np.abs(ref_pooled.astype(np.float32)).max(axis=-1).astype(np.float64)
    amax_ch = np.abs(ref_pooled.astype(np.float32)).argmax(axis=-1)
    A_amax = np.take_along_axis(A, amax_ch[..., None], axis=-1)[..., 0]
    s = ref_s.astype(np.float64)
    # scales
    tol_s = POOL_RTOL * A_amax / 448.0 + 2.0 ** -23 * s
    bad = np.abs(gpu_scales - s) > tol_s
    assert not bad.any(), f"scale mismatch at {np.argwhere(bad)[:5].tolist()}"
    # codes
    diff = gpu_codes != ref_codes
    n_flip = int(diff.sum())
    if n_flip:
        vg = e4m3_decode(gpu_codes[diff])
        vr = e4m3_decode(ref_codes[diff])
        rr = r[diff]
        finite = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
        lo = np.minimum(np.abs(vg), np.abs(vr))
        hi = np.maximum(np.abs(vg), np.abs(vr))
        # neighbours: no finite magnitude strictly between them, same sign unless one is zero
        between = ((finite[None, :] > lo[:, None]) & (finite[None, :] < hi[:, None])).any(axis=1)
        same_sign = (np.sign(vg) == np.sign(vr)) | (vg == 0) | (vr == 0)
        mid = (lo + hi) / 2.0
        Ad = np.broadcast_to(A, r.shape)[diff]
        sd = np.broadcast_to(s[..., None], r.shape)[diff]
        eps_s = np.broadcast_to((POOL_RTOL * A_amax / amax.clip(1e-300))[..., None], r.shape)[diff]
        delta = POOL_RTOL * Ad / sd + np.abs(rr) * eps_s + 2.0 ** -22 * np.abs(rr)
        ok = ~between & same_sign & (np.abs(np.abs(rr) - mid) <= delta)
        assert ok.all(), (f"{int((~ok).sum())} code mismatches are not near-midpoint flips, e.g. "
                          f"gpu={gpu_codes[diff][~ok][:5]} ref={ref_codes[diff][~ok][:5]} r={rr[~ok][:5]}")
    return n_flip


def check_attention(gpu_out_bf16, gpu_lse, ref_out, ref_lse):
    import torch
    g = gpu_out_bf16.float().cpu().numpy().astype(np.float64) if isinstance(gpu_out_bf16, torch.Tensor) \
        else np.asarray(gpu_out_bf16, dtype=np.float64)
    err = np.abs(g - ref_out).max(axis=-1)
    scale = np.abs(ref_out).max(axis=-1)
    bad = err > OUT_RTOL * scale
    assert not bad.any(), (f"attention mismatch at {np.argwhere(bad)[:5].tolist()}: "
                           f"worst err/max|ref| = {(err / scale).max():.3g}")
    if gpu_lse is not None:
        gl = gpu_lse.cpu().numpy().astype(np.float64) if hasattr(gpu_lse, "cpu") else np.asarray(gpu_lse)
        lerr = np.abs(gl - ref_lse)
        assert lerr.max() <= LSE_ATOL, f"lse mismatch: max err {lerr.max():.3g}"
    return float((err / scale).max())


def check_topk_tolerant(gpu_idx, gpu_score, ref_score, mag, n_vis, K, rtol=MX_RTOL):
    """Tie-tolerant check of one block of rows.

    gpu_idx int [R, K], gpu_score [R, K] (or None), ref_score / mag float64
    [R, N] from the oracle, n_vis [R].  Raises AssertionError naming the
    first violated rule; returns the number of rows whose list differs from
    the oracle's exact rank order (near-ties that swapped).
    """
    gpu_idx = np.asarray(gpu_idx)
    swapped = 0
    for r in range(gpu_idx.shape[0]):
        nv = int(n_vis[r])
        k = min(K, nv)
        g = gpu_idx[r]
        assert (g[k:] == -1).all(), f"row {r}: padding past {k} entries"
        sel = g[:k].astype(np.int64)
        assert ((sel >= 0) & (sel < nv)).all(), f"row {r}: an index outside the {nv} visible entries"
        assert np.unique(sel).size == k, f"row {r}: repeated index"
        ref = np.asarray(ref_score[r, :nv], dtype=np.float64)
        err = rtol * np.asarray(mag[r, :nv], dtype=np.float64)
        if gpu_score is not None:
            gs = np.asarray(gpu_score[r], dtype=np.float64)
            assert (np.abs(gs[:k] - ref[sel]) <= err[sel] + 1e-30).all(), f"row {r}: a score outside its bound"
            assert (np.diff(gs[:k]) <= 0).all(), f"row {r}: scores not in descending order"
            assert (gs[k:] == 0).all(), f"row {r}: padding score not 0"
        if k < nv:
            rest = np.ones(nv, dtype=bool)
            rest[sel] = False
            lo_sel = (ref[sel] + err[sel]).min()
            hi_rest = (ref[rest] - err[rest]).max()
            assert lo_sel >= hi_rest, (f"row {r}: a left-out entry beats a listed one "
                                       f"({hi_rest:.9g} > {lo_sel:.9g})")
        exact = np.lexsort((np.arange(nv), -ref))[:k]
        swapped += int(not np.array_equal(exact, sel))
    return swapped
