"""CPU oracle for hybrid compressed attention (CSA / HCA) -- fp64, slow, plain.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import
this module.  It shares no code with the CUDA library and imports nothing
from it.  Inputs are numpy arrays; the caller produces them once with the
seeded generators in ``synth`` and hands the same bytes to both sides.

What the pages say (cited by page title and section)
----------------------------------------------------
* "DeepSeek V4とOpenCode" (hazakura.dev), section "衝撃1：CSA + HCA":
  CSA folds every 4 tokens into one entry, a Lightning Indexer picks the
  top-k entries at FP4 precision, and a 128-token sliding window keeps local
  context; HCA folds 128 tokens into one entry and attends densely.
* jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
  Attention (CSA)": the KV of m adjacent tokens becomes one entry (length
  1/m); each query scores the compressed entries with a lightweight indexer
  and a top-k selector keeps k of them (DSA); shared key-value MQA then runs
  over the k selected entries.  Section "Heavily Compressed Attention (HCA)":
  m' >> m, no sparse selection, dense attention; a sliding-window branch over
  recent uncompressed tokens runs alongside.
* "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
  (studioglobal.ai), section "アテンションのブレイクスルー：CSAとHCA": the
  compression is softmax-gated pooling, the indexer keeps the top 512
  compressed blocks per query, HCA compresses 128:1, and the window covers
  the latest 128 tokens.
* "DeepSeek V4 1M context window agent efficient inference" (ai-papers.net),
  section "ハイブリッドアテンションの仕組み": KV entries mostly in FP8, the
  indexer in FP4.

Readings where the pages are silent (this library's contract)
-------------------------------------------------------------
* Pooling: for block b and channel c, a softmax over the m gate logits of the
  block's tokens, taken independently per channel, weights the m token
  values.  Only full blocks become entries.
* FP8 entry: one fp32 scale per entry, s = amax_c |C| / 448 (s = 1 when the
  entry is all zero), codes = E4M3(C / s) rounded to nearest-even and
  saturated.  The scale and the division are taken in fp32, the kernel's
  precision, so both implementations make the same rounding decision on the
  same fp32 value.
* Causality: entry b is visible to the query at position t iff its last token
  b*m + m - 1 <= t, i.e. n_vis(t) = floor((t + 1) / m).
* Indexer score: score(t, s) = sum_h w[t,h] * ReLU(sum_j qI[t,h,j] * kI[s,j])
  with E2M1 qI, kI and w a multiple of 1/16 in [0, 1].  Every product of two
  E2M1 values is a multiple of 1/4, so 64 * score is an integer; the oracle
  computes that integer exactly.
* Block-scaled indexer (MXFP4 queries and keys, each 32-element block with
  its own E8M0 power-of-two scale): the same score, no longer an exact
  integer; a fixed-precision evaluation differs from it by at most a small
  multiple of the rounding unit times mag = sum_h w_h sum_j |q_hj k_j|, so
  entries whose scores lie that close to the k-th may swap places.
* Top-k: the K highest scores among visible entries, ties to the lower
  index; fewer than K visible -> all of them; rows are in rank order
  (score descending, index ascending) and padded with -1.
* Window: positions max(0, t-W+1) .. t, the query's own token included,
  stored per token as E4M3 with a per-token scale (pooling with m = 1).
* Attention: shared K = V; one softmax over the union of selected entries and
  window tokens, no de-duplication; logit = scale * q . v; output and the
  natural-log log-sum-exp per head.
* HCA: the selection is every visible entry.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_decode, e2m1_decode, e2m1_unpack, e4m3_decode, e4m3_encode

E4M3_MAX = 448.0


# --------------------------------------------------------------------------
# (1) softmax-gated pooling
# --------------------------------------------------------------------------


def pool_blocks(xb: np.ndarray, zb: np.ndarray) -> np.ndarray:
    """Softmax-gated pooling of token blocks.

    xb, zb: [..., m, D] token values and gate logits.  Returns [..., D]:
    C[c] = sum_i exp(z_i,c - max_i z_i,c) * x_i,c / sum_i exp(z_i,c - max_i z_i,c).
    Page: studioglobal.ai, "アテンションのブレイクスルー：CSAとHCA" (softmax-gated
    pooling, 4x along the sequence); hazakura.dev "衝撃1" (m = 4, m' = 128).
    """
    x = np.asarray(xb, dtype=np.float64)
    z = np.asarray(zb, dtype=np.float64)
    mx = z.max(axis=-2, keepdims=True)
    e = np.exp(z - mx)
    return (e * x).sum(axis=-2) / e.sum(axis=-2)


def compress(x: np.ndarray, z: np.ndarray, m: int) -> np.ndarray:
    """Pool every full block of m tokens of x, z [B, T, D] -> [B, T // m, D]."""
    x = np.asarray(x)
    B, T, D = x.shape
    n = T // m
    xb = np.asarray(x, dtype=np.float64)[:, : n * m].reshape(B, n, m, D)
    zb = np.asarray(z, dtype=np.float64)[:, : n * m].reshape(B, n, m, D)
    return pool_blocks(xb, zb)


# --------------------------------------------------------------------------
# FP8 entry quantisation (decision taken in fp32)
# --------------------------------------------------------------------------


def quantize_entries(pooled: np.ndarray):
    """Quantise pooled entries [..., D] to (codes u8 [..., D], scales f32 [...]).

    The pooled value is first rounded to fp32 (the kernel's working type);
    amax, the scale amax/448 and the ratio C/s are then formed with IEEE fp32
    operations, and the ratio is rounded to E4M3 exactly.
    Page: ai-papers.net "ハイブリッドアテンションの仕組み" (KV mostly FP8).
    """
    c32 = np.asarray(pooled, dtype=np.float64).astype(np.float32)
    amax = np.abs(c32).max(axis=-1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    r = (c32 / s[..., None]).astype(np.float32)
    codes = e4m3_encode(r.astype(np.float64))
    return codes, s


def quantize_ratio(pooled: np.ndarray) -> np.ndarray:
    """The pre-rounding fp32 ratio C/s of ``quantize_entries`` (for tolerances)."""
    c32 = np.asarray(pooled, dtype=np.float64).astype(np.float32)
    amax = np.abs(c32).max(axis=-1)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    return (c32 / s[..., None]).astype(np.float32).astype(np.float64)


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """E4M3 codes [..., D] times their per-entry fp32 scale [...] -> float64."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------
# causal visibility
# --------------------------------------------------------------------------


def n_visible(t, m: int, n_entries: int | None = None):
    """Number of compressed entries visible at query position t: floor((t+1)/m).

    Entry b covers tokens [b*m, b*m + m) and is visible iff b*m + m - 1 <= t.
    When the cache holds fewer entries (n_entries), the count is capped.
    """
    t = np.asarray(t, dtype=np.int64)
    v = (t + 1) // m
    if n_entries is not None:
        v = np.minimum(v, n_entries)
    return v


# --------------------------------------------------------------------------
# (2) Lightning Indexer, exact integer form
# --------------------------------------------------------------------------


def indexer_scores64(qI_packed, w, kI_packed) -> np.ndarray:
    """64 * score for every (query, entry) pair, as exact int64.

    qI_packed: u8 [B, Tq, H_I, d_I/2]  (E2M1, two per byte)
    w:         f32 [B, Tq, H_I]        (multiples of 1/16 in [0, 1])
    kI_packed: u8 [B, N, d_I/2]
    returns    int64 [B, Tq, N] = sum_h (16 w_h) * max(0, sum_j (2 q_hj)(2 k_j)).
    Pages: jiwasawa "Compressed Sparse Attention (CSA)" (indexer scores the
    compressed entries per query), hazakura.dev "衝撃1" (FP4 precision).
    """
    qi = np.rint(2.0 * e2m1_decode(e2m1_unpack(qI_packed))).astype(np.int64)  # [B,Tq,H,d]
    ki = np.rint(2.0 * e2m1_decode(e2m1_unpack(kI_packed))).astype(np.int64)  # [B,N,d]
    w = np.asarray(w, dtype=np.float64)
    w16 = np.rint(16.0 * w)
    if not np.array_equal(w16, 16.0 * w) or (w16 < 0).any():
        raise ValueError("indexer weights must be non-negative multiples of 1/16")
    w16 = w16.astype(np.int64)
    B, Tq, H, d = qi.shape
    N = ki.shape[1]
    out = np.zeros((B, Tq, N), dtype=np.int64)
    for b in range(B):
        # integer inner products, |q.k| <= 12*12*d: float64 matmul is exact here
        dots = np.rint(qi[b].reshape(Tq * H, d).astype(np.float64) @ ki[b].T.astype(np.float64))
        dots = dots.astype(np.int64).reshape(Tq, H, N)
        out[b] = (w16[b][:, :, None] * np.maximum(dots, 0)).sum(axis=1)
    return out


# --------------------------------------------------------------------------
# (2b) Lightning Indexer on block-scaled FP4 (MXFP4) queries and keys
# --------------------------------------------------------------------------


def mx_values(packed, scale_codes) -> np.ndarray:
    """MXFP4 rows to float64: element j of a row is its E2M1 value times
    2**(E8M0 code of block j // 32 - 127).

    packed: u8 [..., d/2]; scale_codes: u8 [..., d/32].  Exact in float64.
    Pages: studioglobal.ai "FP4/FP8混合精度" (MXFP4, two values per byte);
    jiwasawa "限界を押し広げるインフラストラクチャの最適化" (FP4 on the
    indexer's QK path).
    """
    v = e2m1_decode(e2m1_unpack(packed))
    sc = np.asarray(scale_codes).astype(np.int64)
    if (sc == 0xFF).any():
        raise ValueError("E8M0 code 0xFF (NaN) is not a scale")
    f = np.exp2((sc - 127).astype(np.float64))
    return v * np.repeat(f, 32, axis=-1)


def indexer_scores_mx(qI_packed, qI_scales, w, kI_packed, kI_scales):
    """Indexer scores on MXFP4 queries and keys, and the magnitude their
    rounding error scales with.

    qI_packed u8 [B, Tq, H_I, d_I/2], qI_scales u8 [B, Tq, H_I, d_I/32];
    w f32 [B, Tq, H_I] (non-negative); kI_packed u8 [B, N, d_I/2],
    kI_scales u8 [B, N, d_I/32].
    Returns float64 [B, Tq, N] pairs (score, mag):
        score = sum_h w_h * max(0, sum_j q_hj k_j)
        mag   = sum_h w_h * sum_j |q_hj k_j|
    Within one 32-element block every product is a multiple of the same
    power of two and the block's sum is exact in float64; only the sum over
    blocks and heads rounds, at float64 precision.  Pages: jiwasawa
    "Compressed Sparse Attention (CSA)" (the indexer's score),
    "限界を押し広げるインフラストラクチャの最適化" (FP4 QK path);
    studioglobal.ai "FP4/FP8混合精度" (MXFP4).
    """
    q = mx_values(qI_packed, qI_scales)          # [B, Tq, H, d]
    k = mx_values(kI_packed, kI_scales)          # [B, N, d]
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    if (w < 0).any() or not np.isfinite(w).all():
        raise ValueError("indexer weights must be finite and non-negative")
    B, Tq, H, d = q.shape
    N = k.shape[1]
    score = np.zeros((B, Tq, N))
    mag = np.zeros((B, Tq, N))
    for b in range(B):
        qq = q[b].reshape(Tq * H, d)
        dots = (qq @ k[b].T).reshape(Tq, H, N)
        absd = (np.abs(qq) @ np.abs(k[b]).T).reshape(Tq, H, N)
        score[b] = (w[b][:, :, None] * np.maximum(dots, 0.0)).sum(axis=1)
        mag[b] = (w[b][:, :, None] * absd).sum(axis=1)
    return score, mag


# --------------------------------------------------------------------------
# (3) top-k with ties to the lower index
# --------------------------------------------------------------------------


def topk(score64: np.ndarray, n_vis: np.ndarray, K: int):
    """Per query, the K best visible entries in rank order, padded with -1.

    score64: int64 [B, Tq, N]; n_vis: [B, Tq] visible counts.
    Returns (idx int32 [B, Tq, K], score float64 [B, Tq, K] (score64/64, 0 for pads)).
    Rank order is score descending, then index ascending.  Pages: jiwasawa
    "Compressed Sparse Attention (CSA)" (top-k selector), studioglobal.ai
    "アテンションのブレイクスルー" (top 512 compressed blocks per query).
    """
    B, Tq, N = score64.shape
    idx = np.full((B, Tq, K), -1, dtype=np.int32)
    sc = np.zeros((B, Tq, K), dtype=np.float64)
    for b in range(B):
        for t in range(Tq):
            nv = int(n_vis[b, t])
            s = score64[b, t, :nv]
            order = np.lexsort((np.arange(nv), -s))   # primary -score, then index
            take = order[: min(K, nv)]
            idx[b, t, : take.size] = take
            sc[b, t, : take.size] = s[take] / 64.0
    return idx, sc


# --------------------------------------------------------------------------
# (4)/(5) shared-KV multi-query attention over selection + window
# --------------------------------------------------------------------------


def window_positions(t: int, W: int) -> np.ndarray:
    """Positions of the sliding window for a query at t: max(0, t-W+1) .. t."""
    return np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)


def attend_one(q: np.ndarray, U: np.ndarray, scale: float = 1.0):
    """One query: q [H, D] (float64), U [n, D] values (K = V).

    Returns (out [H, D], lse [H]) with one softmax over the n rows of U.
    Page: jiwasawa "Compressed Sparse Attention (CSA)" (shared key-value MQA).
    """
    S = scale * (q @ U.T)                       # [H, n]
    mx = S.max(axis=1, keepdims=True)
    e = np.exp(S - mx)
    l = e.sum(axis=1, keepdims=True)
    out = (e @ U) / l
    lse = (mx + np.log(l))[:, 0]
    return out, lse


def attend(q_bits, entries, sel, win_vals, q_pos, W: int, scale: float = 1.0):
    """Sparse attention for every query.

    q_bits:   u16 [B, Tq, H, D] bf16 patterns of the queries
    entries:  f64 [B, N, D] dequantised compressed entries
    sel:      int [B, Tq, K] selected entry indices (-1 = unused)
    win_vals: callable (b, positions) -> f64 [n, D] dequantised window tokens
    q_pos:    int [B, Tq] query positions
    Returns (out f64 [B, Tq, H, D], lse f64 [B, Tq, H]).
    """
    q = bf16_decode(q_bits)
    B, Tq, H, D = q.shape
    out = np.zeros((B, Tq, H, D))
    lse = np.zeros((B, Tq, H))
    for b in range(B):
        for i in range(Tq):
            t = int(q_pos[b, i])
            s = np.asarray(sel[b, i])
            s = s[s >= 0]
            U = np.concatenate([entries[b, s], win_vals(b, window_positions(t, W))], axis=0)
            out[b, i], lse[b, i] = attend_one(q[b, i], U, scale)
    return out, lse


def hca_selection(q_pos, m: int, n_entries: int):
    """Dense HCA selection: every visible entry, as an index list per query."""
    q_pos = np.asarray(q_pos)
    nv = n_visible(q_pos, m, n_entries)
    width = max(int(nv.max()), 1) if nv.size else 1
    sel = np.full(q_pos.shape + (width,), -1, dtype=np.int64)
    for pos in np.ndindex(*q_pos.shape):
        sel[pos][: nv[pos]] = np.arange(nv[pos])
    return sel


def hca_attend(q_bits, entries, win_vals, q_pos, m: int, W: int, scale: float = 1.0):
    """HCA: attention over all visible compressed entries plus the window.

    Pages: jiwasawa "Heavily Compressed Attention (HCA)" (no sparse selection,
    dense), hazakura.dev "衝撃1" (m' = 128).
    """
    sel = hca_selection(q_pos, m, entries.shape[1])
    return attend(q_bits, entries, sel, win_vals, q_pos, W, scale)


# --------------------------------------------------------------------------
# convenience: window tokens from raw inputs
# --------------------------------------------------------------------------


def window_token_values(x_tokens: np.ndarray) -> np.ndarray:
    """Dequantised window tokens from raw token values x [..., D].

    A window token is a pooled block of one token (the softmax over a single
    logit is 1), stored as E4M3 with its own scale.
    """
    codes, s = quantize_entries(np.asarray(x_tokens, dtype=np.float64))
    return dequantize(codes, s)
