"""GPU parity of csa_compress against the oracle (softmax-gated pooling and
FP8 quantisation), through the C ABI."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from oracle import csa as ocsa
from tests import parity

pytestmark = pytest.mark.gpu


def _run(B, T, D, m, seed, ring_cap=0, dst_first=0, cap=None, scale=1.0):
    x, z = synth.tokens(B, T, D, seed)
    if scale != 1.0:
        x = x * scale
    n = T // m
    cap = cap or (dst_first + n if ring_cap == 0 else ring_cap)
    xg, zg = x.cuda(), z.cuda()
    codes = torch.full((B, cap, D), 0x55, dtype=torch.uint8, device="cuda")
    scales = torch.full((B, cap), -7.0, device="cuda")
    pooled = torch.empty((B, n, D), device="cuda")
    csa.compress(xg, zg, m, codes, scales, dst_first=dst_first, ring_cap=ring_cap, pooled=pooled)
    csa.sync_status()
    return x.numpy(), z.numpy(), codes.cpu().numpy(), scales.cpu().numpy(), pooled.cpu().numpy()


@pytest.mark.parametrize("B,T,D,m", [(1, 512, 64, 4), (2, 2051, 512, 4), (3, 777, 512, 1),
                                     (2, 128 * 9 + 77, 512, 128), (1, 1000, 128, 7), (2, 64, 256, 4),
                                     (2, 700, 64, 32), (1, 300, 256, 16), (2, 600, 512, 17)])
def test_compress_parity(B, T, D, m):
    x, z, codes, scales, pooled = _run(B, T, D, m, seed=B * 1000 + T + m)
    n = T // m
    ref, A = parity.pooled_and_scale(x, z, m)
    parity.check_pooled(pooled, ref, A)
    flips = parity.check_codes(codes[:, :n], scales[:, :n], ref, A)
    assert flips <= max(2, codes[:, :n].size // 10000)


def test_compress_m1_is_bit_exact_window():
    """m = 1 stores single tokens: pooling is the identity on both sides, so
    codes and scales must agree bit for bit."""
    x, z, codes, scales, pooled = _run(2, 300, 512, 1, seed=5)
    assert np.array_equal(pooled, x)
    ref_codes, ref_s = ocsa.quantize_entries(x.astype(np.float64))
    assert np.array_equal(codes, ref_codes)
    assert np.array_equal(scales, ref_s)


def test_compress_ring_and_offset_slots():
    B, T, D, W = 2, 50, 64, 16
    x, z, codes, scales, _ = _run(B, T, D, 1, seed=9, ring_cap=W, dst_first=1000)
    ref_codes, ref_s = ocsa.quantize_entries(x.astype(np.float64))
    for p in range(T - W, T):          # the last W tokens survive in the ring
        slot = (1000 + p) % W
        assert np.array_equal(codes[:, slot], ref_codes[:, p])
        assert np.array_equal(scales[:, slot], ref_s[:, p])
    x, z, codes, scales, _ = _run(B, 40, D, 4, seed=10, dst_first=3, cap=20)
    ref_codes, _ = ocsa.quantize_entries(ocsa.compress(x, z, 4))
    # untouched slots keep their fill bytes
    assert (codes[:, :3] == 0x55).all() and (codes[:, 13:] == 0x55).all() and (scales[:, 13:] == -7).all()
    assert (codes[:, 3:13] != 0x55).any()


def test_compress_edge_values():
    """All-zero entries (scale 1, codes 0), huge and tiny magnitudes."""
    B, T, D = 1, 16, 64
    x = torch.zeros(B, T, D)
    x[0, 4:8] = 1e30
    x[0, 8:12] = 1e-30
    x[0, 12:16, :32] = -3.0
    z = torch.zeros(B, T, D)
    codes = torch.empty((B, 4, D), dtype=torch.uint8, device="cuda")
    scales = torch.empty((B, 4), device="cuda")
    csa.compress(x.cuda(), z.cuda(), 4, codes, scales)
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    ref_codes, ref_s = ocsa.quantize_entries(ocsa.compress(x.numpy(), z.numpy(), 4))
    assert np.array_equal(c, ref_codes) and np.array_equal(s, ref_s)
    assert (c[0, 0] == 0).all() and s[0, 0] == 1.0


def test_compress_full_hca_config_sampled():
    """1M-token HCA context (16 x 1,048,576 x 512, m = 128): the launch the
    bench's cache build uses; 256 sampled blocks per sequence checked."""
    B, T, D, m = 16, 1 << 20, 512, 128
    x = synth.normal((B, T, D), 0, "hca:x", "cuda")
    z = synth.normal((B, T, D), 0, "hca:z", "cuda")
    n = T // m
    codes = torch.empty((B, n, D), dtype=torch.uint8, device="cuda")
    scales = torch.empty((B, n), device="cuda")
    pooled = torch.empty((B, n, D), device="cuda")
    csa.compress(x, z, m, codes, scales, pooled=pooled)
    csa.sync_status()
    rng = np.random.default_rng(0)
    blocks = np.concatenate([[0, n - 1], rng.choice(np.arange(1, n - 1), 254, replace=False)])
    for b in (0, 7, 15):
        bl = torch.from_numpy(blocks).cuda()
        tok = (bl[:, None] * m + torch.arange(m, device="cuda")[None]).reshape(-1)
        xs = x[b, tok].reshape(len(blocks), m, D).cpu().numpy()
        zs = z[b, tok].reshape(len(blocks), m, D).cpu().numpy()
        ref = ocsa.pool_blocks(xs, zs)
        A = ocsa.pool_blocks(np.abs(xs.astype(np.float64)), zs)
        parity.check_pooled(pooled[b, bl].cpu().numpy(), ref, A)
        parity.check_codes(codes[b, bl].cpu().numpy(), scales[b, bl].cpu().numpy(), ref, A)
    del x, z
    torch.cuda.empty_cache()


def _ew_pair(B, T, D, m, cap, wcap, dst_first=0, ring=0, win_first=0, win_ring=0, seed=0, pooled=False):
    """csa_compress_ew against csa_compress (entries) + csa_compress with m = 1
    (window), on sentinel-filled outputs: every byte equal."""
    x, z = synth.tokens(B, T, D, seed, device="cuda")
    outs = []
    for fused in (True, False):
        codes = torch.full((B, cap, D), 0xA5, dtype=torch.uint8, device="cuda")
        scales = torch.full((B, cap), -3.0, device="cuda")
        wc = torch.full((B, wcap, D), 0x5A, dtype=torch.uint8, device="cuda")
        ws = torch.full((B, wcap), -5.0, device="cuda")
        pl = torch.full((B, T // m, D), -7.0, device="cuda") if pooled else None
        if fused:
            csa.compress_ew(x, z, m, codes, scales, wc, ws, dst_first=dst_first, ring_cap=ring, win_first=win_first,
                            win_ring_cap=win_ring, pooled=pl)
        else:
            csa.compress(x, z, m, codes, scales, dst_first=dst_first, ring_cap=ring, pooled=pl)
            csa.compress(x, z, 1, wc, ws, dst_first=win_first, ring_cap=win_ring)
        csa.sync_status()
        outs.append([t.cpu() for t in (codes, scales, wc, ws) + ((pl,) if pooled else ())])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,T,D,m", [(2, 1030, 512, 4), (3, 64, 64, 2), (1, 96, 1024, 8), (2, 40, 128, 4)])
def test_compress_ew_equals_two_passes(B, T, D, m):
    """Entries and window in one pass: bit-identical to the two calls, with a
    ragged tail of tokens that enter only the window, and the pooled output."""
    _ew_pair(B, T, D, m, cap=T // m + 3, wcap=T + 2, seed=B * 7 + m, pooled=True)


def test_compress_ew_rings_and_offsets():
    """Decode-style appends: entries at an offset, the window as a ring that
    wraps, and a window ring smaller than the call (only its last tokens
    survive)."""
    _ew_pair(3, 8, 512, 4, cap=200, wcap=16, dst_first=100, win_first=30, win_ring=16, seed=1)
    _ew_pair(2, 12, 512, 4, cap=40, wcap=5, dst_first=7, win_first=3, win_ring=5, seed=2)
    _ew_pair(2, 16, 512, 4, cap=3, wcap=64, dst_first=1, ring=3, win_first=0, seed=3)   # entry ring too


@pytest.mark.parametrize("m", [1, 16])
def test_compress_ew_unfused_shapes(m):
    """m outside the fused range runs the two passes inside the call."""
    _ew_pair(2, 64, 512, m, cap=64 // m + 1, wcap=70, seed=m)


@pytest.mark.parametrize("B,T,D", [(2, 128 * 3 + 50, 512), (1, 256, 64), (3, 128, 256)])
def test_compress_ew_m128_equals_two_passes(B, T, D):
    """m' = 128 (the HCA block): entries and window in one channel-split
    cluster pass, bit-identical to the two calls (including a ragged tail of
    window-only tokens and the pooled output)."""
    _ew_pair(B, T, D, 128, cap=T // 128 + 2, wcap=T + 3, seed=B + T, pooled=True)


def test_compress_ew_m128_rings():
    """The HCA append: one 128-token block per sequence at an entry offset,
    its tokens into a window ring smaller than the call (only the last ring
    slots' tokens survive) and an entry ring that wraps."""
    _ew_pair(2, 128, 512, 128, cap=50, wcap=100, dst_first=40, win_first=7, win_ring=100, seed=11)
    _ew_pair(2, 384, 512, 128, cap=2, wcap=128, dst_first=1, ring=2, win_first=0, win_ring=128, seed=12)
