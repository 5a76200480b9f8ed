"""Pins for the oracle's number-format codecs against an independent library
(ml_dtypes, whose float8_e4m3fn / float4_e2m1fn follow the OCP definitions)
and against brute-force nearest-value search."""
import ml_dtypes
import numpy as np
import pytest

from oracle.formats import (E2M1_GRID, bf16_decode, e2m1_decode, e2m1_encode, e2m1_pack, e2m1_unpack, e4m3_decode,
                            e4m3_encode, e8m0_decode, mxfp4_quantize)

ALL = np.arange(256, dtype=np.uint8)


def test_e4m3_decode_matches_ml_dtypes_all_codes():
    ref = ALL.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = e4m3_decode(ALL)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    # sign of zero as well
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok]))
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


def _finite_values():
    v = e4m3_decode(ALL)
    return np.unique(v[~np.isnan(v)])


def test_e4m3_encode_roundtrips_every_code():
    finite = ALL[~np.isnan(e4m3_decode(ALL))]
    back = e4m3_encode(e4m3_decode(finite))
    assert np.array_equal(back, finite)


def _probe_values(rng):
    """fp32 probes (the encoder's inputs are fp32 ratios): every code value,
    every midpoint between neighbours and the fp32 numbers either side of it,
    log-uniform random magnitudes, and a few edge values."""
    vals = _finite_values().astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2.0).astype(np.float32)  # exact
    probes = [vals, mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(-np.inf))]
    mag = np.exp2(rng.uniform(-12, 9.2, 20000))
    probes.append((mag * np.where(rng.random(20000) < 0.5, -1, 1)).astype(np.float32))
    probes.append(np.array([0.0, -0.0, 2.0 ** -10, 2.0 ** -10 * 3, 447.99, 455.9, 463.99], np.float32))
    return np.concatenate(probes).astype(np.float64)


def test_e4m3_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(0)
    v = _probe_values(rng)
    v = v[np.abs(v) < 464.0]                  # ml_dtypes does not saturate beyond
    ref = v.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = e4m3_encode(v)
    assert np.array_equal(got, ref)


def test_e4m3_encode_is_nearest_even_bruteforce():
    """Independent of any library: nearest finite value by search, ties to the
    code with an even mantissa (even code pattern)."""
    rng = np.random.default_rng(1)
    v = _probe_values(rng)
    v = v[np.abs(v) < 448.0]
    codes = np.arange(0x7F, dtype=np.uint8)          # non-negative finite codes 0..0x7E
    mags = e4m3_decode(codes)
    a = np.abs(v)
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among ties pick the even code
    pick = np.where(cand & ((codes[None, :] & 1) == 0), codes[None, :], 255).min(axis=1)
    pick = np.where(cand.sum(axis=1) == 1, codes[np.argmax(cand, axis=1)], pick).astype(np.uint8)
    expect = pick | (np.signbit(v).astype(np.uint8) << 7)
    assert np.array_equal(e4m3_encode(v), expect)


def test_e4m3_encode_saturates():
    got = e4m3_encode(np.array([448.0, 464.0, 500.0, 1e30, -1e30, -449.0]))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    with pytest.raises(ValueError):
        e4m3_encode(np.array([np.nan]))


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(e2m1_decode(codes), ref)
    assert sorted(set(np.abs(ref))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_unpack_nibble_order():
    packed = np.array([[0x21, 0xF3]], dtype=np.uint8)
    assert e2m1_unpack(packed).tolist() == [[1, 2, 3, 15]]


def test_bf16_decode_matches_ml_dtypes():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 1 << 16, 5000, dtype=np.uint16)
    ref = bits.view(ml_dtypes.bfloat16).astype(np.float64)
    got = bf16_decode(bits)
    ok = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.array_equal(ref[ok], got[ok])


# ---------------------------------------------------------------- E2M1 encode, E8M0, MXFP4


def _e2m1_grid_inputs():
    """Every grid value, every midpoint (the ties), points one fp32 ulp either
    side of each midpoint, values past 6, and the negatives of all of them."""
    g = np.asarray(E2M1_GRID)
    mids = (g[:-1] + g[1:]) / 2
    pts = np.concatenate([g, mids, np.nextafter(mids.astype(np.float32), np.float32(0)).astype(np.float64),
                          np.nextafter(mids.astype(np.float32), np.float32(9)).astype(np.float64),
                          [6.5, 7.0, 7.999, 100.0, 1e-30, 0.1, 0.2499, 0.2501]])
    rng = np.random.default_rng(5)
    pts = np.concatenate([pts, rng.uniform(0, 7.99, 2000).astype(np.float32).astype(np.float64)])
    return np.concatenate([pts, -pts])


def test_e2m1_encode_matches_ml_dtypes():
    v = _e2m1_grid_inputs()
    ref = v.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(e2m1_encode(v), ref)


def test_e2m1_encode_is_nearest_even_bruteforce():
    v = _e2m1_grid_inputs()
    got = e2m1_encode(v)
    dec = e2m1_decode(got)
    grid = np.asarray(E2M1_GRID)
    for x, c, d in zip(v, got, dec):
        mag = min(abs(x), 6.0)
        dist = np.abs(grid - mag)
        best = np.flatnonzero(dist == dist.min())
        k = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert abs(d) == grid[k] and (c & 0x8) == (0x8 if np.signbit(x) else 0)


def test_e2m1_pack_inverts_unpack():
    c = np.random.default_rng(6).integers(0, 16, (5, 64)).astype(np.uint8)
    assert np.array_equal(e2m1_unpack(e2m1_pack(c)), c)


def test_e8m0_decode_matches_ml_dtypes():
    codes = np.arange(255, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(e8m0_decode(codes), ref)
    assert np.isnan(e8m0_decode(np.array([255], dtype=np.uint8)))[0]


def test_mxfp4_worked_block():
    """One block worked by hand: max |v| = 13 -> floor(log2 13) = 3 -> X = 1
    (scale code 128, 2^1); v / 2 = 3, -0.375, 0.125, 6.5, -0.25, 2.25, ...;
    codes 3 -> 0b0101, -0.375 -> -0.5 (0b1001), 0.125 -> 0, 6.5 -> 6 (0b0111),
    -0.25 -> -0 (tie to the even code, 0b1000), 2.25 -> 2 (0b0100)."""
    v = np.zeros((1, 32), dtype=np.float32)
    v[0, :6] = [6.0, -0.75, 0.25, 13.0, -0.5, 4.5]
    codes, scales = mxfp4_quantize(v)
    assert scales.tolist() == [[128]]
    assert e2m1_unpack(codes)[0, :6].tolist() == [0x5, 0x9, 0x0, 0x7, 0x8, 0x4]
    assert (e2m1_unpack(codes)[0, 6:] == 0).all()


def test_mxfp4_scale_range_and_error_bound():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((40, 128)) * np.exp2(rng.integers(-40, 40, (40, 1)))).astype(np.float32)
    x[3, 32:64] = 0.0                      # an all-zero block
    x[5, :32] = 1e-42                      # subnormal block
    codes, scales = mxfp4_quantize(x)
    X = scales.astype(np.int64) - 127
    blocks = x.astype(np.float64).reshape(40, 4, 32)
    amax = np.abs(blocks).max(-1)
    normal = amax >= 2.0 ** -125
    ratio = amax[normal] / np.exp2(X[normal])
    assert ((ratio >= 4) & (ratio < 8)).all()
    assert X[3, 1] == -127 and X[5, 0] == -127
    dq = e2m1_decode(e2m1_unpack(codes)).reshape(40, 4, 32) * np.exp2(X)[..., None]
    r = np.abs(blocks) / np.exp2(X)[..., None]
    # half a grid step below 4 (at most 1 in the scaled units), saturation above 6
    bound = np.where(r <= 6, np.where(r < 4, 0.5, 1.0), r - 6) * np.exp2(X)[..., None]
    assert (np.abs(dq - blocks) <= bound + 1e-300).all()
    assert (dq[3, 1] == 0).all()
