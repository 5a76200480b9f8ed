"""Pins for the oracle's number-format codecs against an independent library
(ml_dtypes, whose float8_e4m3fn / float4_e2m1fn follow the OCP definitions)
and against brute-force nearest-value search."""
import ml_dtypes
import numpy as np
import pytest

from oracle.formats import bf16_decode, e2m1_decode, e2m1_unpack, e4m3_decode, e4m3_encode

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
