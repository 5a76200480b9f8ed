"""The seeded input generators follow the stated recipe: the workloads'
shapes, N(0,1) tokens and gate logits, N(0,1)·q_scale bf16 queries, E2M1
indexer codes uniform over the 15 distinct values (never -0), indexer
weights on the 1/16 grid of [0, 1], finite E4M3 cache bytes with scales in
[0.5, 1.5)/448, and determinism in (seed, tag)."""
import numpy as np
import pytest
import torch

import synth
from oracle.formats import e2m1_unpack, e4m3_decode

RECIPE = {
    # name: (kind, B, T, m, K, W, H, D, HI, dI, q_scale, steps)
    "tiny_prefill": ("prefill", 1, 512, 4, 16, 32, 4, 64, 2, 32, 1 / 8, 1),
    "csa_decode_64k": ("decode", 16, 65536, 4, 512, 128, 128, 512, 4, 64, 512 ** -0.5, 1),
    "hca_decode_1m": ("hca_decode", 16, 1048576, 128, 0, 128, 128, 512, 0, 0, 512 ** -0.5, 1),
    "csa_prefill_128k": ("prefill", 1, 131072, 4, 512, 128, 64, 512, 4, 64, 512 ** -0.5, 1),
    "csa_decode_1m_incremental": ("decode_incremental", 4, 1048576, 4, 512, 128, 128, 512, 4, 64, 512 ** -0.5, 64),
}


@pytest.mark.parametrize("name", sorted(RECIPE))
def test_workload_shapes(name):
    wl = synth.WORKLOADS[name]
    kind, B, T, m, K, W, H, D, HI, dI, qs, steps = RECIPE[name]
    assert (wl.kind, wl.B, wl.T, wl.m, wl.K, wl.W, wl.H, wl.D, wl.HI, wl.dI, wl.steps) == \
        (kind, B, T, m, K, W, H, D, HI, dI, steps)
    assert wl.q_scale == pytest.approx(qs)
    assert wl.N == T // m


def test_tokens_and_queries_moments():
    x, z = synth.tokens(2, 4096, 64, 0)
    for t in (x, z):
        assert t.dtype == torch.float32 and abs(float(t.mean())) < 0.01 and abs(float(t.std()) - 1) < 0.01
    assert not torch.equal(x, z)
    q = synth.queries(1, 256, 16, 512, 512 ** -0.5, 0)
    assert q.dtype == torch.bfloat16
    assert abs(float(q.float().std()) * 512 ** 0.5 - 1) < 0.02


def test_e2m1_codes_uniform_over_15_values():
    ind = synth.indexer_inputs(2, 64, 4096, 4, 64, 0)
    for packed in (ind.qI, ind.kI):
        c = e2m1_unpack(packed.numpy()).ravel()
        counts = np.bincount(c, minlength=16)
        assert counts[8] == 0                                   # no -0
        used = np.delete(counts, 8)
        assert (used > 0).all()
        expect = c.size / 15
        assert np.abs(used - expect).max() < 0.1 * expect


def test_indexer_weights_on_sixteenths():
    w = synth.indexer_weights(4, 4096, 4, 0)
    k = (w * 16).numpy()
    assert np.array_equal(k, np.round(k)) and k.min() == 0 and k.max() == 16
    assert len(np.unique(k)) == 17


def test_e4m3_cache_finite_and_scales_in_range():
    codes, scales = synth.e4m3_cache(2, 2048, 512, 0)
    c = codes.numpy()
    assert not np.isin(c, [0x7F, 0xFF]).any()
    assert np.isfinite(e4m3_decode(c)).all()
    assert len(np.unique(c)) == 254
    s = scales.numpy() * 448
    assert s.min() >= 0.5 and s.max() < 1.5


def test_deterministic_in_seed_and_tag():
    a = synth.tokens(1, 64, 64, 3)[0]
    assert torch.equal(a, synth.tokens(1, 64, 64, 3)[0])
    assert not torch.equal(a, synth.tokens(1, 64, 64, 4)[0])
    assert not torch.equal(a, synth.tokens(1, 64, 64, 3, tag="other")[0])
