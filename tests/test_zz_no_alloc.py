"""The allocation-free indexer entry point (csa_index_topk_noalloc), called
through the C ABI.

Callers that cannot allocate device memory (allocator hooks, runtimes that
plan all memory at load time, plug-ins handed only their inputs and outputs)
use this entry point; its scratch is a fixed array inside the library.  Calls
in a row with different inputs, each taking a different indexer path through
the same scratch, must each give exactly the oracle's indices and scores and
the workspace version's (csa_index_topk) results: both are exact, so every
comparison is bit-exact.  This file is collected last so that a run stopping
at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims
from oracle import csa as ocsa

pytestmark = pytest.mark.gpu


def _with_workspace(inp, q_pos, d):
    idx = torch.empty((d.B, d.Tq, d.K), dtype=torch.int32, device="cuda")
    sc = torch.empty((d.B, d.Tq, d.K), device="cuda")
    ws = torch.empty(csa.index_topk_workspace(d), dtype=torch.uint8, device="cuda")
    csa.index_topk(inp.qI, inp.w, inp.kI, q_pos, d, idx, sc, workspace=ws)
    return idx, sc


def _noalloc(inp, q_pos, d):
    idx = torch.full((d.B, d.Tq, d.K), -9, dtype=torch.int32, device="cuda")
    sc = torch.full((d.B, d.Tq, d.K), -9.0, device="cuda")
    rc = csa.lib().csa_index_topk_noalloc(
        inp.qI.data_ptr(), inp.w.data_ptr(), inp.kI.data_ptr(), q_pos.data_ptr(), ctypes.byref(d),
        idx.data_ptr(), sc.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, csa.lib().csa_last_error().decode()
    return idx, sc


def _oracle(inp, q_pos, d):
    s64 = ocsa.indexer_scores64(inp.qI.cpu().numpy(), inp.w.cpu().numpy(), inp.kI[:, :d.n_entries].cpu().numpy())
    nv = ocsa.n_visible(q_pos.cpu().numpy().astype(np.int64), d.m, d.n_entries)
    return ocsa.topk(s64, nv, d.K)


# (B, Tq, entries, query position or None for random ones, seed); consecutive
# calls take different paths through the one scratch array:
#   16 x 1 at 16,384 entries: the one-launch decode kernel (64K-context decode shape)
#   64 x 1 at 20,000 entries: the two-kernel tensor-core path (its counters live in the scratch)
#   3 x 40 at 5,000 entries, random positions: the one-launch decode kernel, 120 rows of ragged visibility
#   1 x 300 at 2,500 entries: the prefill tensor-core path
SHAPES = [(16, 1, 16384, 65535, 1), (64, 1, 20000, 79999, 4), (3, 40, 5000, None, 2), (1, 300, 2500, None, 5),
          (16, 1, 16384, 65535, 6)]


def test_noalloc_matches_oracle_and_workspace_version_in_a_row():
    for B, Tq, N, pos, seed in SHAPES:
        inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed, device="cuda")
        if pos is None:
            q_pos = torch.randint(0, 4 * N + 8, (B, Tq), generator=torch.Generator().manual_seed(seed),
                                  dtype=torch.int32).cuda()
        else:
            q_pos = torch.full((B, Tq), pos, dtype=torch.int32, device="cuda")
        d = Dims(B=B, Tq=Tq, HI=4, dI=64, K=512, m=4, n_entries=N)
        assert csa.index_topk_workspace(d) <= 8 << 20
        gi, gs = _noalloc(inp, q_pos, d)
        ri, rs = _with_workspace(inp, q_pos, d)
        torch.cuda.synchronize()
        oi, osc = _oracle(inp, q_pos, d)
        assert np.array_equal(gi.cpu().numpy(), oi), (B, Tq, N)
        assert np.array_equal(gs.cpu().numpy().astype(np.float64), osc), (B, Tq, N)
        assert torch.equal(gi, ri) and torch.equal(gs, rs)
    csa.sync_status()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # a valid prefill shape that needs B * Tq * K * 4 = 256 MiB of scratch; real
    # (small) device buffers are passed so that no launch could touch a bogus address
    small = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    p = small.data_ptr()
    d = Dims(B=1, Tq=131072, HI=4, dI=64, K=512, m=4, n_entries=32768)
    rc = csa.lib().csa_index_topk_noalloc(p, p, p, p, ctypes.byref(d), p, None, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED
    assert b"8388608" in csa.lib().csa_last_error()
    # an invalid shape is reported as such, not as a scratch-size problem
    bad = Dims(B=1, Tq=131072, HI=4, dI=64, K=4096, m=4, n_entries=32768)
    rc = csa.lib().csa_index_topk_noalloc(p, p, p, p, ctypes.byref(bad), p, None, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and b"K=4096" in csa.lib().csa_last_error()
    bad = Dims(B=1, Tq=8, HI=4, dI=64, K=16, m=4, n_entries=100, entry_cap=50)
    rc = csa.lib().csa_index_topk_noalloc(p, p, p, p, ctypes.byref(bad), p, None, None)
    assert rc == csa.CSA_ERR_INVALID
    torch.cuda.synchronize()
    assert torch.count_nonzero(small) == 0
