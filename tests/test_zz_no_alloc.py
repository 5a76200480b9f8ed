"""The allocation-free indexer entry point (csa_index_topk_noalloc), called
through the C ABI, against the workspace version (csa_index_topk).

Callers that cannot allocate device memory (allocator hooks, runtimes that
plan all memory at load time, plug-ins handed only their inputs and outputs)
use this entry point; its scratch is a fixed array inside the library.  Two
calls in a row with different inputs must each give exactly the results of
the workspace version: indices and scores are exact, so the comparison is
bit-exact.  This file is collected last so that a run stopping at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims

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


def test_noalloc_matches_workspace_version_twice():
    # decode shape of the 64K-context workload: 16 rows x 16,384 entries (1 MiB of scratch),
    # then a second, different call that reuses the same scratch
    shapes = [(16, 1, 16384, 65535, 1), (3, 40, 5000, None, 2)]
    for B, Tq, N, pos, seed in shapes:
        inp = synth.indexer_inputs(B, Tq, N, 4, 64, seed, device="cuda")
        if pos is None:
            q_pos = torch.randint(0, 4 * N + 8, (B, Tq), generator=torch.Generator().manual_seed(seed),
                                  dtype=torch.int32).cuda()
        else:
            q_pos = torch.full((B, Tq), pos, dtype=torch.int32, device="cuda")
        d = Dims(B=B, Tq=Tq, HI=4, dI=64, K=512, m=4, n_entries=N)
        ri, rs = _with_workspace(inp, q_pos, d)
        gi, gs = _noalloc(inp, q_pos, d)
        torch.cuda.synchronize()
        assert torch.equal(gi, ri)
        assert torch.equal(gs, rs)
    csa.sync_status()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    d = Dims(B=1, Tq=131072, HI=4, dI=64, K=512, m=4, n_entries=32768)   # 17 GB of scores
    fake = ctypes.c_void_p(1 << 20)
    rc = csa.lib().csa_index_topk_noalloc(fake, fake, fake, fake, ctypes.byref(d), fake, None, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED
    assert b"8388608" in csa.lib().csa_last_error()
