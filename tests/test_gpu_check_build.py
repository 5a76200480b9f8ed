"""The CSA_CHECK debug build and the device-side top-k check.

csa_check_topk must flag each kind of broken list (out of order, repeated
index, index out of range, bad padding, bad score) through the status word
(CSA_ERR_CHECK) without faulting, and accept correct lists; the CSA_CHECK
build (libcsa_check.so) must run the small parity shapes of every indexer
path, the block-scaled indexer and a fused decode step with all its checks
passing."""
import os
import subprocess
import sys

import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
from compressed_sparse_attention_16_b200 import Dims, build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lists():
    # two rows at positions 39 (10 visible with m = 4) and 7 (2 visible), K = 4
    idx = torch.tensor([[[7, 3, 5, 0], [1, 0, -1, -1]]], dtype=torch.int32)
    sc = torch.tensor([[[9.0, 4.0, 4.0, 1.0], [2.0, 2.0, 0.0, 0.0]]])
    pos = torch.tensor([[39, 7]], dtype=torch.int32)
    return idx, sc, pos


def _status(idx, sc, pos, use_score=True):
    d = Dims(B=1, Tq=2, K=4, m=4, n_entries=100)
    csa.check_topk(idx.cuda(), sc.cuda() if use_score else None, pos.cuda(), d)
    try:
        csa.sync_status()
        return 0
    except csa.CsaError as e:
        return e.code


def test_correct_lists_pass():
    idx, sc, pos = _lists()
    idx[0, 1] = torch.tensor([0, 1, -1, -1], dtype=torch.int32)   # equal scores: ascending index
    assert _status(idx, sc, pos) == 0
    assert _status(idx, sc, pos, use_score=False) == 0


@pytest.mark.parametrize("what", ["order", "tie_order", "range", "padding", "pad_score", "negative", "count"])
def test_broken_lists_are_flagged(what):
    idx, sc, pos = _lists()
    idx[0, 1] = torch.tensor([0, 1, -1, -1], dtype=torch.int32)
    if what == "order":
        sc[0, 0, 1] = 0.5                      # 9, 0.5, 4, 1
    elif what == "tie_order":
        idx[0, 0, 1], idx[0, 0, 2] = 5, 3      # equal scores, descending indices
    elif what == "range":
        idx[0, 0, 3] = 10                      # only 10 visible: 0..9
    elif what == "padding":
        idx[0, 1, 3] = 4
    elif what == "pad_score":
        sc[0, 1, 2] = 1.0
    elif what == "negative":
        sc[0, 0, 3] = -1.0
    elif what == "count":
        idx[0, 1, 1] = -1                      # two visible but one listed
    assert _status(idx, sc, pos) == csa.CSA_ERR_CHECK
    # the context is still usable
    idx2, sc2, pos2 = _lists()
    idx2[0, 1] = torch.tensor([0, 1, -1, -1], dtype=torch.int32)
    assert _status(idx2, sc2, pos2) == 0


def test_check_build_runs_the_small_parity_shapes_clean():
    lib = build.build_check()
    env = dict(os.environ, CSA_LIBRARY=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "tests.check_build_run"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "check build: clean" in r.stdout
    assert not csa.is_check_build()          # this process keeps the default build
