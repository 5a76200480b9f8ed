"""Run in a child process with CSA_LIBRARY naming the CSA_CHECK build: the
small parity shapes of each indexer path, the block-scaled indexer and a
fused decode step, each followed by the build's own top-k checks; exits 0
when every call and every check passed (see test_gpu_check_build.py)."""
import sys

import numpy as np
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims, pipeline
from oracle import csa as ocsa


def index_case(B, Tq, N, HI, dI, K, seed, pos=None):
    inp = synth.indexer_inputs(B, Tq, N, HI, dI, seed=seed)
    if pos is None:
        g = torch.Generator().manual_seed(seed)
        pos = torch.randint(0, 4 * N + 10, (B, Tq), generator=g, dtype=torch.int32)
    d = Dims(B=B, Tq=Tq, HI=HI, dI=dI, K=K, m=4, n_entries=N)
    idx = torch.empty((B, Tq, K), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, Tq, K), device="cuda")
    ws = torch.empty(max(1, csa.index_topk_workspace(d)), dtype=torch.uint8, device="cuda")
    csa.index_topk(inp.qI.cuda(), inp.w.cuda(), inp.kI.cuda(), pos.cuda(), d, idx, sc, workspace=ws)
    csa.sync_status()
    ri, _ = ocsa.topk(ocsa.indexer_scores64(inp.qI.numpy(), inp.w.numpy(), inp.kI[:, :N].numpy()),
                      ocsa.n_visible(pos.numpy(), 4, N), K)
    assert np.array_equal(idx.cpu().numpy(), ri)


def main():
    assert csa.is_check_build(), "not the CSA_CHECK build"
    n0 = csa.launch_count()
    index_case(2, 300, 3000, 4, 64, 100, seed=1)                 # prefill path (> 64 rows)
    index_case(16, 1, 16384, 4, 64, 512, seed=2,
               pos=torch.full((16, 1), 4 * 16384 - 1, dtype=torch.int32))   # decode path
    index_case(1, 16, 5000, 8, 32, 512, seed=3)                  # split / merge path
    index_case(1, 64, 20000, 4, 64, 512, seed=4)                 # scan / collect path
    index_case(2, 9, 700, 2, 32, 16, seed=5)                     # generic path
    mx = synth.indexer_inputs_mx(4, 3, 2000, 4, 64, seed=6)
    d = Dims(B=4, Tq=3, HI=4, dI=64, K=128, m=4, n_entries=2000)
    idx = torch.empty((4, 3, 128), dtype=torch.int32, device="cuda")
    sc = torch.empty((4, 3, 128), device="cuda")
    ws = torch.empty(max(1, csa.index_topk_mx_workspace(d)), dtype=torch.uint8, device="cuda")
    pos = torch.randint(0, 8010, (4, 3), generator=torch.Generator().manual_seed(6), dtype=torch.int32)
    csa.index_topk_mx(mx.qI.cuda(), mx.qs.cuda(), mx.w.cuda(), mx.kI.cuda(), mx.ks.cuda(), pos.cuda(), d, idx, sc,
                      workspace=ws)
    csa.sync_status()
    # a short fused decode chain (128 heads x 512)
    B, T0, m, K, W, H, D = 2, 2048, 4, 64, 128, 128, 512
    N = T0 // m + 8
    x, z = synth.tokens(B, T0 + 8, D, seed=7)
    ind = synth.indexer_inputs(B, 2, N, 4, 64, seed=7)
    st = pipeline.DecodeState(B, D, H, m, W, entry_cap=N, K=K, fused=True)
    st.prefill_context(x.cuda(), z.cuda(), T0, kI=ind.kI.cuda())
    for s in range(2):
        lo = T0 + 4 * s
        q = synth.queries(B, 1, H, D, 1 / 8, seed=10 + s).cuda()
        st.step(x[:, lo:lo + 4].cuda().contiguous(), z[:, lo:lo + 4].cuda().contiguous(), q,
                ind.qI[:, s:s + 1].cuda().contiguous(), ind.w[:, s:s + 1].cuda().contiguous(),
                ind.kI[:, T0 // m + s:T0 // m + s + 1].cuda().contiguous())
        csa.sync_status()
    print("check build: clean,", csa.launch_count() - n0, "launches")
    return 0


if __name__ == "__main__":
    sys.exit(main())
