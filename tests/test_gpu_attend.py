"""GPU parity of csa_attend / hca_attend against the oracle's fp64 attention,
through the C ABI.  The compressed cache and the window ring are random E4M3
bytes from the seeded generator (the same bytes go to both sides)."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims
from oracle import csa as ocsa
from oracle.formats import e4m3_decode
from tests import parity

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _random_selection(rng, q_pos, m, n_entries, K, pad_anywhere=False):
    B, Tq = q_pos.shape
    idx = np.full((B, Tq, K), -1, dtype=np.int32)
    for b in range(B):
        for i in range(Tq):
            nv = int(ocsa.n_visible(q_pos[b, i], m, n_entries))
            k = min(K, nv)
            if k:
                pick = rng.choice(nv, k, replace=False)
                if pad_anywhere:
                    slots = np.sort(rng.choice(K, k, replace=False))
                    idx[b, i, slots] = pick
                else:
                    idx[b, i, :k] = pick
    return idx


def _setup(B, Tq, H, D, N, win_cap, q_pos, seed, q_scale):
    codes, scales = synth.e4m3_cache(B, N, D, seed)
    wcodes, wscales = synth.e4m3_cache(B, win_cap, D, seed, tag="win")
    q = synth.queries(B, Tq, H, D, q_scale, seed)
    ent = ocsa.dequantize(codes.numpy(), scales.numpy())
    wv = ocsa.dequantize(wcodes.numpy(), wscales.numpy())
    return codes, scales, wcodes, wscales, q, ent, wv


def _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d):
    B, Tq, H, D = q.shape
    out = torch.empty((B, Tq, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Tq, H), device="cuda")
    dense = idx is None
    nb = csa.attend_workspace(d, dense)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    args = (q.cuda(), codes.cuda(), scales.cuda())
    tail = (wcodes.cuda(), wscales.cuda(), torch.from_numpy(q_pos).cuda(), d, out, lse)
    if dense:
        csa.hca_attend(*args, *tail, workspace=ws)
    else:
        csa.attend(*args, torch.from_numpy(idx).cuda(), *tail, workspace=ws)
    csa.sync_status()
    return out, lse


CASES = [
    # B, Tq, H, D, m, N, K, W, win_cap, q_scale
    (2, 7, 4, 64, 4, 128, 16, 32, 512, 1 / 8),
    (2, 5, 128, 512, 4, 3000, 512, 128, 128, 512 ** -0.5),
    (1, 9, 64, 512, 4, 2100, 512, 128, 8400, 512 ** -0.5),
    (3, 4, 16, 256, 4, 700, 100, 50, 64, 0.1),
    (1, 6, 8, 128, 2, 400, 33, 7, 7, 0.2),
    # 64 heads x 512 (items as MMA rows): partial tiles, -1 anywhere, window-only rows
    (2, 6, 64, 512, 4, 300, 100, 50, 1200, 0.1),
    (1, 3, 64, 512, 4, 600, 512, 128, 128, 512 ** -0.5),
]


@pytest.mark.parametrize("B,Tq,H,D,m,N,K,W,win_cap,qs", CASES)
def test_csa_attend_parity(B, Tq, H, D, m, N, K, W, win_cap, qs):
    rng = np.random.default_rng(B * 100 + H + D)
    tmax = min(m * N + m - 1, win_cap * 50)
    q_pos = rng.integers(0, tmax, (B, Tq)).astype(np.int32)
    q_pos[0, 0] = 0
    q_pos[-1, -1] = m * N - 1
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, Tq, H, D, N, win_cap, q_pos, 7, qs)
    idx = _random_selection(rng, q_pos, m, N, K, pad_anywhere=(K == 100))
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=win_cap)
    out, lse = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: wv[b, p % win_cap], q_pos, W)
    parity.check_attention(out, lse, ro, rl)


@pytest.mark.parametrize("B,Tq,H,D,m,N,W", [(2, 5, 128, 512, 128, 300, 128), (1, 4, 4, 64, 4, 200, 32),
                                             (2, 3, 64, 512, 4, 1500, 128)])
def test_hca_attend_parity(B, Tq, H, D, m, N, W):
    rng = np.random.default_rng(N)
    q_pos = rng.integers(0, m * N + 3 * m, (B, Tq)).astype(np.int32)
    q_pos[0, 0] = m - 2          # before the first entry completes: window only
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, Tq, H, D, N, W, q_pos, 8, 512 ** -0.5)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=1, W=W, m=m, n_entries=N, win_cap=W)
    out, lse = _run_gpu(q, codes, scales, None, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.hca_attend(_bits(q), ent, lambda b, p: wv[b, p % W], q_pos, m, W)
    parity.check_attention(out, lse, ro, rl)



# The 128-head kernel splits each (row, half of D) into 1, 2, 4 or 8 item
# splits, one thread-block cluster, from the row count and the longest item
# list (splits * 2 * rows <= 148, at least two 64-item chunks per split); the
# cases above all take 4.  These reach 8 (few rows, long lists; the last splits
# of a row get no chunk at all), 2 and 1 (many rows), sparse and dense.
SPLIT_CASES = [
    # B, Tq, m, N, K, W, dense, splits the plan gives
    (1, 1, 4, 1200, 1, 128, True, 8),     # 1,328 items = 21 chunks: 7 splits of 3, one empty
    (1, 2, 4, 1500, 1024, 128, False, 8),  # 1,152 items = 18 chunks: 6 splits of 3, two empty
    (2, 12, 4, 400, 64, 32, False, 2),     # 24 rows
    (2, 20, 4, 300, 1, 32, True, 1),       # 40 rows
]


@pytest.mark.parametrize("B,Tq,m,N,K,W,dense,splits", SPLIT_CASES)
def test_128_head_split_counts(B, Tq, m, N, K, W, dense, splits):
    H, D = 128, 512
    rng = np.random.default_rng(1000 + 10 * B + Tq)
    if splits == 8:
        # every row sees its whole list: the plan's longest list is reached
        q_pos = (m * N - 1 - 37 * np.arange(B * Tq)).reshape(B, Tq).astype(np.int32)
    else:
        q_pos = rng.integers(0, m * N, (B, Tq)).astype(np.int32)
        q_pos[0, 0] = 0
        q_pos[-1, -1] = m * N - 1
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, Tq, H, D, N, W, q_pos, 17, 512 ** -0.5)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=W)
    if dense:
        out, lse = _run_gpu(q, codes, scales, None, wcodes, wscales, q_pos, d)
        ro, rl = ocsa.hca_attend(_bits(q), ent, lambda b, p: wv[b, p % W], q_pos, m, W)
    else:
        idx = _random_selection(rng, q_pos, m, N, K)
        out, lse = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
        ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: wv[b, p % W], q_pos, W)
    parity.check_attention(out, lse, ro, rl)

def test_softmax_scale_is_applied():
    B, Tq, H, D, m, N, K, W = 1, 3, 8, 64, 4, 50, 8, 16
    q_pos = np.array([[199, 100, 40]], dtype=np.int32)
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, Tq, H, D, N, W, q_pos, 9, 1.0)
    idx = _random_selection(np.random.default_rng(3), q_pos, m, N, K)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=W, softmax_scale=0.125)
    out, lse = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: wv[b, p % W], q_pos, W, scale=0.125)
    parity.check_attention(out, lse, ro, rl)


def test_out_of_range_index_is_reported():
    B, Tq, H, D, m, N, K, W = 1, 1, 4, 64, 4, 20, 4, 8
    q_pos = np.array([[79]], dtype=np.int32)
    codes, scales, wcodes, wscales, q, _, _ = _setup(B, Tq, H, D, N, W, q_pos, 10, 0.1)
    idx = np.array([[[1, 2, 20, -1]]], dtype=np.int32)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=W)
    with pytest.raises(csa.CsaError) as e:
        _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    assert e.value.code == csa.CSA_ERR_INVALID


def test_csa_decode_64k_full_size():
    """Attention step of the 64K-context decode workload: 16 sequences, 128
    heads, D = 512, K = 512 selected of 16,384 entries plus a 128-token window."""
    B, H, D, m, N, K, W = 16, 128, 512, 4, 16384, 512, 128
    rng = np.random.default_rng(12)
    q_pos = np.full((B, 1), m * N - 1, dtype=np.int32)
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, 1, H, D, N, W, q_pos, 12, 512 ** -0.5)
    idx = _random_selection(rng, q_pos, m, N, K)
    d = Dims(B=B, Tq=1, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=W)
    out, lse = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: wv[b, p % W], q_pos, W)
    parity.check_attention(out, lse, ro, rl)


def test_hca_decode_1m_full_size():
    """Attention step of the 1M-context HCA workload: 16 sequences x (8,192
    entries + 128 window tokens) x 128 heads x 512."""
    B, H, D, m, N, W = 16, 128, 512, 128, 8192, 128
    q_pos = np.full((B, 1), m * N - 1, dtype=np.int32)
    codes, scales, wcodes, wscales, q, ent, wv = _setup(B, 1, H, D, N, W, q_pos, 13, 512 ** -0.5)
    d = Dims(B=B, Tq=1, H=H, D=D, K=1, W=W, m=m, n_entries=N, win_cap=W)
    out, lse = _run_gpu(q, codes, scales, None, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.hca_attend(_bits(q), ent, lambda b, p: wv[b, p % W], q_pos, m, W)
    parity.check_attention(out, lse, ro, rl)


@pytest.mark.parametrize("H", [64, 128, 16])
@pytest.mark.parametrize("qexp,sexp", [((-16, -6), (-12, 12)), ((6, 10), (-30, -20))])
def test_wide_dynamic_range(H, qexp, sexp):
    """Per-head query magnitudes 2^qexp and per-entry scales 2^sexp / 448 far
    from 1: the kernels that compute in fp16 bring both into range with exact
    powers of two, which must not cost accuracy anywhere in these ranges."""
    B, Tq, D, m, N, K, W, win_cap = 1, 5, 512, 4, 900, 512, 128, 128
    rng = np.random.default_rng(H + qexp[0])
    q_pos = rng.integers(0, m * N, (B, Tq)).astype(np.int32)
    q_pos[0, 0] = 3
    codes, _, wcodes, _, q, _, _ = _setup(B, Tq, H, D, N, win_cap, q_pos, 21, 1.0)
    scales = torch.from_numpy((2.0 ** rng.uniform(*sexp, (B, N)) / 448.0).astype(np.float32))
    wscales = torch.from_numpy((2.0 ** rng.uniform(*sexp, (B, win_cap)) / 448.0).astype(np.float32))
    hf = torch.from_numpy(2.0 ** rng.integers(qexp[0], qexp[1] + 1, H).astype(np.float32))
    q = (q.float() * hf[None, None, :, None]).to(torch.bfloat16)
    ent = ocsa.dequantize(codes.numpy(), scales.numpy())
    wv = ocsa.dequantize(wcodes.numpy(), wscales.numpy())
    idx = _random_selection(rng, q_pos, m, N, K)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=win_cap, softmax_scale=D ** -0.5)
    out, lse = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: wv[b, p % win_cap], q_pos, W, scale=D ** -0.5)
    parity.check_attention(out, lse, ro, rl)


def _all_codes_row(D):
    """D E4M3 codes: column d holds byte d mod 256, except the two NaN codes
    (0x7F, 0xFF), which the library's quantiser never writes, set to 0.  Each
    256-column half of D = 512 holds every finite code, subnormals included."""
    c = (np.arange(D) % 256).astype(np.uint8)
    c[(c == 0x7F) | (c == 0xFF)] = 0
    return c


@pytest.mark.parametrize("dense", [False, True])
def test_every_e4m3_code_decodes_exactly(dense):
    """Every attended item holds the same codes (every finite E4M3 byte, in
    both halves of D) with scale 1, so all logits are equal, every weight is
    exactly 1 / n and the output row is the decoded codes: each code's bf16
    image must come out exactly, the 7 subnormal magnitudes and the zeros
    included.  (The fused decode step shares the same
    conversion.)  A per-row tolerance could not see a wrong subnormal."""
    B, Tq, H, D, m, N, K, W = 2, 3, 128, 512, 4, 700, 512, 128
    row = _all_codes_row(D)
    codes = torch.from_numpy(np.broadcast_to(row, (B, N, D)).copy())
    wcodes = torch.from_numpy(np.broadcast_to(row, (B, W, D)).copy())
    scales = torch.ones((B, N), dtype=torch.float32)
    wscales = torch.ones((B, W), dtype=torch.float32)
    q = synth.queries(B, Tq, H, D, 512 ** -0.5, 5)
    q_pos = np.array([[m * N - 1, 1000, 3]] * B, dtype=np.int32)
    rng = np.random.default_rng(7)
    idx = None if dense else _random_selection(rng, q_pos, m, N, K)
    d = Dims(B=B, Tq=Tq, H=H, D=D, K=K, W=W, m=m, n_entries=N, win_cap=W)
    out, _ = _run_gpu(q, codes, scales, idx, wcodes, wscales, q_pos, d)
    want = torch.from_numpy(e4m3_decode(row)).to(torch.bfloat16)
    got = out.cpu()
    assert torch.equal(got, want.expand_as(got)), (
        f"{int((got != want.expand_as(got)).sum())} outputs differ from the decoded codes")
