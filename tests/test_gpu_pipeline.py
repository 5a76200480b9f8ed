"""End-to-end parity: the GPU chain (compress -> index/top-k -> attend)
against the oracle's own chain from the same raw synthetic inputs.  Neither
side consumes the other's intermediates; indices must match bit for bit and
outputs within the attention tolerance."""
import numpy as np
import pytest
import torch

import synth
from compressed_sparse_attention_16_b200 import pipeline
from oracle import csa as ocsa
from oracle.formats import bf16_decode
from tests import parity

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _entry_values(x, z, b, entries, m):
    """Oracle entries (dequantised) for the given entry ids of sequence b;
    x, z may live on the GPU -- only the needed tokens are copied."""
    if len(entries) == 0:
        return np.zeros((0, x.shape[-1]))
    e = torch.as_tensor(np.asarray(entries, dtype=np.int64), device=x.device)
    tok = (e[:, None] * m + torch.arange(m, device=x.device)[None]).reshape(-1)
    xs = x[b, tok].reshape(len(entries), m, -1).cpu().numpy()
    zs = z[b, tok].reshape(len(entries), m, -1).cpu().numpy()
    codes, s = ocsa.quantize_entries(ocsa.pool_blocks(xs, zs))
    return ocsa.dequantize(codes, s)


def _window_values(x, b, positions):
    p = torch.as_tensor(np.asarray(positions, dtype=np.int64), device=x.device)
    return ocsa.window_token_values(x[b, p].cpu().numpy())


def _oracle_decode(x, z, qI, w, kI, q, t, m, K, W, n_entries):
    """Oracle for one query per sequence at position t with n_entries entries."""
    B = q.shape[0]
    s64 = ocsa.indexer_scores64(qI.cpu().numpy(), w.cpu().numpy(), kI[:, :n_entries].cpu().numpy())
    nv = np.full((B, 1), ocsa.n_visible(t, m, n_entries))
    idx, _ = ocsa.topk(s64, nv, K)
    qv = bf16_decode(_bits(q))
    outs, lses = [], []
    for b in range(B):
        sel = idx[b, 0][idx[b, 0] >= 0]
        U = np.concatenate([_entry_values(x, z, b, sel, m), _window_values(x, b, ocsa.window_positions(t, W))])
        o, l = ocsa.attend_one(qv[b, 0], U)
        outs.append(o)
        lses.append(l)
    return idx, np.stack(outs)[:, None], np.stack(lses)[:, None]


def test_tiny_prefill_chain():
    """512-token prefill, m = 4, K = 16, W = 32, 4 heads x 64, indexer 2 x 32."""
    wl = synth.WORKLOADS["tiny_prefill"]
    x, z = synth.tokens(wl.B, wl.T, wl.D, 0)
    q = synth.queries(wl.B, wl.T, wl.H, wl.D, wl.q_scale, 0)
    ind = synth.indexer_inputs(wl.B, wl.T, wl.N, wl.HI, wl.dI, 0)
    pooled = torch.empty((wl.B, wl.N, wl.D), device="cuda")
    r = pipeline.prefill(x.cuda(), z.cuda(), q.cuda(), ind.qI.cuda(), ind.w.cuda(), ind.kI.cuda(),
                         m=wl.m, K=wl.K, W=wl.W, pooled=pooled)
    torch.cuda.synchronize()
    xn, zn = x.numpy(), z.numpy()
    ref_pool, A = parity.pooled_and_scale(xn, zn, wl.m)
    parity.check_pooled(pooled.cpu().numpy(), ref_pool, A)
    parity.check_codes(r.codes.cpu().numpy(), r.scales.cpu().numpy(), ref_pool, A)
    ent = ocsa.dequantize(*ocsa.quantize_entries(ref_pool))
    win = ocsa.window_token_values(xn)
    pos = np.arange(wl.T)[None]
    s64 = ocsa.indexer_scores64(ind.qI.numpy(), ind.w.numpy(), ind.kI.numpy())
    idx, sc = ocsa.topk(s64, ocsa.n_visible(pos, wl.m, wl.N), wl.K)
    assert np.array_equal(r.idx.cpu().numpy(), idx)
    assert np.array_equal(r.score.cpu().numpy().astype(np.float64), sc)
    ro, rl = ocsa.attend(_bits(q), ent, idx, lambda b, p: win[b, p], pos, wl.W)
    parity.check_attention(r.out, r.lse, ro, rl)


def test_decode_state_small_chain():
    """A decode cache grown step by step (window ring wraps many times) equals
    the oracle at every step; an HCA cache alongside."""
    B, D, H, m, W, K, HI, dI = 2, 64, 4, 4, 16, 8, 2, 32
    T0, steps = 64, 6
    Ttot = T0 + 4 * steps
    x, z = synth.tokens(B, Ttot, D, 3, device="cuda")
    ind = synth.indexer_inputs(B, steps, Ttot // m, HI, dI, 3, device="cuda")
    qs = synth.queries(B, steps, H, D, 0.3, 3, device="cuda")
    st = pipeline.DecodeState(B, D, H, m, W, entry_cap=Ttot // m, K=K, HI=HI, dI=dI)
    hs = pipeline.DecodeState(B, D, H, m, W, entry_cap=Ttot // m, dense=True)
    st.prefill_context(x, z, T0, kI=ind.kI)
    hs.prefill_context(x, z, T0)
    for i in range(steps):
        t0 = T0 + 4 * i
        sl = slice(t0, t0 + 4)
        q = qs[:, i:i + 1].contiguous()
        out, lse = st.step(x[:, sl].contiguous(), z[:, sl].contiguous(), q,
                           ind.qI[:, i:i + 1].contiguous(), ind.w[:, i:i + 1].contiguous(),
                           kI_new=ind.kI[:, t0 // m:(t0 + 4) // m])
        hout, hlse = hs.step(x[:, sl].contiguous(), z[:, sl].contiguous(), q)
        torch.cuda.synchronize()
        t = t0 + 3
        n = (t0 + 4) // m
        ridx, ro, rl = _oracle_decode(x, z, ind.qI[:, i:i + 1], ind.w[:, i:i + 1], ind.kI, q, t, m, K, W, n)
        assert np.array_equal(st.idx.cpu().numpy(), ridx)
        parity.check_attention(out, lse, ro, rl)
        # HCA: every visible entry
        qv = bf16_decode(_bits(q))
        for b in range(B):
            U = np.concatenate([_entry_values(x, z, b, np.arange(n), m),
                                _window_values(x, b, ocsa.window_positions(t, W))])
            o, l = ocsa.attend_one(qv[b, 0], U)
            parity.check_attention(hout[b:b + 1], hlse[b:b + 1], o[None, None], l[None, None])


@pytest.mark.parametrize("name", ["csa_decode_64k", "csa_decode_1m_incremental"])
def test_decode_workload_chain_full_size(name):
    """Full-size decode workloads through the same DecodeState calls the bench
    times: every query of the first steps checked end to end."""
    wl = synth.WORKLOADS[name]
    steps = 3 if wl.kind == "decode_incremental" else 1
    T0 = wl.T if wl.kind == "decode_incremental" else wl.T - 4
    Ttot = T0 + 4 * steps
    N = Ttot // wl.m
    x, z = synth.tokens(wl.B, Ttot, wl.D, 0, device="cuda")
    ind = synth.indexer_inputs(wl.B, steps, N, wl.HI, wl.dI, 0, device="cuda")
    qs = synth.queries(wl.B, steps, wl.H, wl.D, wl.q_scale, 0, device="cuda")
    st = pipeline.DecodeState(wl.B, wl.D, wl.H, wl.m, wl.W, entry_cap=N, K=wl.K, HI=wl.HI, dI=wl.dI)
    st.prefill_context(x, z, T0, kI=ind.kI)
    st.kI.copy_(ind.kI)
    for i in range(steps):
        t0 = T0 + 4 * i
        q = qs[:, i:i + 1].contiguous()
        out, lse = st.step(x[:, t0:t0 + 4].contiguous(), z[:, t0:t0 + 4].contiguous(), q,
                           ind.qI[:, i:i + 1].contiguous(), ind.w[:, i:i + 1].contiguous())
        torch.cuda.synchronize()
        ridx, ro, rl = _oracle_decode(x, z, ind.qI[:, i:i + 1], ind.w[:, i:i + 1], ind.kI, q,
                                      t0 + 3, wl.m, wl.K, wl.W, (t0 + 4) // wl.m)
        assert np.array_equal(st.idx.cpu().numpy(), ridx)
        parity.check_attention(out, lse, ro, rl)
    del x, z, st
    torch.cuda.empty_cache()


def test_prefill_128k_full_size_sampled():
    """128K prefill through pipeline.prefill (the launches the bench times):
    1,024 sampled query rows checked end to end."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    x, z = synth.tokens(wl.B, wl.T, wl.D, 0, device="cuda")
    q = synth.queries(wl.B, wl.T, wl.H, wl.D, wl.q_scale, 0, device="cuda")
    ind = synth.indexer_inputs(wl.B, wl.T, wl.N, wl.HI, wl.dI, 0, device="cuda")
    r = pipeline.prefill(x, z, q, ind.qI, ind.w, ind.kI, m=wl.m, K=wl.K, W=wl.W)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 4, 127, 128, 2047, 2048, wl.T - 1],
                                     rng.choice(wl.T, 1014, replace=False)]))
    rr = torch.from_numpy(rows).cuda()
    s64 = ocsa.indexer_scores64(ind.qI[:, rr].cpu().numpy(), ind.w[:, rr].cpu().numpy(), ind.kI.cpu().numpy())
    idx, _ = ocsa.topk(s64, ocsa.n_visible(rows[None], wl.m, wl.N), wl.K)
    assert np.array_equal(r.idx[:, rr].cpu().numpy(), idx)
    qv = bf16_decode(_bits(q[:, rr]))
    ro = np.zeros((1, len(rows), wl.H, wl.D))
    rl = np.zeros((1, len(rows), wl.H))
    for i, t in enumerate(rows):
        sel = idx[0, i][idx[0, i] >= 0]
        U = np.concatenate([_entry_values(x, z, 0, sel, wl.m), _window_values(x, 0, ocsa.window_positions(t, wl.W))])
        ro[0, i], rl[0, i] = ocsa.attend_one(qv[0, i], U)
    parity.check_attention(r.out[:, rr], r.lse[:, rr], ro, rl)


def test_bounded_wait_expiry_is_reported_and_context_survives():
    """A device wait that nothing satisfies gives up after its limit, sets the
    timeout status, and the context stays usable for the next call."""
    import compressed_sparse_attention_16_b200 as csa
    csa.sync_status()
    csa.selftest_timeout(2_000_000)
    with pytest.raises(csa.CsaError) as e:
        csa.sync_status()
    assert e.value.code == csa.CSA_ERR_TIMEOUT
    csa.sync_status()                        # the bit was cleared
    x = torch.randn(1, 8, 64, device="cuda")
    codes = torch.empty((1, 2, 64), dtype=torch.uint8, device="cuda")
    scales = torch.empty((1, 2), device="cuda")
    csa.compress(x, torch.zeros_like(x), 4, codes, scales)
    csa.sync_status()


def test_sharded_prefill_one_rank_equals_prefill():
    """prefill_sharded on a one-rank NCCL group runs the same calls on the
    same data as prefill: identical outputs (the multi-rank plumbing is
    covered with gloo ranks on the CPU)."""
    import socket
    from datetime import timedelta

    import torch.distributed as dist

    from compressed_sparse_attention_16_b200 import shard
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60))
    try:
        B, T, D, H, m, K, W = 1, 1030, 512, 64, 4, 64, 128
        x, z = synth.tokens(B, T, D, 3)
        q = synth.queries(B, T, H, D, 512 ** -0.5, 3)
        ind = synth.indexer_inputs(B, T, T // m, 4, 64, 3)
        x, z, q = x.cuda(), z.cuda(), q.cuda()
        qI, w, kI = ind.qI.cuda(), ind.w.cuda(), ind.kI.cuda()
        ref = pipeline.prefill(x, z, q, qI, w, kI, m=m, K=K, W=W)
        got = shard.prefill_sharded(x, z, kI, q, qI, w, T=T, m=m, K=K, W=W)
        torch.cuda.synchronize()
        assert torch.equal(got.pos.cuda().long(), torch.arange(T, device="cuda"))
        assert torch.equal(got.idx, ref.idx) and torch.equal(got.score, ref.score)
        assert torch.equal(got.out, ref.out) and torch.equal(got.lse, ref.lse)
    finally:
        dist.destroy_process_group()
