"""The fused decode step (csa_decode_step: append, index, select and attend
in one launch) against the oracle, through DecodeState.step, and against the
separate calls it replaces.

Indices and scores are exact on both sides and must match the oracle bit for
bit; the appended cache rows must be bit-identical to csa_compress's; the
attention output is held to the library's bf16 tolerance against the fp64
oracle."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_16_b200 as csa
import synth
from compressed_sparse_attention_16_b200 import Dims, pipeline
from oracle import csa as ocsa
from oracle.formats import bf16_decode
from tests import parity

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_step(x, z, qI, w, kI, q, t, m, K, W, n_entries):
    """Oracle of one query per sequence at position t with n_entries entries;
    the entries and window tokens it needs are pooled from x, z by the oracle."""
    B = q.shape[0]
    s64 = ocsa.indexer_scores64(qI.cpu().numpy(), w.cpu().numpy(), kI[:, :n_entries].cpu().numpy())
    nv = np.full((B, 1), ocsa.n_visible(t, m, n_entries))
    idx, sc = ocsa.topk(s64, nv, K)
    qv = bf16_decode(_bits(q))
    outs, lses = [], []
    for b in range(B):
        sel = idx[b, 0][idx[b, 0] >= 0]
        if len(sel):
            e = torch.as_tensor(sel.astype(np.int64), device=x.device)
            tok = (e[:, None] * m + torch.arange(m, device=x.device)[None]).reshape(-1)
            xs = x[b, tok].reshape(len(sel), m, -1).cpu().numpy()
            zs = z[b, tok].reshape(len(sel), m, -1).cpu().numpy()
            ent = ocsa.dequantize(*ocsa.quantize_entries(ocsa.pool_blocks(xs, zs)))
        else:
            ent = np.zeros((0, x.shape[-1]))
        wp = torch.as_tensor(np.asarray(ocsa.window_positions(t, W), dtype=np.int64), device=x.device)
        win = ocsa.window_token_values(x[b, wp].cpu().numpy())
        o, l = ocsa.attend_one(qv[b, 0], np.concatenate([ent, win]))
        outs.append(o)
        lses.append(l)
    return idx, sc, np.stack(outs)[:, None], np.stack(lses)[:, None]


def _run_chain(B, T0, steps, *, K=512, W=128, HI=4, n_new=4, m=4, seed=0, pass_keys=True, win_cap=None,
               q_scale=512 ** -0.5, check_every=1, kI_override=None):
    D, H, dI = 512, 128, 64
    Ttot = T0 + n_new * steps
    N = Ttot // m
    x, z = synth.tokens(B, Ttot, D, seed, device="cuda")
    ind = synth.indexer_inputs(B, steps, N, HI, dI, seed, device="cuda")
    kI_all = ind.kI if kI_override is None else kI_override
    qs = synth.queries(B, steps, H, D, q_scale, seed, device="cuda")
    st = pipeline.DecodeState(B, D, H, m, W, entry_cap=N, K=K, HI=HI, dI=dI, win_cap=win_cap, fused=True)
    st.prefill_context(x, z, T0, kI=kI_all)
    if not pass_keys:
        st.kI.copy_(kI_all)
    assert st.step_workspace(n_new) is not None, "shape should take the fused step"
    n0 = csa.launch_count()
    for i in range(steps):
        t0 = T0 + n_new * i
        q = qs[:, i:i + 1].contiguous()
        kn = kI_all[:, t0 // m:(t0 + n_new) // m].contiguous() if pass_keys else None
        out, lse = st.step(x[:, t0:t0 + n_new].contiguous(), z[:, t0:t0 + n_new].contiguous(), q,
                           ind.qI[:, i:i + 1].contiguous(), ind.w[:, i:i + 1].contiguous(), kI_new=kn)
        if i % check_every and i != steps - 1:
            continue
        torch.cuda.synchronize()
        t = t0 + n_new - 1
        ridx, rsc, ro, rl = _oracle_step(x, z, ind.qI[:, i:i + 1], ind.w[:, i:i + 1], kI_all, q, t, m, K, W,
                                         (t + 1) // m)
        assert np.array_equal(st.idx.cpu().numpy(), ridx), f"step {i}: indices differ"
        assert np.array_equal(st.score.cpu().numpy().astype(np.float64), rsc), f"step {i}: scores differ"
        parity.check_attention(out, lse, ro, rl)
    assert csa.launch_count() - n0 == steps, "one launch per step expected"
    csa.sync_status()
    return st, x, z, kI_all


def test_small_chain_against_oracle():
    """2 sequences, 2,048-token context, 6 steps: every step checked."""
    _run_chain(2, 2048, 6, seed=1)


def test_short_context_fewer_entries_than_k():
    """Context of 60 tokens: 16..19 visible entries < K, -1 padding; window
    shorter than W at first."""
    _run_chain(3, 60, 4, K=512, seed=2)


@pytest.mark.parametrize("HI", [1, 2, 3])
def test_indexer_head_counts(HI):
    _run_chain(2, 4096, 2, HI=HI, seed=3 + HI)


def test_two_blocks_per_step_and_keys_already_cached():
    """8 tokens (two entries) per step; the new keys are already in the cache
    (kI_new = None)."""
    _run_chain(2, 1024, 3, n_new=8, pass_keys=False, seed=7)


def test_small_k_and_window():
    _run_chain(4, 3000, 3, K=1, W=1, win_cap=4, seed=8)
    _run_chain(4, 2000, 2, K=37, W=5, seed=9)



@pytest.mark.parametrize("B", [1, 9, 37])
def test_sequence_counts(B):
    """One sequence (every SM scans a share of its keys; five attention splits
    of one chunk per quarter of D), nine (16 scanning CTAs per sequence, three
    splits of two chunks: the online softmax across chunks) and 37, the most
    the step accepts (four scanning CTAs per sequence, one split of five
    chunks per quarter, written without a merge)."""
    _run_chain(B, 4096 if B == 1 else 2048, 3 if B == 1 else 2, seed=12 + B)

def test_massive_ties_take_the_refinement():
    """Every indexer key equal: all scores tie, the threshold bin holds every
    entry and the exact tie refinement must pick the lowest indices."""
    B, T0, steps, m = 2, 32768, 2, 4
    N = (T0 + 4 * steps) // m
    k = synth.indexer_inputs(B, 1, 1, 4, 64, 11, device="cuda").kI
    _run_chain(B, T0, steps, seed=11, kI_override=k.expand(B, N, 32).contiguous())


def test_bit_identical_to_separate_calls():
    """Caches, indices and scores equal the separate calls' exactly; the
    outputs agree to bf16 rounding of a different split merge."""
    B, T0, steps, m, D, H = 3, 8192, 3, 4, 512, 128
    Ttot = T0 + 4 * steps
    N = Ttot // m
    x, z = synth.tokens(B, Ttot, D, 12, device="cuda")
    ind = synth.indexer_inputs(B, steps, N, 4, 64, 12, device="cuda")
    qs = synth.queries(B, steps, H, D, 512 ** -0.5, 12, device="cuda")
    a = pipeline.DecodeState(B, D, H, m, 128, entry_cap=N, K=512, fused=True)
    b = pipeline.DecodeState(B, D, H, m, 128, entry_cap=N, K=512, fused=False)
    for st in (a, b):
        st.prefill_context(x, z, T0, kI=ind.kI)
    for i in range(steps):
        t0 = T0 + 4 * i
        args = (x[:, t0:t0 + 4].contiguous(), z[:, t0:t0 + 4].contiguous(), qs[:, i:i + 1].contiguous(),
                ind.qI[:, i:i + 1].contiguous(), ind.w[:, i:i + 1].contiguous())
        kn = ind.kI[:, t0 // m:(t0 + 4) // m].contiguous()
        oa, la = a.step(*args, kI_new=kn)
        ob, lb = b.step(*args, kI_new=kn)
        torch.cuda.synchronize()
        for name in ("codes", "scales", "win_codes", "win_scales", "kI", "idx", "score"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert (oa.float() - ob.float()).abs().max().item() <= 1e-2 * ob.float().abs().max().item()
        assert (la - lb).abs().max().item() <= 1e-4
    csa.sync_status()


@pytest.mark.parametrize("name", ["csa_decode_64k", "csa_decode_1m_incremental"])
def test_decode_workloads_full_size(name):
    """The two decode workloads at full size, through the fused step the bench
    times: every query of the first steps checked end to end."""
    wl = synth.WORKLOADS[name]
    steps = 3 if wl.kind == "decode_incremental" else 1
    T0 = wl.T if wl.kind == "decode_incremental" else wl.T - 4
    _run_chain(wl.B, T0, steps, K=wl.K, W=wl.W, HI=wl.HI, seed=0)
    torch.cuda.empty_cache()


def test_misaligned_position_is_reported():
    """A query position that does not end a block: the append is skipped and
    the status word reports it; the context stays usable."""
    B, D, H, m = 1, 512, 128, 4
    N = 64
    st = pipeline.DecodeState(B, D, H, m, 16, entry_cap=N, K=8, fused=True)
    x, z = synth.tokens(B, 4, D, 0, device="cuda")
    ind = synth.indexer_inputs(B, 1, N, 4, 64, 0, device="cuda")
    q = synth.queries(B, 1, H, D, 0.05, 0, device="cuda")
    d = Dims(B=B, Tq=1, H=H, D=D, HI=4, dI=64, K=8, W=16, m=m, n_entries=10, entry_cap=N, win_cap=16)
    ws = torch.zeros(csa.decode_step_workspace(d, 4), dtype=torch.uint8, device="cuda")
    q_pos = torch.tensor([41], dtype=torch.int32, device="cuda")       # (41 + 1) % 4 != 0
    csa.sync_status()
    csa.decode_step(x, z, None, q, ind.qI, ind.w, q_pos, st.codes, st.scales, st.kI, st.win_codes,
                    st.win_scales, d, st.idx, st.score, st.out, st.lse, ws)
    with pytest.raises(csa.CsaError) as e:
        csa.sync_status()
    assert e.value.code == csa.CSA_ERR_INVALID
    q_pos.fill_(39)
    csa.decode_step(x, z, None, q, ind.qI, ind.w, q_pos, st.codes, st.scales, st.kI, st.win_codes,
                    st.win_scales, d, st.idx, st.score, st.out, st.lse, ws)
    csa.sync_status()


def test_unsupported_shapes_are_refused_before_launch():
    base = dict(B=2, Tq=1, H=128, D=512, HI=4, dI=64, K=512, W=128, m=4, n_entries=1000, entry_cap=1000)
    assert csa.decode_step_workspace(Dims(**base), 4) > 0
    for k, v in [("H", 64), ("D", 256), ("dI", 32), ("Tq", 2), ("HI", 8), ("B", 200)]:
        assert csa.decode_step_workspace(Dims(**{**base, k: v}), 4) == 0, k
    assert csa.decode_step_workspace(Dims(**base), 6) == 0       # not a multiple of m
    assert csa.decode_step_workspace(Dims(**base), 32) == 0      # more than 16 new tokens
