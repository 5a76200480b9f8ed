"""Host orchestration of the hybrid-attention path over the C ABI.

Nothing here computes: each function allocates caller-side buffers with
torch (device memory) and sequences the library's asynchronous calls on the
current CUDA stream.

* :func:`prefill` -- CSA over a whole sequence: pool every m-token block into
  the FP8 cache, store every token as a window entry, run the indexer + top-k
  for every position and attend.
* :class:`DecodeState` -- a decode-time cache (compressed entries, indexer
  keys, a window ring of ``win_cap`` tokens) that grows by one compressed
  entry per ``m`` appended tokens, with :meth:`DecodeState.step` running one
  append + query step (CSA: index, top-k, attend -- one fused launch when the
  shape allows it; HCA: dense attend).
"""
from __future__ import annotations

import dataclasses

import torch

from . import (Dims, attend, attend_workspace, compress, compress_ew, decode_step, decode_step_workspace, hca_attend,
               index_topk, index_topk_workspace)


def prefer_fused_step(B: int, device=None) -> bool:
    """Whether one csa_decode_step launch beats the separate calls for B
    sequences.  The fused step's attention phase gives each (sequence,
    quarter of D) unit SMs // (4 * B) CTAs; measured on B200 it wins with
    at least four per unit (4 sequences: 58 vs 61 us per 1M-context step)
    and loses with two (16 sequences: 76 vs 63 us per 64K-context step)."""
    sms = torch.cuda.get_device_properties(device or torch.cuda.current_device()).multi_processor_count
    return 16 * B <= sms


def _ws(nbytes: int, device) -> torch.Tensor | None:
    return torch.empty(nbytes, dtype=torch.uint8, device=device) if nbytes else None


@dataclasses.dataclass
class PrefillResult:
    out: torch.Tensor        # bf16 [B, T, H, D]
    lse: torch.Tensor        # f32 [B, T, H]
    idx: torch.Tensor        # int32 [B, T, K]
    score: torch.Tensor      # f32 [B, T, K]
    codes: torch.Tensor      # u8 [B, N, D]
    scales: torch.Tensor     # f32 [B, N]
    win_codes: torch.Tensor  # u8 [B, T, D]
    win_scales: torch.Tensor  # f32 [B, T]


def prefill(x, z, q, qI, w, kI, *, m: int, K: int, W: int, softmax_scale: float = 1.0,
            pooled: torch.Tensor | None = None) -> PrefillResult:
    """CSA prefill: every position 0..T-1 of each sequence is a query.

    x, z: f32 [B, T, D]; q: bf16 [B, T, H, D]; qI: u8 [B, T, HI, dI/2];
    w: f32 [B, T, HI]; kI: u8 [B, T // m, dI/2].
    """
    B, T, D = x.shape
    H = q.shape[2]
    HI, dI = qI.shape[2], 2 * qI.shape[3]
    dev = x.device
    N = T // m
    codes = torch.empty((B, N, D), dtype=torch.uint8, device=dev)
    scales = torch.empty((B, N), dtype=torch.float32, device=dev)
    win_codes = torch.empty((B, T, D), dtype=torch.uint8, device=dev)
    win_scales = torch.empty((B, T), dtype=torch.float32, device=dev)
    compress_ew(x, z, m, codes, scales, win_codes, win_scales, pooled=pooled)
    q_pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    dims = Dims(B=B, Tq=T, H=H, D=D, HI=HI, dI=dI, K=K, W=W, m=m, n_entries=N, entry_cap=N,
                win_cap=T, softmax_scale=softmax_scale)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    score = torch.empty((B, T, K), dtype=torch.float32, device=dev)
    index_topk(qI, w, kI, q_pos, dims, idx, score, workspace=_ws(index_topk_workspace(dims), dev))
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    attend(q, codes, scales, idx, win_codes, win_scales, q_pos, dims, out, lse,
           workspace=_ws(attend_workspace(dims), dev))
    return PrefillResult(out, lse, idx, score, codes, scales, win_codes, win_scales)


class DecodeState:
    """Decode cache for B sequences: compressed entries, indexer keys and a
    window ring.  Capacity is fixed at construction (``entry_cap`` entries).

    ``dense=True`` makes it an HCA cache (no indexer, dense attention).
    ``fused=True`` runs each CSA step as one csa_decode_step launch where
    the shape allows it; ``fused=False`` always uses the separate calls;
    ``fused=None`` (the default) picks by :func:`prefer_fused_step`.
    """

    def __init__(self, B: int, D: int, H: int, m: int, W: int, entry_cap: int, *, K: int = 512,
                 HI: int = 4, dI: int = 64, win_cap: int | None = None, dense: bool = False,
                 softmax_scale: float = 1.0, device="cuda", fused: bool | None = None):
        self.B, self.D, self.H, self.m, self.W, self.K = B, D, H, m, W, K
        self.HI, self.dI, self.dense = HI, dI, dense
        self.win_cap = W if win_cap is None else win_cap
        self.entry_cap = entry_cap
        self.softmax_scale = softmax_scale
        self.device = torch.device(device)
        dev = self.device
        self.codes = torch.zeros((B, entry_cap, D), dtype=torch.uint8, device=dev)
        self.scales = torch.ones((B, entry_cap), dtype=torch.float32, device=dev)
        self.win_codes = torch.zeros((B, self.win_cap, D), dtype=torch.uint8, device=dev)
        self.win_scales = torch.ones((B, self.win_cap), dtype=torch.float32, device=dev)
        self.kI = None if dense else torch.zeros((B, entry_cap, dI // 2), dtype=torch.uint8, device=dev)
        self.n_tokens = 0
        self.q_pos = torch.zeros((B, 1), dtype=torch.int32, device=dev)
        self.idx = None if dense else torch.empty((B, 1, K), dtype=torch.int32, device=dev)
        self.score = None if dense else torch.empty((B, 1, K), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, 1, H, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, 1, H), dtype=torch.float32, device=dev)
        self._ws_index = None
        self._ws_attend = None
        self._ws_step = None
        self._side = None
        if fused is None:
            fused = prefer_fused_step(B, self.device)
        self.fused = fused and not dense

    @property
    def n_entries(self) -> int:
        return self.n_tokens // self.m

    def dims(self, n_tokens: int | None = None) -> Dims:
        n = self.n_tokens if n_tokens is None else n_tokens
        return Dims(B=self.B, Tq=1, H=self.H, D=self.D, HI=self.HI, dI=self.dI, K=self.K, W=self.W,
                    m=self.m, n_entries=n // self.m, entry_cap=self.entry_cap,
                    win_cap=self.win_cap, softmax_scale=self.softmax_scale)

    def step_workspace(self, n_new: int) -> torch.Tensor | None:
        """The zero-filled workspace of the fused step for n_new appended
        tokens (grown when needed), or None if the shape is not fused."""
        nb = decode_step_workspace(self.dims(self.n_tokens + n_new), n_new)
        if not nb:
            return None
        if self._ws_step is None or self._ws_step.numel() < nb:
            self._ws_step = torch.zeros(nb, dtype=torch.uint8, device=self.device)
        return self._ws_step

    def prefill_context(self, x: torch.Tensor, z: torch.Tensor, T: int, kI: torch.Tensor | None = None):
        """Compress tokens [0, T) of x, z [B, >=T, D] into the cache (setup).

        kI (u8 [B, >= T//m, dI/2]) gives the indexer keys of those entries.
        """
        assert self.n_tokens == 0 and T // self.m <= self.entry_cap
        compress(x, z, self.m, self.codes, self.scales, T=T)
        lo = max(0, T - self.win_cap)
        if T > lo:
            compress(x[:, lo:T].contiguous(), z[:, lo:T].contiguous(), 1, self.win_codes,
                     self.win_scales, dst_first=lo, ring_cap=self.win_cap)
        if kI is not None and self.kI is not None:
            self.kI[:, : T // self.m].copy_(kI[:, : T // self.m])
        self.n_tokens = T

    def append(self, x_new: torch.Tensor, z_new: torch.Tensor, kI_new: torch.Tensor | None = None):
        """Append n tokens (x_new, z_new: f32 [B, n, D], n a multiple of m when the
        cache is block aligned): completed blocks become entries, every token
        enters the window ring.  kI_new (u8 [B, n//m, dI/2]) are the new
        entries' indexer keys."""
        n = x_new.shape[1]
        assert self.n_tokens % self.m == 0 and n % self.m == 0
        first = self.n_entries
        assert first + n // self.m <= self.entry_cap
        compress_ew(x_new, z_new, self.m, self.codes, self.scales, self.win_codes, self.win_scales,
                    dst_first=first, win_first=self.n_tokens, win_ring_cap=self.win_cap)
        if kI_new is not None and self.kI is not None:
            self.kI[:, first:first + n // self.m].copy_(kI_new)
        self.n_tokens += n

    def query(self, q: torch.Tensor, qI: torch.Tensor | None = None, w: torch.Tensor | None = None,
              after: torch.cuda.Stream | None = None):
        """One query per sequence at position n_tokens - 1.  q: bf16 [B, 1, H, D];
        qI: u8 [B, 1, HI, dI/2], w: f32 [B, 1, HI] (CSA only).  The attention
        waits for the stream `after` (if given)."""
        self.q_pos.fill_(self.n_tokens - 1)
        d = self.dims()
        if self.dense:
            nb = attend_workspace(d, True)
            if nb and (self._ws_attend is None or self._ws_attend.numel() < nb):
                self._ws_attend = _ws(nb, self.device)
            hca_attend(q, self.codes, self.scales, self.win_codes, self.win_scales, self.q_pos, d,
                       self.out, self.lse, workspace=self._ws_attend)
            return self.out, self.lse
        nb = index_topk_workspace(d)
        if nb and (self._ws_index is None or self._ws_index.numel() < nb):
            self._ws_index = _ws(nb, self.device)
        index_topk(qI, w, self.kI, self.q_pos, d, self.idx, self.score, workspace=self._ws_index)
        if after is not None:
            torch.cuda.current_stream(self.device).wait_stream(after)
        nb = attend_workspace(d, False)
        if nb and (self._ws_attend is None or self._ws_attend.numel() < nb):
            self._ws_attend = _ws(nb, self.device)
        attend(q, self.codes, self.scales, self.idx, self.win_codes, self.win_scales, self.q_pos, d,
               self.out, self.lse, workspace=self._ws_attend)
        return self.out, self.lse

    def step(self, x_new, z_new, q, qI=None, w=None, kI_new=None):
        """Append tokens then run one query per sequence at the newest position.

        CSA: one csa_decode_step launch (append, index, select, attend) when
        the shape is in its set and ``fused`` is on.  Otherwise the separate
        calls: the new entries' indexer keys are stored first; the compression
        of the new tokens (needed only by the attention) runs on a side stream
        beside the indexer, and the attention waits for both."""
        if self.dense:
            self.append(x_new, z_new, kI_new)
            return self.query(q, qI, w)
        n = x_new.shape[1]
        ws = self.step_workspace(n) if self.fused else None
        if ws is not None:
            assert self.n_tokens % self.m == 0 and n % self.m == 0
            assert (self.n_tokens + n) // self.m <= self.entry_cap
            self.q_pos.fill_(self.n_tokens + n - 1)
            decode_step(x_new, z_new, kI_new, q, qI, w, self.q_pos, self.codes, self.scales, self.kI,
                        self.win_codes, self.win_scales, self.dims(self.n_tokens + n), self.idx, self.score,
                        self.out, self.lse, ws)
            self.n_tokens += n
            return self.out, self.lse
        main = torch.cuda.current_stream(self.device)
        if self._side is None:
            self._side = torch.cuda.Stream(device=self.device)
        side = self._side
        n = x_new.shape[1]
        assert self.n_tokens % self.m == 0 and n % self.m == 0
        first = self.n_entries
        assert first + n // self.m <= self.entry_cap
        if kI_new is not None and self.kI is not None:
            self.kI[:, first:first + n // self.m].copy_(kI_new)
        side.wait_stream(main)
        with torch.cuda.stream(side):
            compress_ew(x_new, z_new, self.m, self.codes, self.scales, self.win_codes, self.win_scales,
                        dst_first=first, win_first=self.n_tokens, win_ring_cap=self.win_cap)
        x_new.record_stream(side)
        z_new.record_stream(side)
        self.n_tokens += n
        return self.query(q, qI, w, after=side)
