"""Seeded synthetic inputs for the compressed-attention workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no pooling, no quantisation, no scores).  Both the CUDA
library's tests/bench and the CPU oracle consume the SAME tensors produced
here: they are generated once (on the host for small cases, on the GPU for
the large ones) and copied to wherever they are needed.

Distributions follow the workload definitions of this library:
* raw token values x and gate logits z: N(0, 1), fp32;
* queries: N(0, 1) * q_scale, rounded to bf16 by torch's cast;
* indexer queries / keys: uniform over the 15 distinct E2M1 values
  (the code 0x8, negative zero, is never drawn), packed two per byte with the
  even element in the low nibble;
* indexer head weights: k/16 with k uniform in {0, ..., 16};
* (attention-only tests) compressed-cache bytes: uniform over the 254 finite
  E4M3 codes, with per-entry scales uniform in [0.5, 1.5) / 448.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math

import torch

# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic workload.

    kind: "prefill" (every position 0..T-1 is a query),
          "decode"  (one query per sequence at position T-1),
          "hca_decode" (dense HCA, one query at T-1),
          "decode_incremental" (decode with 4 appended tokens per step).
    """

    name: str
    kind: str
    B: int
    T: int
    m: int
    K: int
    W: int
    H: int
    D: int
    HI: int
    dI: int
    q_scale: float
    steps: int = 1

    @property
    def N(self) -> int:
        return self.T // self.m

    @property
    def Tq(self) -> int:
        return self.T if self.kind == "prefill" else 1


WORKLOADS = {
    "tiny_prefill": Workload("tiny_prefill", "prefill", B=1, T=512, m=4, K=16, W=32, H=4, D=64,
                             HI=2, dI=32, q_scale=1.0 / 8.0),
    "csa_decode_64k": Workload("csa_decode_64k", "decode", B=16, T=65536, m=4, K=512, W=128, H=128,
                               D=512, HI=4, dI=64, q_scale=1.0 / math.sqrt(512.0)),
    "hca_decode_1m": Workload("hca_decode_1m", "hca_decode", B=16, T=1 << 20, m=128, K=0, W=128,
                              H=128, D=512, HI=0, dI=0, q_scale=1.0 / math.sqrt(512.0)),
    "csa_prefill_128k": Workload("csa_prefill_128k", "prefill", B=1, T=131072, m=4, K=512, W=128,
                                 H=64, D=512, HI=4, dI=64, q_scale=1.0 / math.sqrt(512.0)),
    "csa_decode_1m_incremental": Workload("csa_decode_1m_incremental", "decode_incremental", B=4,
                                          T=1 << 20, m=4, K=512, W=128, H=128, D=512, HI=4, dI=64,
                                          q_scale=1.0 / math.sqrt(512.0), steps=64),
}


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------


def _gen(seed: int, tag: str, device) -> torch.Generator:
    """A torch generator whose seed depends on (seed, tag) only."""
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def normal(shape, seed: int, tag: str, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """fp32 N(0, scale^2) samples, generated in chunks to bound peak memory."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    g = _gen(seed, tag, device)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n].normal_(0.0, 1.0, generator=g)
    if scale != 1.0:
        out.mul_(scale)
    return out


def tokens(B: int, T: int, D: int, seed: int, device="cpu", tag: str = "kv"):
    """Raw token values x and per-channel gate logits z, both fp32 [B, T, D]."""
    x = normal((B, T, D), seed, tag + ":x", device)
    z = normal((B, T, D), seed, tag + ":z", device)
    return x, z


def queries(B: int, Tq: int, H: int, D: int, q_scale: float, seed: int, device="cpu",
            tag: str = "q") -> torch.Tensor:
    """Attention queries, bf16 [B, Tq, H, D], from N(0, 1) * q_scale."""
    return normal((B, Tq, H, D), seed, tag, device, q_scale).to(torch.bfloat16)


# E2M1 codes of the 15 distinct values (negative zero, 0x8, excluded)
_E2M1_CODES = torch.tensor([0, 1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15], dtype=torch.uint8)


def e2m1_packed(shape_prefix, d: int, seed: int, tag: str, device="cpu") -> torch.Tensor:
    """Packed E2M1 codes u8 [*shape_prefix, d/2]; values uniform over 15 codes."""
    assert d % 2 == 0
    g = _gen(seed, tag, device)
    r = torch.randint(0, 15, tuple(shape_prefix) + (d,), generator=g, device=device, dtype=torch.int64)
    c = _E2M1_CODES.to(device)[r]
    return (c[..., 0::2] | (c[..., 1::2] << 4)).contiguous()


def indexer_weights(B: int, Tq: int, HI: int, seed: int, device="cpu", tag: str = "w") -> torch.Tensor:
    """Indexer head weights fp32 [B, Tq, HI]: k/16, k uniform in 0..16."""
    g = _gen(seed, tag, device)
    k = torch.randint(0, 17, (B, Tq, HI), generator=g, device=device, dtype=torch.int64)
    return k.to(torch.float32) / 16.0


def e4m3_cache(B: int, N: int, D: int, seed: int, device="cpu", tag: str = "cache"):
    """Random compressed-cache bytes: codes u8 [B, N, D] over the 254 finite
    E4M3 patterns, scales fp32 [B, N] uniform in [0.5, 1.5) / 448."""
    g = _gen(seed, tag + ":codes", device)
    r = torch.randint(0, 254, (B, N, D), generator=g, device=device, dtype=torch.int32)
    # skip the two NaN patterns 0x7F and 0xFF
    r = r + (r >= 0x7F).to(torch.int32)
    codes = r.to(torch.uint8)
    g2 = _gen(seed, tag + ":scales", device)
    scales = (torch.rand((B, N), generator=g2, device=device) + 0.5) / 448.0
    return codes, scales


@dataclasses.dataclass
class IndexerInputs:
    qI: torch.Tensor   # u8 [B, Tq, HI, dI/2]
    w: torch.Tensor    # f32 [B, Tq, HI]
    kI: torch.Tensor   # u8 [B, Ncap, dI/2]


def indexer_inputs(B: int, Tq: int, Ncap: int, HI: int, dI: int, seed: int, device="cpu") -> IndexerInputs:
    return IndexerInputs(
        qI=e2m1_packed((B, Tq, HI), dI, seed, "qI", device),
        w=indexer_weights(B, Tq, HI, seed, device),
        kI=e2m1_packed((B, Ncap), dI, seed, "kI", device),
    )


@dataclasses.dataclass
class IndexerInputsMX:
    qI: torch.Tensor   # u8 [B, Tq, HI, dI/2]  E2M1 codes
    qs: torch.Tensor   # u8 [B, Tq, HI, dI/32] UE8M0 block scales
    w: torch.Tensor    # f32 [B, Tq, HI]        non-negative
    kI: torch.Tensor   # u8 [B, Ncap, dI/2]
    ks: torch.Tensor   # u8 [B, Ncap, dI/32]


def ue8m0_codes(shape, seed: int, tag: str, device="cpu", spread: int = 8) -> torch.Tensor:
    """Block scale codes 127 + u, u uniform in [-spread, spread] (scales
    2^-spread .. 2^spread around 1)."""
    g = _gen(seed, tag + ":scales", device)
    u = torch.randint(-spread, spread + 1, shape, generator=g, device=device, dtype=torch.int32)
    return (127 + u).to(torch.uint8)


def indexer_inputs_mx(B: int, Tq: int, Ncap: int, HI: int, dI: int, seed: int, device="cpu",
                      spread: int = 8) -> IndexerInputsMX:
    """MXFP4 indexer inputs: E2M1 codes as `indexer_inputs`, one UE8M0 scale
    per 32 elements drawn by `ue8m0_codes`, weights uniform in [0, 1)."""
    g = _gen(seed, "wmx", device)
    return IndexerInputsMX(
        qI=e2m1_packed((B, Tq, HI), dI, seed, "qI", device),
        qs=ue8m0_codes((B, Tq, HI, dI // 32), seed, "qI", device, spread),
        w=torch.rand((B, Tq, HI), generator=g, device=device),
        kI=e2m1_packed((B, Ncap), dI, seed, "kI", device),
        ks=ue8m0_codes((B, Ncap, dI // 32), seed, "kI", device, spread),
    )
