"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random tensors only; it holds none of the method's
arithmetic.  Every draw uses a torch CPU generator seeded explicitly, in a
fixed order (q, k, v, then masks or weights), so the GPU path and the CPU
oracle receive identical values.  bf16 tensors are drawn in fp32 and rounded
to bf16 once; the oracle widens those bf16 values exactly to float64.

Workloads (shapes from the LTE paper's timing setup: heads of a ~1.4B model,
batch 32, 4K-token prompts; no dataset or trained weights are used):

* ``tiny``      B=1, T=512, Hq=Hkv=4, D=64, fp32, s=4, w=64, C=32, tau=0.5,
                CNN 128->32 (k=5, +-2) -> 32->1 (k=3, +-1), weights N(0, 0.02).
* ``prefill``   B=32, T=4096, Hq=16, Hkv=4, D=128, bf16, s=4, w=512, C=512,
                retention mask Bernoulli(0.1) per (token, KV head), fed.
* ``decode``    prefill shapes, 4096-token prompt + 512 decode tokens, the
                CNN (256->32->1) scored live, tau=0.5, deferred batch 64.
* ``sweep``     B=4, T=16384, Hq=16, Hkv=4, D=128, bf16, w=1024, s=4,
                C in {0,1024,4096,16384}, rate in {0,5,25,100}%, per-KV-head
                rate ~ U[0, 2*rate] clipped to [0, 1] (100% -> every token).
* ``hybrid``    gated linear attention (16 heads, dk=dv=128, a=sigmoid(N(2,0.5)))
                + an LTE layer as ``decode``; B=32, 4096 + 256 tokens.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    dtype: torch.dtype
    sink: int
    window: int
    cap: int
    tau: float = 0.5
    mask_rate: float | None = None   # fed Bernoulli mask; None = CNN scored
    decode_steps: int = 0
    score_batch: int = 64
    c_hid: int = 32
    k1: int = 5
    past1: int = 2
    k2: int = 3
    past2: int = 1
    w_std: float = 0.02
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, T=512, Hq=4, Hkv=4, D=64, dtype=torch.float32,
                     sink=4, window=64, cap=32, tau=0.5, seed=0),
    "prefill": Workload("prefill", B=32, T=4096, Hq=16, Hkv=4, D=128, dtype=torch.bfloat16,
                        sink=4, window=512, cap=512, mask_rate=0.1, seed=1),
    "decode": Workload("decode", B=32, T=4096, Hq=16, Hkv=4, D=128, dtype=torch.bfloat16,
                       sink=4, window=512, cap=512, tau=0.5, decode_steps=512,
                       score_batch=64, seed=2),
    "sweep": Workload("sweep", B=4, T=16384, Hq=16, Hkv=4, D=128, dtype=torch.bfloat16,
                      sink=4, window=1024, cap=4096, mask_rate=0.05, seed=3),
    "hybrid": Workload("hybrid", B=32, T=4096, Hq=16, Hkv=4, D=128, dtype=torch.bfloat16,
                       sink=4, window=512, cap=512, tau=0.5, decode_steps=256,
                       score_batch=64, seed=4),
}

SWEEP_CAPS = (0, 1024, 4096, 16384)
SWEEP_RATES = (0.0, 0.05, 0.25, 1.0)


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, dtype: torch.dtype, g: torch.Generator) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, then rounded once to `dtype`."""
    x = torch.randn(*shape, generator=g, dtype=torch.float32) * std
    return x.to(dtype)


def qkv(B, T, Hq, Hkv, D, dtype, g, std=None):
    """q [B,T,Hq,D], k, v [B,T,Hkv,D] ~ N(0, 1/D) (std 1/sqrt(D) unless given)."""
    std = 1.0 / math.sqrt(D) if std is None else std
    q = normal((B, T, Hq, D), std, dtype, g)
    k = normal((B, T, Hkv, D), std, dtype, g)
    v = normal((B, T, Hkv, D), std, dtype, g)
    return q, k, v


def cnn_weights(Hkv, D, c_hid, k1, k2, g, std=0.02):
    """Per-KV-head CNN weights: w1 [Hkv,c_hid,2D,k1], b1 [Hkv,c_hid] (zeros),
    w2 [Hkv,c_hid,k2], b2 [Hkv] (zeros); fp32."""
    w1 = normal((Hkv, c_hid, 2 * D, k1), std, torch.float32, g)
    w2 = normal((Hkv, c_hid, k2), std, torch.float32, g)
    b1 = torch.zeros(Hkv, c_hid, dtype=torch.float32)
    b2 = torch.zeros(Hkv, dtype=torch.float32)
    return w1, b1, w2, b2


def bernoulli_mask(B, Hkv, T, p, g) -> torch.Tensor:
    """uint8 [B,Hkv,T], i.i.d. Bernoulli(p)."""
    u = torch.rand(B, Hkv, T, generator=g, dtype=torch.float64)
    return (u < p).to(torch.uint8)


def grid_scores(B, Hkv, T, levels, g) -> torch.Tensor:
    """fp32 [B,Hkv,T] scores drawn uniformly from {0, 1/levels, ..., (levels-1)/levels}:
    exact in fp32 (levels a power of two), with equal scores frequent when
    levels is small."""
    x = torch.randint(0, levels, (B, Hkv, T), generator=g, dtype=torch.int64)
    return x.to(torch.float32) / levels


def rate_mask(B, Hkv, T, rate, g) -> torch.Tensor:
    """Per-KV-head rates ~ U[0, 2*rate] clipped to [0,1], then Bernoulli per
    token; rate >= 1 gives every token."""
    if rate >= 1.0:
        return torch.ones(B, Hkv, T, dtype=torch.uint8)
    rates = (torch.rand(B, Hkv, 1, generator=g, dtype=torch.float64) * 2 * rate).clamp(0, 1)
    u = torch.rand(B, Hkv, T, generator=g, dtype=torch.float64)
    return (u < rates).to(torch.uint8)


def lte_inputs(wl: Workload, T: int | None = None, B: int | None = None):
    """Draw q, k, v (and the fed mask or the CNN weights) for an LTE layer.

    Returns a dict with q, k, v and either ``mask`` or ``cnn`` = (w1,b1,w2,b2).
    T defaults to the prompt plus the decode tokens.
    """
    B = wl.B if B is None else B
    T = wl.T + wl.decode_steps if T is None else T
    g = generator(wl.seed)
    q, k, v = qkv(B, T, wl.Hq, wl.Hkv, wl.D, wl.dtype, g)
    out = {"q": q, "k": k, "v": v}
    if wl.mask_rate is not None:
        out["mask"] = bernoulli_mask(B, wl.Hkv, T, wl.mask_rate, g)
    else:
        out["cnn"] = cnn_weights(wl.Hkv, wl.D, wl.c_hid, wl.k1, wl.k2, g, wl.w_std)
    return out


def gla_inputs(B, T, H, dk, dv, g, dtype=torch.bfloat16):
    """q, k [B,T,H,dk], v [B,T,H,dv] ~ N(0, 1/dk) in `dtype`;
    a [B,T,H,dk] = sigmoid(N(2, 0.5)) in fp32 (the decay gates)."""
    std = 1.0 / math.sqrt(dk)
    q = normal((B, T, H, dk), std, dtype, g)
    k = normal((B, T, H, dk), std, dtype, g)
    v = normal((B, T, H, dv), std, dtype, g)
    a = torch.sigmoid(torch.randn(B, T, H, dk, generator=g, dtype=torch.float32) * 0.5 + 2.0)
    return q, k, v, a
