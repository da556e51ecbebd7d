"""Seeded synthetic decode-step inputs, shared by the tests, the smoke check and
the benchmark.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no projection, scoring, selection or attention), so the
oracle and the CUDA path can both consume the bytes it produces without
sharing any computation.

Workload shapes follow the method pages' evaluation models (LLaMA-3.1-8B-like
GQA layers, a Gemma-like hybrid global/sliding-window layer and a
DeepSeek-like MLA latent cache).  The pages' datasets and trained weights are
not available, so seeded Gaussian tensors with the same layouts stand in:

* ``plain``   q, K, V ~ N(0, 1).
* ``spiked``  per (batch, KV head) a random unit direction u; every query head
  of the group gets q = N(0, I) + q_spike * u; a random 1 % of the tokens
  (drawn without replacement) get K = N(0, I) + k_spike * u, the other keys
  K = N(0, I); V ~ N(0, 1).  The spikes make the top-k a real competition.
* ``P``       per KV head the orthonormal Q factor of a d x r Gaussian
  (sign-fixed so that diag(R) > 0), stored fp32.  It stands in for the
  calibrated basis, whose data and objective are not available.

Values are drawn in fp32 and rounded once to the storage dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_BASE = 20261202


@dataclass
class Workload:
    """Shape of one decode-step workload (one attention layer)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int  # cached tokens per sequence (seq_len of every batch row)
    r: int
    k: int
    dv: int | None = None  # value width; None = d
    kind: str = "spiked"  # "plain" | "spiked"
    latent: bool = False  # V is the first dv dims of the K row (MLA latent cache)
    window: int = 0  # sliding window of the local layer (hybrid workload), 0 = none
    T_cap: int | None = None  # cache capacity; None = T
    seed: int = SEED_BASE
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def Dv(self) -> int:
        return self.d if self.dv is None else self.dv

    @property
    def cap(self) -> int:
        return self.T if self.T_cap is None else self.T_cap

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The five workloads of the method's decode-step evaluation, as synthetic shapes.
WORKLOADS = {
    "gqa_4k_b1": Workload("gqa_4k_b1", B=1, Hq=32, Hkv=8, d=128, T=4096, r=32, k=256, kind="plain",
                          seed=SEED_BASE + 0),
    "gqa_32k_b4": Workload("gqa_32k_b4", B=4, Hq=32, Hkv=8, d=128, T=32768, r=32, k=256, seed=SEED_BASE + 1),
    "gqa_128k_b16": Workload("gqa_128k_b16", B=16, Hq=32, Hkv=8, d=128, T=131072, r=32, k=256,
                             seed=SEED_BASE + 2),
    "hybrid_global_128k_b8": Workload("hybrid_global_128k_b8", B=8, Hq=16, Hkv=2, d=256, T=131072, r=64,
                                      k=256, window=1024, seed=SEED_BASE + 3),
    "mla_64k_b8": Workload("mla_64k_b8", B=8, Hq=128, Hkv=1, d=576, dv=512, T=65536, r=64, k=2048,
                           latent=True, seed=SEED_BASE + 4),
}


def make_basis(Hkv: int, d: int, r: int, seed: int) -> torch.Tensor:
    """Per-KV-head orthonormal d x r basis (fp32, CPU): Q of a Gaussian's QR."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn(Hkv, d, r, generator=g, dtype=torch.float64)
    Q, R = torch.linalg.qr(A)
    sgn = torch.sign(torch.diagonal(R, dim1=-2, dim2=-1))
    sgn[sgn == 0] = 1.0
    return (Q * sgn.unsqueeze(-2)).to(torch.float32).contiguous()


def _randn(shape, g, device, dtype):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def make_inputs(w: Workload, device="cpu", dtype=torch.bfloat16, q_spike=2.0, k_spike=3.0,
                spike_frac=0.01, seq_lens=None):
    """Draw (q, K, V, P, seq_lens) for workload ``w`` on ``device``.

    K is [B, T_cap, Hkv, d]; V is [B, T_cap, Hkv, dv] (None for a latent
    cache, where V aliases K); q is [B, Hq, d]; P is [Hkv, d, r] fp32 on
    ``device``; seq_lens is int32 [B] (default: T for every row).  Rows past
    seq_lens are drawn too, so that capacity tails hold finite values."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    B, Hq, Hkv, d, cap = w.B, w.Hq, w.Hkv, w.d, w.cap
    G = w.G
    q = _randn((B, Hq, d), g, dev, torch.float32)
    K = torch.empty((B, cap, Hkv, d), device=dev, dtype=dtype)
    V = None if w.latent else torch.empty((B, cap, Hkv, w.Dv), device=dev, dtype=dtype)
    for b in range(B):  # one batch row at a time bounds the fp32 temporaries
        K[b] = _randn((cap, Hkv, d), g, dev, dtype)
        if V is not None:
            V[b] = _randn((cap, Hkv, w.Dv), g, dev, dtype)
    if w.kind == "spiked":
        nspike = int(math.floor(spike_frac * w.T))
        for b in range(B):
            for h in range(Hkv):
                u = torch.randn(d, generator=g, device=dev, dtype=torch.float32)
                u = u / torch.linalg.vector_norm(u)
                q[b, h * G:(h + 1) * G, :] += q_spike * u
                if nspike > 0:
                    sel = torch.randperm(w.T, generator=g, device=dev)[:nspike]
                    rows = K[b, sel, h, :].to(torch.float32) + k_spike * u
                    K[b, sel, h, :] = rows.to(dtype)
    elif w.kind != "plain":
        raise ValueError("unknown workload kind %r" % w.kind)
    q = q.to(dtype).contiguous()
    P = make_basis(Hkv, d, w.r, w.seed + 7919).to(dev)
    if seq_lens is None:
        seq_lens = torch.full((B,), w.T, dtype=torch.int32, device=dev)
    else:
        seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32, device=dev)
    return q, K, V, P, seq_lens


def make_queries(w: Workload, n: int, device="cpu", dtype=torch.bfloat16, seed_offset=1):
    """n extra query tensors [B, Hq, d] ~ N(0, 1) (for multi-step timing)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed + 104729 * seed_offset)
    return [_randn((w.B, w.Hq, w.d), g, dev, dtype).contiguous() for _ in range(n)]
