"""Seeded synthetic inputs for the Gated Delta Rule forward.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no normalisation, no cumulative sums, no decay), so both
the CUDA path's tests and the oracle can take their inputs from it.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in a fixed order -- sequence lengths (when random), q, k, v, g, beta, initial
states, slot indices -- and only then moved to the requested device, so a
given (config, seed) yields bit-identical values on any machine.

The named workloads follow the shapes and distributions of the operator's
published configuration ranges (Qwen3Next Samples: T up to 1M+, B up to 128,
Nqk in {2, 4, 16}, Nv in {4, 8, 32}, D = L = 128) and the decode page's example
recipe (beta = U*0.9 + 0.05, g = -(U + 0.01)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

D = 128


@dataclass
class GdnInputs:
    name: str
    q: torch.Tensor            # bf16 [T, Nqk, 128]
    k: torch.Tensor            # bf16 [T, Nqk, 128]
    v: torch.Tensor            # bf16 [T, Nv, 128]
    g: torch.Tensor            # fp32 [T, Nv]   log-space gate (negative)
    beta: torch.Tensor         # bf16 [T, Nv]
    cu_seqlens: torch.Tensor   # int32 [B+1]
    state_pool: Optional[torch.Tensor]     # fp32 [P, Nv, 128, 128] (Dk, Dv) or None
    state_indices: Optional[torch.Tensor]  # int32 [B] or None
    scale: float
    eps: float
    seqlens: list = field(default_factory=list)

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    @property
    def B(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def Nqk(self) -> int:
        return int(self.q.shape[1])

    @property
    def Nv(self) -> int:
        return int(self.v.shape[1])

    @property
    def P(self) -> int:
        return 0 if self.state_pool is None else int(self.state_pool.shape[0])

    @property
    def max_seqlen(self) -> int:
        return max(self.seqlens) if self.seqlens else 0

    def to(self, device) -> "GdnInputs":
        mv = lambda t: None if t is None else t.to(device)
        return GdnInputs(self.name, mv(self.q), mv(self.k), mv(self.v), mv(self.g), mv(self.beta),
                         mv(self.cu_seqlens), mv(self.state_pool), mv(self.state_indices),
                         self.scale, self.eps, list(self.seqlens))


# name -> recipe.  "lens": list of sequence lengths or ("uniform", lo, hi, B).
# "g": ("uniform_neg", a, b) => g = -(U*a + b); ("softplus", c) => g = -softplus(N(0,1))*c
# "beta": ("uniform", lo, hi) or ("sigmoid",);  "state": None or ("normal", std, P, "identity"|"perm")
CONFIGS = {
    # one sequence of two full chunks
    "single_s256": dict(lens=[256], Nqk=2, Nv=4, g=("uniform_neg", 0.5, 0.01),
                        beta=("uniform", 0.05, 0.95), state=None, seed=0),
    # packed varlen batch with ragged tails and per-sequence initial states
    "varlen_b4": dict(lens=[1000, 513, 128, 2407], Nqk=4, Nv=8, g=("uniform_neg", 0.5, 0.01),
                      beta=("uniform", 0.05, 0.95), state=("normal", 0.02, None, "identity"), seed=1),
    # one layer's prefill at Qwen3-Next head counts
    "prefill_s32k": dict(lens=[32768], Nqk=16, Nv=32, g=("softplus", 0.1),
                         beta=("sigmoid",), state=None, seed=2),
    # 256 short sequences reading their initial states from a 512-slot pool
    "short_pool_b256": dict(lens=("uniform", 1, 8, 256), Nqk=16, Nv=32, g=("uniform_neg", 1.0, 0.01),
                            beta=("uniform", 0.05, 0.95), state=("normal", 0.02, 512, "perm"), seed=3),
    # two 128K-token sequences with initial states
    "long_s128k_b2": dict(lens=[131072, 131072], Nqk=16, Nv=32, g=("softplus", 0.05),
                          beta=("sigmoid",), state=("normal", 0.02, None, "identity"), seed=4),
    # decode step: 256 sequences of one token on a bf16 pool, with the key-dimension gate (key_gate)
    "decode_b256_bf16": dict(lens=[1] * 256, Nqk=16, Nv=32, g=("uniform_neg", 1.0, 0.01),
                             beta=("uniform", 0.05, 0.95), state=("normal", 0.02, 512, "perm"), seed=6),
    # the decode page's example shape (Dk = 64, Dv = 512, 64 heads), one token for each of 128 sequences
    "decode_dk64_dv512": dict(lens=[1] * 128, Nqk=64, Nv=64, g=("uniform_neg", 1.0, 0.01),
                              beta=("uniform", 0.05, 0.95), state=("normal", 0.02, 256, "perm"), seed=7,
                              Dk=64, Dv=512),
    # speculative decoding: 256 sequences of 4 draft tokens, a pool slot per token (see spec_slots)
    "spec_decode_b256x4": dict(lens=[4] * 256, Nqk=16, Nv=32, g=("uniform_neg", 1.0, 0.01),
                               beta=("uniform", 0.05, 0.95), state=("normal", 0.02, 1024, "perm"), seed=5),
}


def spec_slots(inp: GdnInputs, seed: int):
    """Token slots and accepted counts for a speculative step: every token gets its own pool slot
    (a random permutation of the pool's first T slots) and sequence b accepts a uniform 1..n_b of
    its tokens.  Returns (token_slots int32 [T], num_accepted int32 [B]) on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    T, B = inp.T, inp.B
    P = inp.state_pool.shape[0]
    if P < T:
        raise ValueError("the pool needs a slot per token")
    slots = torch.randperm(P, generator=gen)[:T].to(torch.int32)
    n = (inp.cu_seqlens[1:] - inp.cu_seqlens[:-1]).to(torch.int64)
    acc = (torch.floor(torch.rand(B, generator=gen) * n.clamp(min=1)).to(torch.int64) + 1).clamp(max=n.clamp(min=1))
    return slots, acc.to(torch.int32)


def _draw_lens(spec, gen):
    if isinstance(spec, (list, tuple)) and spec and spec[0] == "uniform":
        _, lo, hi, B = spec
        return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=gen)]
    return [int(x) for x in spec]


def make(lens, Nqk, Nv, g=("uniform_neg", 0.5, 0.01), beta=("uniform", 0.05, 0.95), state=None,
         seed=0, name="custom", scale=None, eps=1e-6, device="cpu", Dk=D, Dv=D) -> GdnInputs:
    """Draw one batch.  See CONFIGS for the recipe keys.  Dk, Dv: head dimensions (the chunked path
    takes 128 only; the token recurrence on a pool also takes Dk = 64 and other Dv)."""
    gen = torch.Generator().manual_seed(seed)
    seqlens = _draw_lens(lens, gen)
    B = len(seqlens)
    T = sum(seqlens)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    if B:
        cu[1:] = torch.tensor(seqlens, dtype=torch.int64).cumsum(0).to(torch.int32)
    q = torch.randn(T, Nqk, Dk, generator=gen).to(torch.bfloat16)
    k = torch.randn(T, Nqk, Dk, generator=gen).to(torch.bfloat16)
    v = torch.randn(T, Nv, Dv, generator=gen).to(torch.bfloat16)
    if g[0] == "uniform_neg":
        gg = -(torch.rand(T, Nv, generator=gen) * g[1] + g[2])
    elif g[0] == "softplus":
        gg = -torch.nn.functional.softplus(torch.randn(T, Nv, generator=gen)) * g[1]
    elif g[0] == "zero":
        gg = torch.zeros(T, Nv)
    else:
        raise ValueError(g)
    if beta[0] == "uniform":
        bb = torch.rand(T, Nv, generator=gen) * (beta[2] - beta[1]) + beta[1]
    elif beta[0] == "sigmoid":
        bb = torch.sigmoid(torch.randn(T, Nv, generator=gen))
    elif beta[0] == "const":
        bb = torch.full((T, Nv), float(beta[1]))
    else:
        raise ValueError(beta)
    pool = idx = None
    if state is not None:
        _, std, P, mode = state
        P = B if P is None else P
        pool = torch.randn(P, Nv, Dk, Dv, generator=gen) * std
        if mode == "identity":
            idx = torch.arange(B, dtype=torch.int32)
        elif mode == "perm":
            idx = torch.randperm(P, generator=gen)[:B].to(torch.int32)
        else:
            raise ValueError(mode)
    if scale is None:
        scale = 1.0 / math.sqrt(Dk)
    inp = GdnInputs(name, q, k, v, gg.float().contiguous(), bb.to(torch.bfloat16), cu, pool, idx,
                    float(scale), float(eps), seqlens)
    return inp if str(device) == "cpu" else inp.to(device)


def config(name: str, device="cpu", seed: Optional[int] = None) -> GdnInputs:
    """Inputs of a named workload (see CONFIGS)."""
    rec = dict(CONFIGS[name])
    if seed is not None:
        rec["seed"] = seed
    return make(name=name, device=device, **rec)


def key_gate(inp: GdnInputs, seed: int) -> torch.Tensor:
    """The decode page's key-dimension gate for a batch: gk [T, Nv, Dk] fp32 = -(U + 0.01) * 0.5
    (the page's example draws -(U + 0.01); the factor keeps e^gk away from tiny values)."""
    gen = torch.Generator().manual_seed(seed)
    return -(torch.rand(inp.T, inp.Nv, inp.q.shape[2], generator=gen) + 0.01) * 0.5
