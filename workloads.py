"""Seeded synthetic workloads for the attention core.

This module only draws random inputs and names the workload shapes. It holds none of
the attention arithmetic (no rotation, no softmax, no ALiBi slopes), so both the CUDA
path and the CPU oracle can take their inputs from it without sharing any of the
method.

Recipes:
  * The tiny fp32 block follows the worked example of "Write attention from scratch"
    (inside-the-model lab 2, code listing): numpy ``default_rng(0)``, drawn in the
    order x, Wq, Wk, Wv, Wo from N(0, 1), each weight divided by sqrt(d_model). The
    fp64 draws are rounded to fp32 once; both sides see those fp32 values.
  * Every bf16 workload draws N(0, 1) fp32 values from a CPU ``torch.Generator``
    seeded with the workload's seed, then rounds them to bf16 (round to nearest even).
  * Decode cache lengths are uniform integers in [1024, 8192].
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    T: int
    H: int
    KV: int
    hd: int
    causal: bool = True
    window: int = 0          # <= 0: no window; else key j allowed iff i - W < j <= i
    rope_base: float = 0.0   # <= 0: no rotary embedding
    alibi: bool = False      # ALiBi bias with the slopes 2^(-8(h+1)/H)
    pos0: int = 0
    seed: int = 0

    @property
    def allowed_pairs(self) -> int:
        """Number of allowed (query, key) pairs per (batch, head)."""
        T, W = self.T, self.window
        if not self.causal:
            if W > 0:
                raise ValueError("a window without the causal mask is not a workload here")
            return T * T
        if W <= 0 or W >= T:
            return T * (T + 1) // 2
        # rows i < W see i+1 keys, later rows see W keys
        return W * (W + 1) // 2 + (T - W) * W

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs: 2 for q.k plus 2 for p.v per allowed pair per head-dim element."""
        return 4 * self.B * self.H * self.hd * self.allowed_pairs


@dataclasses.dataclass(frozen=True)
class Decode:
    name: str
    B: int
    H: int
    KV: int
    hd: int
    Lmax: int
    len_lo: int
    len_hi: int
    rope_base: float = 10000.0
    window: int = 0
    alibi: bool = False
    seed: int = 0


@dataclasses.dataclass(frozen=True)
class Block:
    name: str
    B: int
    T: int
    d: int
    H: int
    KV: int
    hd: int
    rope_base: float = 10000.0
    causal: bool = True
    window: int = 0
    alibi: bool = False
    pos0: int = 0
    seed: int = 0

    @property
    def attention(self) -> Prefill:
        """The attention core this block runs between its projections."""
        return Prefill(self.name + "_attention", B=self.B, T=self.T, H=self.H, KV=self.KV,
                       hd=self.hd, causal=self.causal, window=self.window,
                       rope_base=self.rope_base, alibi=self.alibi, pos0=self.pos0, seed=self.seed)

    @property
    def projection_flops(self) -> int:
        """2*M*N*K of x@Wq, x@Wk, x@Wv and ctx@Wo, with M = B*T rows."""
        M = self.B * self.T
        return 2 * M * self.d * (self.H + 2 * self.KV) * self.hd + 2 * M * self.H * self.hd * self.d

    @property
    def flops(self) -> int:
        return self.projection_flops + self.attention.flops


@dataclasses.dataclass(frozen=True)
class Chunk:
    """Tq query rows of each sequence at positions qpos0 .. qpos0+Tq-1, attending a cache that
    holds the sequence's first qpos0 + Tq keys (causal)."""
    name: str
    B: int
    Tq: int
    qpos0: int
    Lmax: int
    H: int
    KV: int
    hd: int
    rope_base: float = 10000.0
    seed: int = 0

    @property
    def allowed_pairs(self) -> int:
        """Allowed (query, key) pairs per (batch, head): row i sees qpos0 + i + 1 keys."""
        return self.Tq * self.qpos0 + self.Tq * (self.Tq + 1) // 2

    @property
    def flops(self) -> int:
        return 4 * self.B * self.H * self.hd * self.allowed_pairs


@dataclasses.dataclass(frozen=True)
class Latent:
    """A latent-attention decode step: a cache of dc-number latents per token and per-head
    up-projections [H, dc, hd]; cache lengths uniform in [len_lo, len_hi]."""
    name: str
    B: int
    H: int
    hd: int
    dc: int
    Lmax: int
    len_lo: int
    len_hi: int
    seed: int = 0


# The workloads of this library, named by what they are.
TINY_BLOCK = Block("tiny_block_fp32_T6_d32_H4_KV2_hd8", B=1, T=6, d=32, H=4, KV=2, hd=8,
                   rope_base=10000.0, causal=True, seed=0)
MHA_ROPE = Prefill("mha_prefill_bf16_B4_T1024_H16_hd64_rope", B=4, T=1024, H=16, KV=16, hd=64,
                   rope_base=10000.0, seed=1)
MHA_ALIBI = Prefill("mha_prefill_bf16_B4_T1024_H16_hd64_alibi", B=4, T=1024, H=16, KV=16, hd=64,
                    rope_base=0.0, alibi=True, seed=1)
GQA = Prefill("gqa_prefill_bf16_B2_T4096_H32_KV8_hd128", B=2, T=4096, H=32, KV=8, hd=128,
              rope_base=500000.0, seed=2)
LONG_WINDOW = Prefill("long_gqa_prefill_bf16_B1_T16384_H32_KV8_hd128_W4096", B=1, T=16384, H=32,
                      KV=8, hd=128, window=4096, rope_base=10000.0, seed=3)
DECODE_GQA = Decode("decode_bf16_B64_H32_KV8_hd128_L1024-8192", B=64, H=32, KV=8, hd=128,
                    Lmax=8192, len_lo=1024, len_hi=8192, seed=4)
DECODE_MQA = Decode("decode_bf16_B64_H32_KV1_hd128_L1024-8192", B=64, H=32, KV=1, hd=128,
                    Lmax=8192, len_lo=1024, len_hi=8192, seed=5)
LATENT_DECODE = Latent("latent_decode_bf16_B64_H32_hd128_dc128_L1024-8192", B=64, H=32, hd=128, dc=128,
                       Lmax=8192, len_lo=1024, len_hi=8192, seed=8)
# The second half of the GQA prefill's sequences as a chunk over a cache of their 4096 keys.
GQA_CHUNK = Chunk("gqa_chunk_bf16_B2_Tq2048_at2048_H32_KV8_hd128", B=2, Tq=2048, qpos0=2048,
                  Lmax=4096, H=32, KV=8, hd=128, rope_base=500000.0, seed=7)
# A Llama-style bf16 block whose attention is the GQA prefill's shape (d_model 4096).
GQA_BLOCK = Block("gqa_block_bf16_B2_T4096_d4096_H32_KV8_hd128", B=2, T=4096, d=4096, H=32, KV=8,
                  hd=128, rope_base=500000.0, causal=True, seed=6)

PREFILLS = {w.name: w for w in (MHA_ROPE, MHA_ALIBI, GQA, LONG_WINDOW)}
DECODES = {w.name: w for w in (DECODE_GQA, DECODE_MQA)}


def tiny_block_inputs(seed: int = 0, T: int = 6, d: int = 32, H: int = 4, KV: int = 2):
    """Inputs of the lab's worked example, rounded once to fp32.

    Returns a dict of fp32 numpy arrays: x [T, d], Wq [d, H*hd], Wk/Wv [d, KV*hd], Wo [H*hd, d].
    """
    hd = d // H
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d))
    Wq = rng.normal(size=(d, H * hd)) / np.sqrt(d)
    Wk = rng.normal(size=(d, KV * hd)) / np.sqrt(d)
    Wv = rng.normal(size=(d, KV * hd)) / np.sqrt(d)
    Wo = rng.normal(size=(H * hd, d)) / np.sqrt(d)
    return {n: a.astype(np.float32) for n, a in
            (("x", x), ("Wq", Wq), ("Wk", Wk), ("Wv", Wv), ("Wo", Wo))}


def normal(shape, seed: int, dtype=torch.bfloat16, gen: Optional[torch.Generator] = None):
    """N(0,1) fp32 draws from a seeded CPU generator, rounded to ``dtype`` (RNE)."""
    if gen is None:
        gen = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)


def prefill_inputs(w: Prefill, dtype=torch.bfloat16):
    """q [B,T,H,hd], k and v [B,T,KV,hd]: N(0,1) drawn in the order q, k, v from one generator."""
    gen = torch.Generator().manual_seed(w.seed)
    q = normal((w.B, w.T, w.H, w.hd), w.seed, dtype, gen)
    k = normal((w.B, w.T, w.KV, w.hd), w.seed, dtype, gen)
    v = normal((w.B, w.T, w.KV, w.hd), w.seed, dtype, gen)
    return q, k, v


def block_inputs(w: Block, dtype=torch.bfloat16):
    """x [B,T,d] ~ N(0,1); Wq [d,H*hd], Wk/Wv [d,KV*hd], Wo [H*hd,d] ~ N(0,1)/sqrt(d), drawn in
    the order x, Wq, Wk, Wv, Wo from one generator (the lab's order and scaling)."""
    gen = torch.Generator().manual_seed(w.seed)
    x = normal((w.B, w.T, w.d), w.seed, dtype, gen)
    scale = 1.0 / float(np.sqrt(w.d))
    Ws = {}
    for n, shape in (("Wq", (w.d, w.H * w.hd)), ("Wk", (w.d, w.KV * w.hd)),
                     ("Wv", (w.d, w.KV * w.hd)), ("Wo", (w.H * w.hd, w.d))):
        Ws[n] = (torch.randn(*shape, generator=gen, dtype=torch.float32) * scale).to(dtype)
    return x, Ws


def chunk_inputs(w: Chunk, dtype=torch.bfloat16):
    """q [B,Tq,H,hd] (the chunk's queries, not rotated) and k, v [B,qpos0+Tq,KV,hd] (the keys
    and values of every position up to the chunk's end, not rotated), drawn in that order."""
    gen = torch.Generator().manual_seed(w.seed)
    n = w.qpos0 + w.Tq
    q = normal((w.B, w.Tq, w.H, w.hd), w.seed, dtype, gen)
    k = normal((w.B, n, w.KV, w.hd), w.seed, dtype, gen)
    v = normal((w.B, n, w.KV, w.hd), w.seed, dtype, gen)
    return q, k, v


def latent_inputs(w: Latent, dtype=torch.bfloat16):
    """seqlens [B]; q [B,H,hd]; latent cache [B,Lmax,dc] (N(0,1) below each length, zero above);
    W_uk, W_uv [H,dc,hd] ~ N(0,1)/sqrt(dc); drawn in that order."""
    gen = torch.Generator().manual_seed(w.seed)
    seqlens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=gen, dtype=torch.int32)
    q = normal((w.B, w.H, w.hd), w.seed, dtype, gen)
    c = torch.zeros(w.B, w.Lmax, w.dc, dtype=dtype)
    for b in range(w.B):
        L = int(seqlens[b])
        c[b, :L] = normal((L, w.dc), 0, dtype, gen)
    scale = 1.0 / float(np.sqrt(w.dc))
    W_uk = (torch.randn(w.H, w.dc, w.hd, generator=gen) * scale).to(dtype)
    W_uv = (torch.randn(w.H, w.dc, w.hd, generator=gen) * scale).to(dtype)
    return q, c, W_uk, W_uv, seqlens


def decode_lengths(w: Decode) -> torch.Tensor:
    gen = torch.Generator().manual_seed(w.seed)
    return torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=gen, dtype=torch.int32)


def decode_inputs(w: Decode, dtype=torch.bfloat16, fill_unused: bool = False):
    """Decode inputs: q [B,H,hd] (not rotated), caches [B,Lmax,KV,hd], seqlens [B], qpos [B].

    Cache slots below each sequence's length hold N(0,1) draws; keys there are taken as
    already rotated at their slot position. Slots at or above the length are zero unless
    ``fill_unused`` (they are never read). The new query sits at position ``len``.
    """
    gen = torch.Generator().manual_seed(w.seed)
    seqlens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=gen, dtype=torch.int32)
    q = normal((w.B, w.H, w.hd), w.seed, dtype, gen)
    kc = torch.zeros(w.B, w.Lmax, w.KV, w.hd, dtype=dtype)
    vc = torch.zeros(w.B, w.Lmax, w.KV, w.hd, dtype=dtype)
    for b in range(w.B):
        L = int(seqlens[b]) if not fill_unused else w.Lmax
        kc[b, :L] = normal((L, w.KV, w.hd), 0, dtype, gen)
        vc[b, :L] = normal((L, w.KV, w.hd), 0, dtype, gen)
    qpos = seqlens.clone()
    return q, kc, vc, seqlens, qpos


def small_prefill(B, T, H, KV, hd, seed, dtype=torch.bfloat16, **flags) -> Prefill:
    """A parity-test case with the same recipe as the named workloads."""
    return Prefill(f"case_B{B}_T{T}_H{H}_KV{KV}_hd{hd}_s{seed}", B=B, T=T, H=H, KV=KV, hd=hd,
                   seed=seed, **flags)
