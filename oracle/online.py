"""Tiled online-softmax attention in fp64: a second route to the oracle's numbers.

This module shares no code with ``oracle.attention``. It follows the key-block recurrences
of "Building grouped-query attention with RoPE and Flash Attention from scratch", Step 3
(running max m, running denominator l, rescaled partial output), which are the equations
of the FlashAttention section of "Building a Transformer from Scratch: Attention,
Architecture, and Memory":
    m_new = max(m, rowmax(S_blk));  alpha = exp(m - m_new)
    l_new = alpha * l + rowsum(exp(S_blk - m_new));  O = alpha * O + exp(S_blk - m_new) V_blk
and divides by l at the end. Causal, window and ALiBi terms are added per block.

Its rotary embedding uses the complex view of the same transform ("Building a
Transformer from Scratch", Part 2 "Rotary Position Embeddings"): feature pair (2i, 2i+1)
is the complex number x + iy, multiplied by exp(i * p * base**(-2i/hd)). Key/value heads
are physically repeated per query head (repeat_interleave over the head axis).
"""
from __future__ import annotations

import numpy as np


def _wide(a):
    if hasattr(a, "detach"):
        import torch
        return a.detach().to("cpu", torch.float32).numpy().astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def rotate_complex(t, positions, base):
    """t [..., n, hd] -> rotated copy; pairs as complex numbers times a unit phasor."""
    t = _wide(t)
    hd = t.shape[-1]
    z = t[..., 0::2] + 1j * t[..., 1::2]
    freq = 1.0 / base ** (np.arange(0, hd, 2) / hd)
    phase = np.exp(1j * np.outer(np.asarray(positions, dtype=np.float64), freq))
    z = z * phase
    out = np.empty(t.shape)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def flash_forward(q, k, v, *, block: int, pos0=0, rope_base=0.0, causal=True, window=0,
                  slopes=None):
    """q [B,T,H,hd], k/v [B,T,KV,hd] -> (out [B,T,H,hd], lse [B,H,T]) by key blocks."""
    q, k, v = _wide(q), _wide(k), _wide(v)
    B, T, H, hd = q.shape
    KV = k.shape[2]
    qh = np.transpose(q, (0, 2, 1, 3))
    kh = np.repeat(np.transpose(k, (0, 2, 1, 3)), H // KV, axis=1)
    vh = np.repeat(np.transpose(v, (0, 2, 1, 3)), H // KV, axis=1)
    if rope_base > 0:
        positions = np.arange(pos0, pos0 + T)
        qh = rotate_complex(qh, positions, rope_base)
        kh = rotate_complex(kh, positions, rope_base)
    scale = 1.0 / np.sqrt(hd)
    qi = np.arange(T)[:, None]
    O = np.zeros((B, H, T, hd))
    m = np.full((B, H, T), -np.inf)
    l = np.zeros((B, H, T))
    for start in range(0, T, block):
        stop = min(start + block, T)
        kj = np.arange(start, stop)[None, :]
        S = np.einsum("bhtd,bhsd->bhts", qh, kh[:, :, start:stop]) * scale
        if slopes is not None:
            S = S - np.asarray(slopes, dtype=np.float64)[None, :, None, None] * np.abs(qi - kj)
        keep = np.ones((T, stop - start), dtype=bool)
        if causal:
            keep &= kj <= qi
        if window > 0:
            keep &= kj > qi - window
        S = np.where(keep, S, -np.inf)
        m_new = np.maximum(m, S.max(axis=-1))
        ref = np.where(np.isneginf(m_new), 0.0, m_new)      # rows with nothing seen yet
        alpha = np.where(np.isneginf(m), 0.0, np.exp(m - ref))
        P = np.exp(S - ref[..., None])
        l = alpha * l + P.sum(axis=-1)
        O = alpha[..., None] * O + np.einsum("bhts,bhsd->bhtd", P, vh[:, :, start:stop])
        m = m_new
    out = O / l[..., None]
    lse = m + np.log(l)
    return np.transpose(out, (0, 2, 1, 3)), lse
