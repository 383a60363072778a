"""The attention core written out as its plain definition, in fp64 (test infrastructure).

Sources (page title, then the place on the page):
  [LAB]   "Write attention from scratch" (Inside the Model, lab 2): the worked example
          (rope, softmax, attention), Property 1, Property 2, exercises 2 and 3.
  [ALIBI] "Building a Multi-Head Self-Attention Block with RoPE and ALiBi from Scratch",
          Step 3 "Implement ALiBi Bias" and Step 4.
  [GQA3]  "Building grouped-query attention with RoPE and Flash Attention from scratch",
          Step 3 (repeat_interleave of K/V over the head axis).
  [XF5]   "Building a Transformer from Scratch: Attention, Architecture, and Memory",
          Part 1 step 2 (stable softmax, causal mask) and Part 3 "KV caching".

Readings where the pages are silent or disagree (each listed in the design notes):
  * RoPE pairs are interleaved (even, odd) features; the angle of pair i at position p is
    p * base**(-2 i / hd) [LAB rope]. Positions of a prefill are pos0 .. pos0+T-1.
  * ALiBi adds -slope_h * |i - j| to the scaled score; slopes are 2**(-8 (h+1) / H).
  * Masked pairs are excluded (weight exactly zero), as the -inf mask of [LAB] does.
  * The sliding window of width W keeps keys j with i - W < j <= i (W <= 0: no window).
  * Query head h reads key/value head h // (H // KV) [LAB np.repeat; GQA3].
  * A query with no allowed key (only possible for a decode step over an empty cache)
    returns zeros and log-sum-exp -inf.
All arithmetic is fp64; inputs are widened from the exact values the GPU sees.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    """Widen a numpy array or a CPU torch tensor (fp32 or bf16) to fp64, exactly."""
    if hasattr(a, "detach"):  # torch tensor; bf16 has no numpy dtype, go through fp32
        import torch
        return a.detach().to("cpu", torch.float32).numpy().astype(F64)
    return np.asarray(a, dtype=F64)


def rope(t, positions, base: float) -> np.ndarray:
    """Rotary embedding of ``t`` [..., n, hd] at ``positions`` (length n), [LAB] rope.

    Features (2i, 2i+1) form a pair that is turned by the angle p * base**(-2i/hd):
    (x, y) -> (x cos a - y sin a, x sin a + y cos a).
    """
    t = _f64(t)
    hd = t.shape[-1]
    if hd % 2:
        raise ValueError("rotary embedding needs an even head dimension")
    p = np.asarray(positions, dtype=F64).reshape(-1, 1)          # [n, 1]
    pair = np.arange(hd // 2, dtype=F64).reshape(1, -1)           # [1, hd/2]
    angle = p * np.power(float(base), -2.0 * pair / hd)           # [n, hd/2]
    cos, sin = np.cos(angle), np.sin(angle)
    pairs = t.reshape(t.shape[:-1] + (hd // 2, 2))
    x, y = pairs[..., 0], pairs[..., 1]
    turned = np.stack((x * cos - y * sin, x * sin + y * cos), axis=-1)
    return turned.reshape(t.shape)


def alibi_slopes(H: int) -> np.ndarray:
    """ALiBi head slopes 2**(-8 (h+1) / H), h = 0..H-1 (geometric, first term 2**(-8/H))."""
    h = np.arange(H, dtype=F64)
    return np.power(2.0, -8.0 * (h + 1.0) / H)


def _allowed(i, j, causal: bool, window: int) -> np.ndarray:
    """Boolean mask of allowed (query position i, key position j) pairs (broadcasting)."""
    ok = np.ones(np.broadcast(i, j).shape, dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= (i - j) < window
    return ok


def _masked_softmax_rows(s: np.ndarray, ok: np.ndarray):
    """Softmax over the last axis restricted to ``ok``; returns (weights, lse).

    The row maximum is subtracted before exponentiating ([LAB] softmax; [XF5] Part 1).
    A row with no allowed entry gets all-zero weights and lse = -inf.
    """
    s = np.where(ok, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    m = np.where(empty, 0.0, m)
    e = np.where(ok, np.exp(s - m), 0.0)
    denom = e.sum(axis=-1, keepdims=True)
    safe = np.where(denom > 0, denom, 1.0)
    w = e / safe
    with np.errstate(divide="ignore"):
        lse = np.where(denom[..., 0] > 0, m[..., 0] + np.log(safe[..., 0]), -np.inf)
    return w, lse


def attention(q, k, v, *, pos0: int = 0, rope_base: float = 0.0, causal: bool = True,
              window: int = 0, slopes=None, rows=None, heads=None):
    """softmax(q k^T / sqrt(hd) + bias, masked) v for every query head, in fp64.

    q [B,T,H,hd]; k, v [B,T,KV,hd]. ``rope_base`` <= 0 turns the rotation off; ``slopes``
    (H values) turns ALiBi on. ``rows`` / ``heads`` restrict which query rows / heads are
    computed (each row is independent), for shapes whose full score matrix is too large.
    Returns out [B, R, Hs, hd] and lse [B, Hs, R] over the selected rows R and heads Hs.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, hd = q.shape
    KV = k.shape[2]
    if H % KV:
        raise ValueError("H must be a multiple of KV")
    group = H // KV
    rows = np.arange(T) if rows is None else np.asarray(rows)
    heads = np.arange(H) if heads is None else np.asarray(heads)
    pos = pos0 + np.arange(T)
    qh = q.transpose(0, 2, 1, 3)                      # [B,H,T,hd]
    kh = k.transpose(0, 2, 1, 3)                      # [B,KV,T,hd]
    vh = v.transpose(0, 2, 1, 3)
    if rope_base > 0:
        qh = rope(qh[:, :, rows], pos[rows], rope_base)
        kh = rope(kh, pos, rope_base)
    else:
        qh = qh[:, :, rows]
    i = rows.reshape(-1, 1)                           # query index within the sequence
    j = np.arange(T).reshape(1, -1)
    ok = _allowed(i, j, causal, window)
    out = np.zeros((B, len(rows), len(heads), hd))
    lse = np.zeros((B, len(heads), len(rows)))
    for b in range(B):
        for n, h in enumerate(heads):
            g = h // group                            # key/value head serving query head h
            s = qh[b, h] @ kh[b, g].T / np.sqrt(hd)
            if slopes is not None:
                s = s - float(slopes[h]) * np.abs(i - j)
            w, lse[b, n] = _masked_softmax_rows(s, ok)
            out[b, :, n] = w @ vh[b, g]
    return out, lse


def decode(q, kcache, vcache, seqlens, qpos, *, rope_base: float = 0.0, window: int = 0,
           slopes=None):
    """One decode step per sequence over a cache ([XF5] "KV caching"; [LAB] exercise 2).

    q [B,H,hd] is the new token's query before rotation; it is turned at position
    ``qpos[b]``. kcache, vcache [B,Lmax,KV,hd] hold keys already rotated at their slot
    index; slots 0..seqlens[b]-1 are attended to (the query sees every cached key; the
    window, if any, keeps slots j with qpos - j < W). Returns out [B,H,hd], lse [B,H].
    """
    q = _f64(q)
    B, H, hd = q.shape
    KV = kcache.shape[2]
    group = H // KV
    out = np.zeros((B, H, hd))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        p = int(qpos[b])
        if L == 0:
            continue
        kb = _f64(kcache[b, :L])                      # [L,KV,hd]
        vb = _f64(vcache[b, :L])
        qb = q[b]
        if rope_base > 0:
            qb = rope(qb[:, None, :], [p], rope_base)[:, 0, :]
        j = np.arange(L)
        ok = (p - j) < window if window > 0 else np.ones(L, dtype=bool)
        for h in range(H):
            g = h // group
            s = kb[:, g] @ qb[h] / np.sqrt(hd)
            if slopes is not None:
                s = s - float(slopes[h]) * np.abs(p - j)
            w, row_lse = _masked_softmax_rows(s[None, :], ok[None, :])
            lse[b, h] = row_lse[0]
            out[b, h] = (w @ vb[:, g])[0]
    return out, lse


def gather_pages(pages, block_table, L: int, page_size: int, b: int) -> np.ndarray:
    """Slots 0..L-1 of sequence b from a paged cache: slot j lives in row j % page_size of
    page block_table[b][j // page_size]. pages [num_pages, page_size, KV, hd]."""
    pages = _f64(pages)
    j = np.arange(L)
    page = np.asarray(block_table)[b][j // page_size]
    return pages[page, j % page_size]                          # [L, KV, hd]


def decode_paged(q, kpages, vpages, block_table, seqlens, qpos, *, page_size: int,
                 rope_base: float = 0.0, window: int = 0, slopes=None):
    """decode() over a paged cache: the cache of sequence b is its pages in block-table order
    (the serving layout the pages' PagedAttention mention stands for). Returns out, lse."""
    B = len(seqlens)
    Lmax = max(1, max(int(x) for x in seqlens))
    KV, hd = kpages.shape[2], kpages.shape[3]
    kc = np.zeros((B, Lmax, KV, hd))
    vc = np.zeros((B, Lmax, KV, hd))
    for b in range(B):
        L = int(seqlens[b])
        kc[b, :L] = gather_pages(kpages, block_table, L, page_size, b)
        vc[b, :L] = gather_pages(vpages, block_table, L, page_size, b)
    return decode(q, kc, vc, seqlens, qpos, rope_base=rope_base, window=window, slopes=slopes)


def latent_decode(q, ccache, W_uk, W_uv, seqlens, qpos, *, window: int = 0, slopes=None):
    """Decode over a latent cache, unfolded ([LAB] exercise 5, latent attention): each cached
    token holds a latent c_j [dc]; head h's key and value are c_j W_uk[h] and c_j W_uv[h]
    (W_uk, W_uv [H, dc, hd]). No rotary embedding on this path (a position rotation between c
    and W_uk would not fold into the query). q [B,H,hd]; ccache [B,Lmax,dc].
    Returns out [B,H,hd], lse [B,H]."""
    q, c = _f64(q), _f64(ccache)
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    B, H, hd = q.shape
    out = np.zeros((B, H, hd))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L, p = int(seqlens[b]), int(qpos[b])
        if L == 0:
            continue
        j = np.arange(L)
        ok = (p - j) < window if window > 0 else np.ones(L, dtype=bool)
        for h in range(H):
            k = c[b, :L] @ W_uk[h]                             # [L, hd]
            v = c[b, :L] @ W_uv[h]
            s = k @ q[b, h] / np.sqrt(hd)
            if slopes is not None:
                s = s - float(slopes[h]) * np.abs(p - j)
            w, row_lse = _masked_softmax_rows(s[None, :], ok[None, :])
            lse[b, h] = row_lse[0]
            out[b, h] = (w @ v)[0]
    return out, lse


def latent_decode_folded(q, ccache, W_uk, W_uv, seqlens, qpos, *, window: int = 0, slopes=None):
    """The same with the key up-projection folded into the query ([LAB] exercise 5): scores
    (W_uk[h] q_h) . c_j / sqrt(hd) against the latent itself, and the value up-projection
    applied once to the weighted latent sum. Returns out [B,H,hd], lse [B,H]."""
    q, c = _f64(q), _f64(ccache)
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    B, H, hd = q.shape
    out = np.zeros((B, H, hd))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L, p = int(seqlens[b]), int(qpos[b])
        if L == 0:
            continue
        j = np.arange(L)
        ok = (p - j) < window if window > 0 else np.ones(L, dtype=bool)
        for h in range(H):
            qlat = W_uk[h] @ q[b, h]                           # [dc]
            s = c[b, :L] @ qlat / np.sqrt(hd)
            if slopes is not None:
                s = s - float(slopes[h]) * np.abs(p - j)
            w, row_lse = _masked_softmax_rows(s[None, :], ok[None, :])
            lse[b, h] = row_lse[0]
            out[b, h] = (w @ c[b, :L])[0] @ W_uv[h]
    return out, lse


def kv_write(k_new, v_new, kcache, vcache, pos0, *, rope_base: float = 0.0):
    """Write a chunk of keys and values into the cache ([XF5] "KV caching"), in fp64.

    k_new, v_new [B,Tn,KV,hd]; row t of sequence b goes to slot pos0[b] + t, its key turned
    at that position (slots are positions). Returns the updated caches (fp64 copies).
    """
    kc, vc = _f64(kcache).copy(), _f64(vcache).copy()
    k_new, v_new = _f64(k_new), _f64(v_new)
    B, Tn = k_new.shape[:2]
    for b in range(B):
        p = int(pos0[b]) + np.arange(Tn)
        kb = k_new[b].transpose(1, 0, 2)                       # [KV,Tn,hd]
        if rope_base > 0:
            kb = rope(kb, p, rope_base)
        kc[b, p] = kb.transpose(1, 0, 2)
        vc[b, p] = v_new[b]
    return kc, vc


def chunk(q, kcache, vcache, seqlens, qpos0, *, rope_base: float = 0.0, causal: bool = True,
          window: int = 0, slopes=None):
    """A chunk of queries against a cache: prefill that continues a sequence ([XF5] "KV
    caching"; [LAB] exercise 2 with several new tokens at once).

    q [B,Tq,H,hd] before rotation; row i of sequence b sits at position qpos0[b] + i and is
    turned there. kcache, vcache [B,Lmax,KV,hd] hold keys already rotated at their slot;
    slots 0..seqlens[b]-1 are candidates, and (query position P, slot j) is allowed under the
    same causal / window rule as a prefill: j <= P, P - j < W. ALiBi adds -slope_h |P - j|.
    Returns out [B,Tq,H,hd] and lse [B,H,Tq]; a row with no allowed slot gets zeros, -inf.
    """
    q = _f64(q)
    B, Tq, H, hd = q.shape
    KV = kcache.shape[2]
    group = H // KV
    out = np.zeros((B, Tq, H, hd))
    lse = np.full((B, H, Tq), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        P = int(qpos0[b]) + np.arange(Tq)                    # query positions
        qb = q[b].transpose(1, 0, 2)                         # [H,Tq,hd]
        if rope_base > 0:
            qb = rope(qb, P, rope_base)
        if L == 0:
            continue
        kb = _f64(kcache[b, :L]).transpose(1, 0, 2)          # [KV,L,hd]
        vb = _f64(vcache[b, :L]).transpose(1, 0, 2)
        i = P.reshape(-1, 1)
        j = np.arange(L).reshape(1, -1)
        ok = _allowed(i, j, causal, window)
        for h in range(H):
            g = h // group
            s = qb[h] @ kb[g].T / np.sqrt(hd)
            if slopes is not None:
                s = s - float(slopes[h]) * np.abs(i - j)
            w, lse[b, h] = _masked_softmax_rows(s, ok)
            out[b, :, h] = w @ vb[g]
    return out, lse


def rmsnorm(x, gamma, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm ([XF5] "RMSNorm and Pre-LN residuals"): x / sqrt(mean(x^2) + eps) * gamma over
    the last axis."""
    x, gamma = _f64(x), _f64(gamma)
    rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x / rms * gamma


def block_fused(x, gamma, Wqkv, Wo, *, H: int, KV: int, pos0: int = 0, rope_base: float = 0.0,
                causal: bool = True, window: int = 0, slopes=None, eps: float = 1e-6, rows=None):
    """The attention sub-layer of a pre-norm decoder block ([XF5] "RMSNorm and Pre-LN
    residuals": x + attn(norm(x))): RMSNorm, one projection x_n @ Wqkv whose columns are
    [q heads | k heads | v heads] (Wqkv [d, (H + 2 KV) hd]), attention, ctx @ Wo, plus x.
    Returns out [B,T,d] and the rows a cache keeps: k turned at positions pos0.., v [B,T,KV,hd].
    ``rows`` (query row indices) restricts out to those rows: out [B,len(rows),d]."""
    x = _f64(x)
    Wqkv, Wo = _f64(Wqkv), _f64(Wo)
    B, T, d = x.shape
    hd = Wqkv.shape[1] // (H + 2 * KV)
    qkv = rmsnorm(x, gamma, eps) @ Wqkv
    q = qkv[..., :H * hd].reshape(B, T, H, hd)
    k = qkv[..., H * hd:(H + KV) * hd].reshape(B, T, KV, hd)
    v = qkv[..., (H + KV) * hd:].reshape(B, T, KV, hd)
    ctx, _ = attention(q, k, v, pos0=pos0, rope_base=rope_base, causal=causal, window=window,
                       slopes=slopes, rows=rows)
    R = T if rows is None else len(rows)
    out = (x if rows is None else x[:, np.asarray(rows)]) + ctx.reshape(B, R, H * hd) @ Wo
    kc = k.transpose(0, 2, 1, 3)                                 # [B,KV,T,hd]
    if rope_base > 0:
        kc = rope(kc, pos0 + np.arange(T), rope_base)
    return out, kc.transpose(0, 2, 1, 3), v


def block(x, Wq, Wk, Wv, Wo, *, H: int, KV: int, pos0: int = 0, rope_base: float = 0.0,
          causal: bool = True, window: int = 0, slopes=None, rows=None):
    """Projections, attention and output projection of [LAB] attention(): x [B,T,d] -> [B,T,d].

    Weights are [in, out] and applied as x @ W; head h is columns h*hd .. h*hd+hd-1 of
    x @ Wq (the reshape to heads of [LAB]). No bias, residual or normalisation. ``rows``
    (query row indices) restricts the result to those rows: [B,len(rows),d].
    """
    x = _f64(x)
    Wq, Wk, Wv, Wo = (_f64(w) for w in (Wq, Wk, Wv, Wo))
    B, T, d = x.shape
    hd = Wq.shape[1] // H
    q = (x @ Wq).reshape(B, T, H, hd)
    k = (x @ Wk).reshape(B, T, KV, hd)
    v = (x @ Wv).reshape(B, T, KV, hd)
    ctx, _ = attention(q, k, v, pos0=pos0, rope_base=rope_base, causal=causal, window=window,
                       slopes=slopes, rows=rows)
    return ctx.reshape(B, T if rows is None else len(rows), H * hd) @ Wo
