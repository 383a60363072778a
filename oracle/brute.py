"""Scalar-loop attention on tiny shapes: a third route to the oracle's numbers.

Plain Python floats and ``math`` only, with no numpy arithmetic and no code shared with
``oracle.attention`` or ``oracle.online``. Each step is written as the loops of its
definition:
  * rotation: an explicit 2x2 rotation matrix applied to each (even, odd) feature pair,
    angle p * base**(-2i/hd) ("Write attention from scratch", worked example);
  * scores: q.k / sqrt(hd) minus slope * |i - j| for ALiBi ("Building a Multi-Head
    Self-Attention Block with RoPE and ALiBi from Scratch", Step 3 and Step 4);
  * the group's key/value rows are copied out per query head before use;
  * softmax over the allowed keys only, then the weighted sum of value rows.
Cost is O(T^2 * H * hd) Python operations: keep T, H, hd small.
"""
from __future__ import annotations

import math


def _rows(t):
    """Nested Python lists of floats from a numpy array or torch tensor."""
    if hasattr(t, "detach"):
        import torch
        t = t.detach().to("cpu", torch.float32).numpy()
    if isinstance(t, list):
        return t
    return t.tolist()


def rotate_vec(vec, p, base):
    hd = len(vec)
    out = [0.0] * hd
    for i in range(hd // 2):
        a = p * base ** (-2.0 * i / hd)
        rot = ((math.cos(a), -math.sin(a)),
               (math.sin(a), math.cos(a)))
        x, y = vec[2 * i], vec[2 * i + 1]
        out[2 * i] = rot[0][0] * x + rot[0][1] * y
        out[2 * i + 1] = rot[1][0] * x + rot[1][1] * y
    return out


def attend_one(qvec, keys, values, qpos, kpos, *, causal, window, slope):
    """Attention of one query vector over lists of (already rotated) keys and values."""
    hd = len(qvec)
    scores, kept = [], []
    for n, kvec in enumerate(keys):
        d = qpos - kpos[n]
        if causal and d < 0:
            continue
        if window > 0 and d >= window:
            continue
        s = 0.0
        for c in range(hd):
            s += qvec[c] * kvec[c]
        s /= math.sqrt(hd)
        if slope is not None:
            s -= slope * abs(d)
        scores.append(s)
        kept.append(n)
    if not kept:
        return [0.0] * hd, -math.inf
    top = max(scores)
    ws = [math.exp(s - top) for s in scores]
    tot = sum(ws)
    out = [0.0] * hd
    for w, n in zip(ws, kept):
        for c in range(hd):
            out[c] += w / tot * values[n][c]
    return out, top + math.log(tot)


def prefill(q, k, v, *, pos0=0, rope_base=0.0, causal=True, window=0, slopes=None):
    """q [B][T][H][hd], k/v [B][T][KV][hd] -> (out [B][T][H][hd], lse [B][H][T])."""
    q, k, v = _rows(q), _rows(k), _rows(v)
    B, T, H, KV = len(q), len(q[0]), len(q[0][0]), len(k[0][0])
    per_kv = H // KV
    out = [[[None] * H for _ in range(T)] for _ in range(B)]
    lse = [[[None] * T for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            g = h // per_kv
            keys = [k[b][t][g] for t in range(T)]
            vals = [v[b][t][g] for t in range(T)]
            if rope_base > 0:
                keys = [rotate_vec(keys[t], pos0 + t, rope_base) for t in range(T)]
            slope = None if slopes is None else float(slopes[h])
            for t in range(T):
                qv = q[b][t][h]
                if rope_base > 0:
                    qv = rotate_vec(qv, pos0 + t, rope_base)
                o, s = attend_one(qv, keys, vals, t, list(range(T)), causal=causal,
                                  window=window, slope=slope)
                out[b][t][h] = o
                lse[b][h][t] = s
    return out, lse


def matmul(a, w):
    """[n][k] x [k][m] with explicit loops."""
    n, kk, m = len(a), len(w), len(w[0])
    return [[sum(a[r][c] * w[c][col] for c in range(kk)) for col in range(m)] for r in range(n)]


def block(x, Wq, Wk, Wv, Wo, *, H, KV, pos0=0, rope_base=0.0, causal=True, window=0,
          slopes=None):
    """One sequence x [T][d] through projections, attention and Wo: returns [T][d]."""
    x, Wq, Wk, Wv, Wo = (_rows(a) for a in (x, Wq, Wk, Wv, Wo))
    T = len(x)
    hd = len(Wq[0]) // H
    qf, kf, vf = matmul(x, Wq), matmul(x, Wk), matmul(x, Wv)
    q = [[[qf[t][h * hd + c] for c in range(hd)] for h in range(H)] for t in range(T)]
    k = [[[kf[t][g * hd + c] for c in range(hd)] for g in range(KV)] for t in range(T)]
    v = [[[vf[t][g * hd + c] for c in range(hd)] for g in range(KV)] for t in range(T)]
    ctx, _ = prefill([q], [k], [v], pos0=pos0, rope_base=rope_base, causal=causal,
                     window=window, slopes=slopes)
    flat = [[ctx[0][t][h][c] for h in range(H) for c in range(hd)] for t in range(T)]
    return matmul(flat, Wo)


def decode(q, kcache, vcache, seqlens, qpos, *, rope_base=0.0, window=0, slopes=None):
    """q [B][H][hd] (not rotated), caches [B][Lmax][KV][hd] with keys already rotated."""
    q, kc, vc = _rows(q), _rows(kcache), _rows(vcache)
    B, H, KV = len(q), len(q[0]), len(kc[0][0])
    out, lse = [], []
    for b in range(B):
        L, p = int(seqlens[b]), int(qpos[b])
        ob, lb = [], []
        for h in range(H):
            g = h // (H // KV)
            qv = rotate_vec(q[b][h], p, rope_base) if rope_base > 0 else q[b][h]
            keys = [kc[b][j][g] for j in range(L)]
            vals = [vc[b][j][g] for j in range(L)]
            slope = None if slopes is None else float(slopes[h])
            o, s = attend_one(qv, keys, vals, p, list(range(L)), causal=False, window=window,
                              slope=slope)
            ob.append(o)
            lb.append(s)
        out.append(ob)
        lse.append(lb)
    return out, lse


def chunk(q, kcache, vcache, seqlens, qpos0, *, rope_base=0.0, causal=True, window=0, slopes=None):
    """q [B][Tq][H][hd] (not rotated), row i at position qpos0[b] + i; caches with rotated keys."""
    q, kc, vc = _rows(q), _rows(kcache), _rows(vcache)
    B, Tq, H, KV = len(q), len(q[0]), len(q[0][0]), len(kc[0][0])
    out = [[[None] * H for _ in range(Tq)] for _ in range(B)]
    lse = [[[None] * Tq for _ in range(H)] for _ in range(B)]
    for b in range(B):
        L = int(seqlens[b])
        for h in range(H):
            g = h // (H // KV)
            keys = [kc[b][j][g] for j in range(L)]
            vals = [vc[b][j][g] for j in range(L)]
            slope = None if slopes is None else float(slopes[h])
            for i in range(Tq):
                p = int(qpos0[b]) + i
                qv = rotate_vec(q[b][i][h], p, rope_base) if rope_base > 0 else q[b][i][h]
                o, s = attend_one(qv, keys, vals, p, list(range(L)), causal=causal, window=window,
                                  slope=slope)
                out[b][i][h] = o
                lse[b][h][i] = s
    return out, lse


def decode_paged(q, kpages, vpages, block_table, seqlens, qpos, *, page_size, rope_base=0.0,
                 window=0, slopes=None):
    """decode() with each cached row looked up through the block table, one slot at a time."""
    q, kp, vp = _rows(q), _rows(kpages), _rows(vpages)
    table = _rows(block_table)
    B, H, KV = len(q), len(q[0]), len(kp[0][0])
    out, lse = [], []
    for b in range(B):
        L, p = int(seqlens[b]), int(qpos[b])
        ob, lb = [], []
        for h in range(H):
            g = h // (H // KV)
            qv = rotate_vec(q[b][h], p, rope_base) if rope_base > 0 else q[b][h]
            keys, vals = [], []
            for j in range(L):
                page, row = int(table[b][j // page_size]), j % page_size
                keys.append(kp[page][row][g])
                vals.append(vp[page][row][g])
            slope = None if slopes is None else float(slopes[h])
            o, s = attend_one(qv, keys, vals, p, list(range(L)), causal=False, window=window,
                              slope=slope)
            ob.append(o)
            lb.append(s)
        out.append(ob)
        lse.append(lb)
    return out, lse
