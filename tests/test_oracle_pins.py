"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test states the passage or closed form it checks. Together they are chosen so that
a plausible slip anywhere in the oracle (a dropped term, a wrong sign or index, a
transposed operand) fails at least one of them; ``test_oracle_mutants.py`` plants such
slips and checks that they are caught.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import attention as A
from oracle import brute, online
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


# ----------------------------------------------------------------------------- rotary
def _read_rope_fixture(golden_dir):
    cases = []
    with open(os.path.join(golden_dir, "rope_closed_forms.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            lhs, rhs = line.split("->")
            hd, base, p, *vec = lhs.split()
            cases.append((int(hd), float(base), int(p), [float(x) for x in vec],
                          [float(x) for x in rhs.split()]))
    return cases


def test_rope_closed_forms(golden_dir):
    """Unit vectors turned by the printed angle formula (worked example, rope())."""
    cases = _read_rope_fixture(golden_dir)
    assert len(cases) >= 5
    for hd, base, p, vec, expect in cases:
        got = A.rope(np.array([vec]), [p], base)[0]
        np.testing.assert_allclose(got, expect, rtol=0, atol=1e-15)


def test_rope_identity_at_zero_and_norm():
    t = _rand((3, 7, 16), 1)
    np.testing.assert_array_equal(A.rope(t, np.zeros(7), 10000.0), t)   # R(0) = I
    r = A.rope(t, np.arange(50, 57), 10000.0)
    # each 2-D pair keeps its length, hence the whole vector too
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(t, axis=-1), rtol=1e-14)
    pr = r.reshape(3, 7, 8, 2)
    pt = t.reshape(3, 7, 8, 2)
    np.testing.assert_allclose(np.hypot(pr[..., 0], pr[..., 1]), np.hypot(pt[..., 0], pt[..., 1]),
                               rtol=1e-14)


def test_rope_relative():
    """R(p)q . R(p')k depends on p' - p only (Part 2 of the Transformer page: RoPE is relative)."""
    q, k = _rand((1, 32), 2), _rand((1, 32), 3)
    for p, dp in [(0, 5), (17, 5), (1000, 5), (3, -2), (250, -2)]:
        ref = A.rope(q, [0], 500000.0) @ A.rope(k, [dp], 500000.0).T
        got = A.rope(q, [p], 500000.0) @ A.rope(k, [p + dp], 500000.0).T
        assert abs(got - ref).max() < 1e-12


def test_rope_matches_complex_view():
    """Real 2x2 form equals the complex-phasor form of the same rotation."""
    t = _rand((2, 9, 12), 4)
    pos = np.arange(100, 109)
    np.testing.assert_allclose(A.rope(t, pos, 10000.0), online.rotate_complex(t, pos, 10000.0),
                               rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- ALiBi
def test_alibi_slopes_fixture(golden_dir):
    with open(os.path.join(golden_dir, "alibi_slopes.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for H, h, val in rows:
        assert A.alibi_slopes(int(H))[int(h)] == pytest.approx(float(val), rel=1e-15)


def test_alibi_geometric_weights():
    """q = 0 leaves only the bias: causal weights fall as exp(-slope * distance)."""
    T = hd = 6
    q = np.zeros((1, T, 1, hd))
    k = _rand((1, T, 1, hd), 5)
    v = np.eye(T)[None, :, None, :]                   # value j is the j-th unit vector
    slope = 0.3
    out, lse = A.attention(q, k, v, causal=True, slopes=[slope])
    for i in range(T):
        w = np.array([math.exp(-slope * (i - j)) for j in range(i + 1)])
        np.testing.assert_allclose(out[0, i, 0, :i + 1], w / w.sum(), rtol=1e-14)
        assert np.all(out[0, i, 0, i + 1:] == 0.0)
        assert lse[0, 0, i] == pytest.approx(math.log(w.sum()), rel=1e-14)
    # nearer keys weigh more: the sign of the bias
    assert out[0, T - 1, 0, T - 1] > out[0, T - 1, 0, 0]


# ----------------------------------------------------------------------------- closed forms
def test_window_one_returns_own_value():
    """Window of one key: each row attends to itself only, out_i = v_i (exactly)."""
    q, k, v = _rand((2, 9, 4, 8), 6), _rand((2, 9, 2, 8), 7), _rand((2, 9, 2, 8), 8)
    out, _ = A.attention(q, k, v, rope_base=10000.0, window=1)
    np.testing.assert_array_equal(out, np.repeat(v, 2, axis=2))


def test_single_token():
    q, k, v = _rand((1, 1, 4, 8), 9), _rand((1, 1, 4, 8), 10), _rand((1, 1, 4, 8), 11)
    out, _ = A.attention(q, k, v, rope_base=10000.0, slopes=A.alibi_slopes(4))
    np.testing.assert_array_equal(out, v)


def test_zero_query_prefix_mean():
    """q = 0 and no bias: uniform weights, so row i is the mean of v_0..v_i."""
    T = 7
    q = np.zeros((1, T, 2, 4))
    k, v = _rand((1, T, 1, 4), 12), _rand((1, T, 1, 4), 13)
    out, lse = A.attention(q, k, v, rope_base=10000.0)
    for i in range(T):
        np.testing.assert_allclose(out[0, i, 0], v[0, :i + 1, 0].mean(0), rtol=1e-14)
        assert lse[0, 1, i] == pytest.approx(math.log(i + 1), rel=1e-14, abs=1e-15)
    # the window of W >= T changes nothing; W = 3 averages the last three rows
    out_w, _ = A.attention(q, k, v, rope_base=10000.0, window=3)
    np.testing.assert_allclose(out_w[0, 5, 0], v[0, 3:6, 0].mean(0), rtol=1e-14)
    out_big, _ = A.attention(q, k, v, rope_base=10000.0, window=T)
    np.testing.assert_array_equal(out_big, out)


def test_weights_sum_to_one():
    """With v = all ones every output is exactly one (up to rounding): the weights sum to 1."""
    q, k = _rand((2, 11, 4, 8), 14), _rand((2, 11, 2, 8), 15)
    v = np.ones((2, 11, 2, 8))
    out, _ = A.attention(q, k, v, rope_base=10000.0, window=4, slopes=A.alibi_slopes(4))
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_scale_is_inverse_sqrt_hd():
    """Two keys, one query: the weight ratio is exp((q.k0 - q.k1)/sqrt(hd)) (no rope)."""
    hd = 16
    q = np.zeros((1, 2, 1, hd)); q[0, 1, 0, 0] = 3.0
    k = np.zeros((1, 2, 1, hd)); k[0, 0, 0, 0] = 1.0; k[0, 1, 0, 0] = -1.0
    v = np.zeros((1, 2, 1, hd)); v[0, 0, 0, 0] = 1.0; v[0, 1, 0, 1] = 1.0
    out, _ = A.attention(q, k, v)
    w0, w1 = out[0, 1, 0, 0], out[0, 1, 0, 1]
    assert w0 / w1 == pytest.approx(math.exp(6.0 / math.sqrt(hd)), rel=1e-14)


# ----------------------------------------------------------------------------- routes agree
FLAGS = [
    dict(rope_base=10000.0, causal=True, window=0, alibi=False),
    dict(rope_base=0.0, causal=True, window=0, alibi=True),
    dict(rope_base=500000.0, causal=True, window=3, alibi=False),
    dict(rope_base=10000.0, causal=True, window=2, alibi=True),
    dict(rope_base=10000.0, causal=False, window=0, alibi=True),
    dict(rope_base=0.0, causal=False, window=0, alibi=False),
]


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("shape", [(1, 5, 4, 2, 8), (2, 7, 4, 1, 6), (1, 8, 3, 3, 4)])
def test_brute_force_agrees(flags, shape):
    """Scalar loops with explicit rotation matrices and copied K/V give the same result."""
    B, T, H, KV, hd = shape
    q, k, v = _rand((B, T, H, hd), 20), _rand((B, T, KV, hd), 21), _rand((B, T, KV, hd), 22)
    slopes = A.alibi_slopes(H) if flags["alibi"] else None
    kw = dict(pos0=3, rope_base=flags["rope_base"], causal=flags["causal"],
              window=flags["window"], slopes=slopes)
    out, lse = A.attention(q, k, v, **kw)
    bo, bl = brute.prefill(q, k, v, **kw)
    np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)


@pytest.mark.parametrize("block", [1, 3, 128])
@pytest.mark.parametrize("flags", FLAGS[:4])
def test_online_softmax_equals_full(block, flags):
    """Tiled online softmax (key blocks of 1, 3, 128) equals the full softmax to ~1e-13."""
    B, T, H, KV, hd = 2, 37, 4, 2, 16
    q, k, v = _rand((B, T, H, hd), 30), _rand((B, T, KV, hd), 31), _rand((B, T, KV, hd), 32)
    slopes = A.alibi_slopes(H) if flags["alibi"] else None
    kw = dict(pos0=11, rope_base=flags["rope_base"], causal=flags["causal"],
              window=flags["window"], slopes=slopes)
    out, lse = A.attention(q, k, v, **kw)
    oo, ol = online.flash_forward(q, k, v, block=block, **kw)
    np.testing.assert_allclose(out, oo, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, ol, rtol=0, atol=1e-13)


def test_gqa_equals_mha_with_repeated_heads():
    """GQA with KV heads = MHA on K/V repeated in contiguous groups; KV=H is MHA, KV=1 is MQA."""
    B, T, H, hd = 1, 9, 8, 8
    q = _rand((B, T, H, hd), 40)
    for KV in (8, 4, 2, 1):
        k, v = _rand((B, T, KV, hd), 41 + KV), _rand((B, T, KV, hd), 51 + KV)
        out, _ = A.attention(q, k, v, rope_base=10000.0)
        krep = np.stack([k[:, :, h * KV // H] for h in range(H)], axis=2)
        vrep = np.stack([v[:, :, h * KV // H] for h in range(H)], axis=2)
        mha, _ = A.attention(q, krep, vrep, rope_base=10000.0)
        np.testing.assert_array_equal(out, mha)
        # query head h really reads group h // (H/KV): make one KV head's values huge
        if KV > 1:
            v2 = v.copy(); v2[:, :, KV - 1] += 1000.0
            out2, _ = A.attention(q, k, v2, rope_base=10000.0)
            changed = np.abs(out2 - out).max(axis=(0, 1, 3)) > 1.0
            assert list(np.nonzero(changed)[0]) == list(range(H - H // KV, H))


# ----------------------------------------------------------------------------- the lab
def test_lab_properties(golden_dir):
    """The worked example's Property 1 (exactly 0.0) and Property 2 (about 1e-15)."""
    with open(os.path.join(golden_dir, "lab_properties.json")) as f:
        gold = json.load(f)
    ex = gold["example"]
    w = workloads.tiny_block_inputs(0)
    kw = dict(H=ex["H"], KV=ex["KV"], rope_base=ex["rope_base"], causal=True)
    out = A.block(w["x"][None], w["Wq"], w["Wk"], w["Wv"], w["Wo"], **kw)[0]
    x2 = w["x"].astype(np.float64).copy(); x2[-1] += 1.0
    out2 = A.block(x2[None], w["Wq"], w["Wk"], w["Wv"], w["Wo"], **kw)[0]
    assert np.abs(out2[:-1] - out[:-1]).max() == gold["causal_check"]["bound"]
    assert np.abs(out2[-1] - out[-1]).max() > 1e-3          # the last row does change
    out3 = A.block(w["x"][None], w["Wq"], w["Wk"], w["Wv"], w["Wo"], pos0=100, **kw)[0]
    rel = np.abs(out3 - out).max()
    assert rel <= gold["relative_check"]["bound"]
    assert rel > 0.0                                           # rounding differs, as printed
    assert out.shape == (ex["T"], ex["d"])


def test_lab_example_draws_match_the_page_recipe():
    """Lab recipe: default_rng(0), x then Wq, Wk, Wv, Wo drawn N(0,1), weights / sqrt(d)."""
    rng = np.random.default_rng(0)
    x = rng.normal(size=(6, 32))
    wq = rng.normal(size=(32, 32)) / np.sqrt(32)
    w = workloads.tiny_block_inputs(0)
    np.testing.assert_array_equal(w["x"], x.astype(np.float32))
    np.testing.assert_array_equal(w["Wq"], wq.astype(np.float32))
    assert w["Wk"].shape == (32, 16) and w["Wo"].shape == (32, 32)


@pytest.mark.parametrize("pos0", [0, 100])
def test_block_brute_force(pos0):
    w = workloads.tiny_block_inputs(0)
    kw = dict(H=4, KV=2, pos0=pos0, rope_base=10000.0, causal=True)
    out = A.block(w["x"][None], w["Wq"], w["Wk"], w["Wv"], w["Wo"], **kw)[0]
    ref = brute.block(w["x"], w["Wq"], w["Wk"], w["Wv"], w["Wo"], **kw)
    np.testing.assert_allclose(out, np.array(ref), rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- decode
def test_decode_token_by_token_equals_full():
    """Lab exercise 2: one token at a time over a growing cache equals the full causal pass."""
    B, T, H, KV, hd, base = 2, 10, 4, 2, 8, 10000.0
    q, k, v = _rand((B, T, H, hd), 60), _rand((B, T, KV, hd), 61), _rand((B, T, KV, hd), 62)
    for window, slopes in [(0, None), (4, None), (0, A.alibi_slopes(H))]:
        full, full_lse = A.attention(q, k, v, rope_base=base, window=window, slopes=slopes)
        kc = np.zeros((B, T, KV, hd)); vc = np.zeros((B, T, KV, hd))
        for t in range(T):
            kc[:, t] = A.rope(k[:, t][:, :, None, :], [t], base)[:, :, 0, :]   # rotate at slot t
            vc[:, t] = v[:, t]
            o, l = A.decode(q[:, t], kc, vc, [t + 1] * B, [t] * B, rope_base=base, window=window,
                            slopes=slopes)
            np.testing.assert_allclose(o, full[:, t], rtol=0, atol=1e-13)
            np.testing.assert_allclose(l, full_lse[:, :, t], rtol=0, atol=1e-13)


def test_decode_brute_force_and_empty_cache():
    B, H, KV, hd, Lmax = 3, 4, 1, 6, 9
    q, kc, vc = _rand((B, H, hd), 70), _rand((B, Lmax, KV, hd), 71), _rand((B, Lmax, KV, hd), 72)
    seqlens, qpos = [5, 0, 9], [5, 0, 9]
    for window, slopes in [(0, None), (3, A.alibi_slopes(H))]:
        out, lse = A.decode(q, kc, vc, seqlens, qpos, rope_base=10000.0, window=window, slopes=slopes)
        bo, bl = brute.decode(q, kc, vc, seqlens, qpos, rope_base=10000.0, window=window, slopes=slopes)
        np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)
        assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))


def test_chunked_prefill_equals_full():
    """A sequence prefilled in chunks over a cache (each chunk's keys written at their own
    positions, then its queries attending the cache) equals the one-pass prefill."""
    B, T, H, KV, hd, base, Lmax = 2, 23, 4, 2, 8, 10000.0, 32
    q, k, v = _rand((B, T, H, hd), 80), _rand((B, T, KV, hd), 81), _rand((B, T, KV, hd), 82)
    bounds = [0, 7, 8, 23]  # chunks of 7, 1 and 15 rows
    for window, slopes in [(0, None), (5, None), (0, A.alibi_slopes(H))]:
        full, full_lse = A.attention(q, k, v, rope_base=base, window=window, slopes=slopes)
        kc = np.zeros((B, Lmax, KV, hd)); vc = np.zeros((B, Lmax, KV, hd))
        for c0, c1 in zip(bounds[:-1], bounds[1:]):
            kc, vc = A.kv_write(k[:, c0:c1], v[:, c0:c1], kc, vc, [c0] * B, rope_base=base)
            o, l = A.chunk(q[:, c0:c1], kc, vc, [c1] * B, [c0] * B, rope_base=base, window=window,
                           slopes=slopes)
            np.testing.assert_allclose(o, full[:, c0:c1], rtol=0, atol=1e-13)
            np.testing.assert_allclose(l, full_lse[:, :, c0:c1], rtol=0, atol=1e-13)


def test_chunk_brute_force_and_cache_route():
    """chunk() against scalar loops over a cache whose keys the loops rotate themselves."""
    B, Tq, H, KV, hd, Lmax, base = 2, 5, 4, 1, 6, 12, 10000.0
    q = _rand((B, Tq, H, hd), 90)
    kraw, vc = _rand((B, Lmax, KV, hd), 91), _rand((B, Lmax, KV, hd), 92)
    kc = [[[brute.rotate_vec(list(kraw[b, j, g]), j, base) for g in range(KV)] for j in range(Lmax)]
          for b in range(B)]
    seqlens, qpos0 = [9, 12], [4, 7]
    for causal, window, slopes in [(True, 0, None), (True, 3, A.alibi_slopes(H)), (False, 0, None)]:
        out, lse = A.chunk(q, np.array(kc), vc, seqlens, qpos0, rope_base=base, causal=causal,
                           window=window, slopes=slopes)
        bo, bl = brute.chunk(q, kc, vc, seqlens, qpos0, rope_base=base, causal=causal, window=window,
                             slopes=slopes)
        np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-12)


def test_chunk_of_one_row_is_a_decode_step_and_empty_cache():
    B, H, KV, hd, Lmax, base = 3, 4, 2, 8, 10, 10000.0
    q, kc, vc = _rand((B, 1, H, hd), 95), _rand((B, Lmax, KV, hd), 96), _rand((B, Lmax, KV, hd), 97)
    seqlens = [6, 0, 10]
    o, l = A.chunk(q, kc, vc, seqlens, [5, 0, 9], rope_base=base)
    do, dl = A.decode(q[:, 0], kc, vc, seqlens, [5, 0, 9], rope_base=base)
    np.testing.assert_allclose(o[:, 0], do, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l[:, :, 0], dl, rtol=0, atol=1e-13)
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(l[1]))


def test_paged_decode_brute_force_and_page_order():
    """Paged decode against slot-by-slot page lookups, and invariance under where the pages sit:
    the same rows in a shuffled page pool give the contiguous cache's result."""
    B, H, KV, hd, ps, base = 3, 4, 2, 6, 4, 10000.0
    seqlens, qpos = [9, 0, 16], [9, 0, 15]
    npages = 14
    rng = np.random.default_rng(7)
    table = rng.permutation(npages)[:12].reshape(3, 4)
    q, kp, vp = _rand((B, H, hd), 100), _rand((npages, ps, KV, hd), 101), _rand((npages, ps, KV, hd), 102)
    for window, slopes in [(0, None), (5, A.alibi_slopes(H))]:
        out, lse = A.decode_paged(q, kp, vp, table, seqlens, qpos, page_size=ps, rope_base=base,
                                  window=window, slopes=slopes)
        bo, bl = brute.decode_paged(q, kp, vp, table, seqlens, qpos, page_size=ps, rope_base=base,
                                    window=window, slopes=slopes)
        np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)
        # contiguous equivalent built by hand, row by row
        kc = np.zeros((B, 16, KV, hd)); vc = np.zeros((B, 16, KV, hd))
        for b in range(B):
            for j in range(seqlens[b]):
                kc[b, j] = kp[table[b][j // ps], j % ps]
                vc[b, j] = vp[table[b][j // ps], j % ps]
        co, cl = A.decode(q, kc, vc, seqlens, qpos, rope_base=base, window=window, slopes=slopes)
        np.testing.assert_allclose(out, co, rtol=0, atol=1e-13)
        assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))


def test_latent_fold_leaves_scores_and_outputs_unchanged():
    """[LAB] exercise 5: folding the key up-projection into the query leaves the scores (and so
    the outputs) unchanged; and the latent decode equals a plain decode over the keys and values
    the up-projections produce, materialised as an H-head cache."""
    B, H, hd, dc, Lmax = 3, 4, 8, 5, 11
    q, c = _rand((B, H, hd), 110), _rand((B, Lmax, dc), 111)
    W_uk, W_uv = _rand((H, dc, hd), 112) / np.sqrt(dc), _rand((H, dc, hd), 113) / np.sqrt(dc)
    seqlens, qpos = [7, 0, 11], [7, 0, 10]
    for window, slopes in [(0, None), (4, A.alibi_slopes(H))]:
        o1, l1 = A.latent_decode(q, c, W_uk, W_uv, seqlens, qpos, window=window, slopes=slopes)
        o2, l2 = A.latent_decode_folded(q, c, W_uk, W_uv, seqlens, qpos, window=window, slopes=slopes)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)
        kc = np.einsum("bld,hde->blhe", c, W_uk)               # [B, Lmax, H, hd]
        vc = np.einsum("bld,hde->blhe", c, W_uv)
        o3, l3 = A.decode(q, kc, vc, seqlens, qpos, window=window, slopes=slopes)
        np.testing.assert_allclose(o3, o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l3, l1, rtol=0, atol=1e-13)
        assert np.all(o1[1] == 0.0) and np.all(np.isneginf(l1[1]))
    # the fold at the level of one score, written out
    s_unfolded = q[0, 2] @ (c[0, 3] @ W_uk[2])
    s_folded = (W_uk[2] @ q[0, 2]) @ c[0, 3]
    assert abs(s_unfolded - s_folded) < 1e-13


def test_rmsnorm_closed_forms():
    """RMSNorm: a constant vector c maps to sign(c) gamma (for eps -> 0); scaling x by s > 0
    changes nothing; each normalised row has root-mean-square |gamma| when gamma is constant."""
    g = np.full(6, 2.5)
    np.testing.assert_allclose(A.rmsnorm(np.full((1, 6), -3.0), g, eps=0.0), np.full((1, 6), -2.5),
                               rtol=0, atol=1e-15)
    x = _rand((4, 6), 120)
    np.testing.assert_allclose(A.rmsnorm(7.0 * x, g, eps=0.0), A.rmsnorm(x, g, eps=0.0), rtol=0, atol=1e-14)
    y = A.rmsnorm(x, g, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 2.5, rtol=0, atol=1e-14)
    # eps enters under the root: x = 0 rows stay 0, tiny rows are damped
    assert np.all(A.rmsnorm(np.zeros((1, 6)), g) == 0.0)
    # where eps sits: a constant row c with eps = 3 c^2 gives c / sqrt(c^2 + 3 c^2) = sign(c) / 2
    # (eps added outside the root would give c / (|c| + 3 c^2) instead: -0.1 gamma for c = -3)
    for c in (-3.0, 0.5, 2.0):
        np.testing.assert_allclose(A.rmsnorm(np.full((2, 6), c), g, eps=3.0 * c * c),
                                   np.full((2, 6), np.sign(c) * 1.25), rtol=0, atol=1e-15)
    # the default eps is 1e-6 (the listing of "RMSNorm and Pre-LN residuals"): a constant row of
    # 1e-3 has mean square 1e-6, so it maps to gamma / sqrt(2); 1e-5 or 1e-8 would give 0.30 or 0.995
    np.testing.assert_allclose(A.rmsnorm(np.full((1, 6), 1e-3), g), np.full((1, 6), 2.5 / np.sqrt(2.0)),
                               rtol=1e-12, atol=0)


def test_fused_block_is_residual_plus_the_plain_block_on_normalised_input():
    """block_fused(x) - x equals the plain block on RMSNorm(x) with Wqkv split into Wq, Wk, Wv;
    its cache rows are the keys turned at their positions and the values."""
    B, T, d, H, KV, base, pos0 = 2, 9, 16, 4, 2, 10000.0, 5
    hd = d // H
    x, gamma = _rand((B, T, d), 121), 1.0 + 0.1 * _rand((d,), 122)
    Wqkv, Wo = _rand((d, (H + 2 * KV) * hd), 123) / 4, _rand((H * hd, d), 124) / 4
    Wq, Wk, Wv = Wqkv[:, :H * hd], Wqkv[:, H * hd:(H + KV) * hd], Wqkv[:, (H + KV) * hd:]
    for window, slopes in [(0, None), (3, A.alibi_slopes(H))]:
        out, kc, vc = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, pos0=pos0, rope_base=base,
                                    window=window, slopes=slopes)
        plain = A.block(A.rmsnorm(x, gamma), Wq, Wk, Wv, Wo, H=H, KV=KV, pos0=pos0, rope_base=base,
                        window=window, slopes=slopes)
        np.testing.assert_allclose(out - x, plain, rtol=0, atol=1e-12)
        k = (A.rmsnorm(x, gamma) @ Wk).reshape(B, T, KV, hd)
        v = (A.rmsnorm(x, gamma) @ Wv).reshape(B, T, KV, hd)
        ek, ev = A.kv_write(k, v, np.zeros((B, 20, KV, hd)), np.zeros((B, 20, KV, hd)), [pos0] * B,
                            rope_base=base)
        np.testing.assert_allclose(kc, ek[:, pos0:pos0 + T], rtol=0, atol=1e-13)
        np.testing.assert_allclose(vc, ev[:, pos0:pos0 + T], rtol=0, atol=0)


# ----------------------------------------------------------------------------- workloads
def test_workload_pair_counts():
    """FLOP counts used by the bench: causal pairs T(T+1)/2, windowed pairs sum min(i+1, W)."""
    assert workloads.GQA.allowed_pairs == 4096 * 4097 // 2 == 8390656
    assert workloads.LONG_WINDOW.allowed_pairs == sum(min(i + 1, 4096) for i in range(16384)) \
        == 58722304
    assert workloads.MHA_ROPE.flops == 4 * 4 * 16 * 64 * 524800
    assert abs(workloads.GQA.flops / 1e9 - 274.9) < 0.1
    assert abs(workloads.LONG_WINDOW.flops / 1e9 - 962.1) < 0.1
    c = workloads.GQA_CHUNK
    assert c.allowed_pairs == sum(c.qpos0 + i + 1 for i in range(c.Tq))
    # the chunk's rows are the second half of the GQA prefill's rows: its pairs plus the first
    # half's make up the whole causal triangle
    assert c.allowed_pairs + 2048 * 2049 // 2 == workloads.GQA.allowed_pairs


def test_block_row_selection_equals_full_rows():
    """block(rows=R) and block_fused(rows=R) are rows R of the full results (each query row's
    output depends on the keys only through the full k, v, which are always computed)."""
    B, T, d, H, KV, base = 2, 11, 16, 4, 2, 10000.0
    hd = d // H
    x = _rand((B, T, d), 130)
    Wq, Wk, Wv, Wo = (_rand(s, 131 + n) / 4 for n, s in
                      enumerate([(d, H * hd), (d, KV * hd), (d, KV * hd), (H * hd, d)]))
    rows = [0, 3, 10, 7]
    for window, slopes in [(0, None), (4, A.alibi_slopes(H))]:
        full = A.block(x, Wq, Wk, Wv, Wo, H=H, KV=KV, pos0=3, rope_base=base, window=window, slopes=slopes)
        part = A.block(x, Wq, Wk, Wv, Wo, H=H, KV=KV, pos0=3, rope_base=base, window=window, slopes=slopes,
                       rows=rows)
        np.testing.assert_array_equal(part, full[:, rows])
        Wqkv = np.concatenate([Wq, Wk, Wv], axis=1)
        gamma = 1.0 + 0.1 * _rand((d,), 140)
        ffull, _, _ = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, pos0=3, rope_base=base, window=window,
                                    slopes=slopes)
        fpart, _, _ = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, pos0=3, rope_base=base, window=window,
                                    slopes=slopes, rows=rows)
        np.testing.assert_allclose(fpart, ffull[:, rows], rtol=0, atol=1e-13)
