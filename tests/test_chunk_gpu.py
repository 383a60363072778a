"""Chunked prefill on the GPU: cache writes and chunks of queries against a cache vs the oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


def test_kv_write_matches_oracle(art):
    B, Tn, KV, hd, Lmax, base = 3, 37, 2, 128, 100, 10000.0
    g = torch.Generator().manual_seed(41)
    k, v = workloads.normal((B, Tn, KV, hd), 41, BF, g), workloads.normal((B, Tn, KV, hd), 41, BF, g)
    pos0 = torch.tensor([0, 50, 63], dtype=torch.int32)
    kc = torch.zeros(B, Lmax, KV, hd, dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    art.attn_kv_write(k.cuda(), v.cuda(), kc, vc, pos0.cuda(), rope_base=base)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    rk, rv = A.kv_write(k, v, np.zeros(kc.shape), np.zeros(vc.shape), pos0.numpy(), rope_base=base)
    assert_close(kc, rk, BF, "rotated keys")
    assert np.array_equal(to_np(vc), rv), "values are copied exactly"
    for b in range(B):  # slots outside the chunk are untouched
        p = int(pos0[b])
        assert torch.count_nonzero(kc[b, :p]) == 0 and torch.count_nonzero(kc[b, p + Tn:]) == 0


CASES = [
    # B, Tq, H, KV, hd, Lmax, qpos0, seqlens (None: qpos0 + Tq), flags
    (2, 200, 8, 2, 128, 640, [300, 37], None, dict(rope_base=1e4)),
    (1, 129, 4, 4, 64, 300, [100], None, dict(alibi=True)),
    (2, 300, 8, 2, 128, 700, [256, 5], None, dict(rope_base=1e4, window=64)),
    (1, 250, 8, 1, 128, 512, [200], [150], dict(rope_base=5e5, causal=False)),
    (2, 1, 16, 2, 128, 400, [399, 12], None, dict(rope_base=1e4)),
    (3, 77, 8, 2, 64, 256, [0, 100, 179], None, dict(rope_base=1e4)),
]


def _cache_case(B, Tq, H, KV, hd, Lmax, qpos0, seqlens, seed):
    g = torch.Generator().manual_seed(seed)
    q = workloads.normal((B, Tq, H, hd), seed, BF, g)
    kc = workloads.normal((B, Lmax, KV, hd), seed, BF, g)
    vc = workloads.normal((B, Lmax, KV, hd), seed, BF, g)
    qp = torch.tensor(qpos0, dtype=torch.int32)
    sl = torch.tensor(seqlens if seqlens is not None else [p + Tq for p in qpos0], dtype=torch.int32)
    for b in range(B):  # slots at or beyond the length are never read: make them loud
        kc[b, int(sl[b]):] = 1e4
        vc[b, int(sl[b]):] = 1e4
    return q, kc, vc, sl, qp


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}Tq{c[1]}H{c[2]}KV{c[3]}hd{c[4]}")
def test_chunk_matches_oracle(art, case):
    B, Tq, H, KV, hd, Lmax, qpos0, seqlens, flags = case
    q, kc, vc, sl, qp = _cache_case(B, Tq, H, KV, hd, Lmax, qpos0, seqlens, seed=Tq + 7 * H)
    base = flags.get("rope_base", 0.0)
    causal = flags.get("causal", True)
    window = flags.get("window", 0)
    slopes = art.alibi_slopes(H) if flags.get("alibi") else None
    lse = torch.empty(B, H, Tq, dtype=torch.float32, device="cuda")
    out = art.attn_prefill_chunk(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), qp.cuda(), lse=lse,
                                 rope_base=base, causal=causal, window=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.chunk(q, kc, vc, sl.numpy(), qp.numpy(), rope_base=base, causal=causal,
                           window=window, slopes=None if slopes is None else np.array(slopes))
    assert_close(out, ref, BF, f"chunk {case}")
    assert_lse_close(lse, ref_lse, BF, f"chunk lse {case}")


def test_chunk_over_empty_cache_is_zero(art):
    B, Tq, H, KV, hd, Lmax = 2, 40, 4, 2, 128, 64
    q, kc, vc, _, _ = _cache_case(B, Tq, H, KV, hd, Lmax, [0, 0], [0, 0], seed=5)
    sl = torch.zeros(B, dtype=torch.int32)
    qp = torch.tensor([0, 10], dtype=torch.int32)
    lse = torch.empty(B, H, Tq, dtype=torch.float32, device="cuda")
    out = art.attn_prefill_chunk(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), qp.cuda(), lse=lse, rope_base=1e4)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0
    assert torch.all(torch.isneginf(lse))


@pytest.mark.parametrize("hd", [64, 128])
def test_chunk_units_without_keys_between_units_with_keys(art, hd):
    """More units than SMs, every other sequence with an empty cache: CTAs of the persistent
    kernel take units with and without keys in turn (zero rows, lse -inf for the empty ones)."""
    B, Tq, H, KV, Lmax = 6, 300, 16, 4, 800
    qpos0 = [0, 120, 7, 400, 0, 33]
    seqlens = [0, 120 + Tq, 0, 400 + Tq, 0, 33 + Tq]
    q, kc, vc, sl, qp = _cache_case(B, Tq, H, KV, hd, Lmax, qpos0, seqlens, seed=31 + hd)
    lse = torch.empty(B, H, Tq, dtype=torch.float32, device="cuda")
    out = art.attn_prefill_chunk(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), qp.cuda(), lse=lse,
                                 rope_base=1e4, window=200)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.chunk(q, kc, vc, sl.numpy(), qp.numpy(), rope_base=1e4, causal=True, window=200)
    assert_close(out, ref, BF, f"mixed empty chunk hd{hd}")
    assert_lse_close(lse, ref_lse, BF, f"mixed empty chunk lse hd{hd}")
    for b in (0, 2, 4):
        assert torch.count_nonzero(out[b]) == 0 and torch.all(torch.isneginf(lse[b]))


def test_chunk_device_argument_error(art):
    """A query position below 0 or a length beyond the cache is reported through
    attn_sync_status; that sequence's rows are zero, the others are unaffected."""
    B, Tq, H, KV, hd, Lmax = 3, 150, 8, 2, 128, 400
    q, kc, vc, sl, qp = _cache_case(B, Tq, H, KV, hd, Lmax, [10, 20, 30], None, seed=41)
    qp_bad = torch.tensor([10, -5, 30], dtype=torch.int32)
    sl_bad = torch.tensor([10 + Tq, 20 + Tq, Lmax + 1], dtype=torch.int32)
    out = art.attn_prefill_chunk(q.cuda(), kc.cuda(), vc.cuda(), sl_bad.cuda(), qp_bad.cuda(), rope_base=1e4)
    torch.cuda.synchronize()
    with pytest.raises(art.AttnError) as e:
        art.attn_sync_status()
    assert e.value.status == -7
    art.attn_sync_status()  # cleared
    assert torch.count_nonzero(out[1]) == 0 and torch.count_nonzero(out[2]) == 0
    ref, _ = A.chunk(q[:1], kc[:1], vc[:1], sl[:1].numpy(), qp[:1].numpy(), rope_base=1e4)
    assert_close(out[:1], ref, BF, "the valid sequence beside the bad ones")


@pytest.mark.parametrize("hd", [64, 128])
def test_chunks_on_the_gpu_equal_the_one_pass_prefill(art, hd):
    """Write each chunk's keys into the cache, run the chunk's queries, compare with the oracle's
    one-pass prefill, and with the GPU's own one-pass prefill."""
    B, T, H, KV, base = 2, 700, 8, 2, 1e4
    w = workloads.small_prefill(B, T, H, KV, hd, seed=17, rope_base=base)
    q, k, v = workloads.prefill_inputs(w)
    full_ref, _ = A.attention(q, k, v, rope_base=base)
    full_gpu = art.attn_prefill(q.cuda(), k.cuda(), v.cuda(), rope_base=base)
    kc = torch.zeros(B, 768, KV, hd, dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for c0, c1 in [(0, 256), (256, 300), (300, 700)]:
        pos = torch.full((B,), c0, dtype=torch.int32, device="cuda")
        art.attn_kv_write(k[:, c0:c1].cuda(), v[:, c0:c1].cuda(), kc, vc, pos, rope_base=base)
        sl = torch.full((B,), c1, dtype=torch.int32, device="cuda")
        outs.append(art.attn_prefill_chunk(q[:, c0:c1].contiguous().cuda(), kc, vc, sl, pos,
                                           rope_base=base))
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    chunked = torch.cat(outs, dim=1)
    assert_close(chunked, full_ref, BF, f"chunked hd{hd}")
    # the two GPU routes differ only by the bf16 rounding of the rotated keys in the cache
    assert (chunked.float() - full_gpu.float()).abs().max().item() <= 2e-2
