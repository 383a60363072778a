"""Decode parity on the GPU: split-KV decode and KV append against the fp64 oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


def run_decode(art, q, kc, vc, seqlens, qpos, base, window=0, alibi=False):
    H = q.shape[1]
    lse = torch.empty(q.shape[0], H, dtype=torch.float32, device="cuda")
    out = art.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), seqlens.cuda(), qpos.cuda(), lse=lse,
                          rope_base=base, window=window,
                          alibi_slopes=art.alibi_slopes(H) if alibi else None)
    torch.cuda.synchronize()
    return out, lse


def small_case(B, H, KV, hd, Lmax, seed, dtype, lens):
    g = torch.Generator().manual_seed(seed)
    q = workloads.normal((B, H, hd), seed, dtype, g)
    kc = workloads.normal((B, Lmax, KV, hd), seed, dtype, g)
    vc = workloads.normal((B, Lmax, KV, hd), seed, dtype, g)
    seqlens = torch.tensor(lens, dtype=torch.int32)
    return q, kc, vc, seqlens, seqlens.clone()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("KV,hd", [(8, 128), (2, 128), (1, 128), (4, 64), (8, 64), (2, 8)])
@pytest.mark.parametrize("variant", ["rope", "window", "alibi"])
def test_small(art, KV, hd, variant, dtype):
    B, H, Lmax = 5, 8, 700
    lens = [0, 1, 700, 333, 64]
    q, kc, vc, sl, qp = small_case(B, H, KV, hd, Lmax, 100 + KV + hd, dtype, lens)
    window = 50 if variant == "window" else 0
    alibi = variant == "alibi"
    base = 10000.0 if variant != "alibi" else 0.0
    out, lse = run_decode(art, q, kc, vc, sl, qp, base, window, alibi)
    slopes = A.alibi_slopes(H) if alibi else None
    ro, rl = A.decode(q, kc, vc, sl.tolist(), qp.tolist(), rope_base=base, window=window,
                      slopes=slopes)
    assert_close(out, ro, dtype, f"decode KV={KV} hd={hd} {variant}")
    assert_lse_close(lse, rl, dtype, f"decode lse KV={KV} hd={hd} {variant}")
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@pytest.mark.parametrize("wname", sorted(workloads.DECODES))
def test_named_workload(art, wname):
    w = workloads.DECODES[wname]
    q, kc, vc, sl, qp = workloads.decode_inputs(w)
    out, lse = run_decode(art, q, kc, vc, sl, qp, w.rope_base)
    ro, rl = A.decode(q, kc, vc, sl.tolist(), qp.tolist(), rope_base=w.rope_base)
    assert_close(out, ro, torch.bfloat16, w.name)
    assert_lse_close(lse, rl, torch.bfloat16, w.name)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_token_by_token_equals_prefill(art, dtype):
    """Lab exercise 2 on the GPU: append each token (rotating its key) then decode it; the
    result matches the prefill's row and the oracle's full causal pass."""
    B, T, H, KV, hd, base = 2, 40, 8, 2, 128, 10000.0
    w = workloads.small_prefill(B, T, H, KV, hd, seed=21, rope_base=base)
    q, k, v = workloads.prefill_inputs(w, dtype)
    full = art.attn_prefill(q.cuda(), k.cuda(), v.cuda(), rope_base=base)
    kc = torch.zeros(B, T, KV, hd, dtype=dtype, device="cuda")
    vc = torch.zeros_like(kc)
    ref, _ = A.attention(q, k, v, rope_base=base)
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
        art.attn_kv_append(k[:, t].contiguous().cuda(), v[:, t].contiguous().cuda(), kc, vc, pos,
                           rope_base=base)
        out = art.attn_decode(q[:, t].contiguous().cuda(), kc, vc, pos + 1, pos, rope_base=base)
        assert_close(out, ref[:, t], dtype, f"token {t}")
        d = (out.float() - full[:, t].float()).abs().max().item()
        assert d <= (2e-2 if dtype == torch.bfloat16 else 1e-5)
    art.attn_sync_status()
    # the appended keys are the oracle's rotated keys
    kr = A.rope(k.permute(0, 2, 1, 3), np.arange(T), base)          # [B,KV,T,hd]
    assert_close(kc.transpose(1, 2), kr, dtype, "appended keys")


def test_device_argument_error(art):
    """A length beyond the cache is reported through attn_sync_status; that row is zero."""
    q, kc, vc, sl, qp = small_case(3, 4, 2, 64, 100, 5, torch.bfloat16, [10, 101, 50])
    out, lse = run_decode(art, q, kc, vc, sl, qp, 10000.0)
    with pytest.raises(art.AttnError) as e:
        art.attn_sync_status()
    assert e.value.status == -7
    assert torch.all(out[1] == 0)
    art.attn_sync_status()  # cleared
    ro, _ = A.decode(q, kc, vc, [10, 0, 50], [10, 0, 50], rope_base=10000.0)
    assert_close(out, ro, torch.bfloat16, "rows beside the bad one")


def test_append_position_error(art):
    kc = torch.zeros(2, 8, 1, 64, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones(2, 1, 64, dtype=torch.bfloat16, device="cuda")
    art.attn_kv_append(kn, kn, kc, vc, torch.tensor([3, 8], dtype=torch.int32, device="cuda"),
                       rope_base=0.0)
    with pytest.raises(art.AttnError):
        art.attn_sync_status()
    assert torch.all(kc[0, 3] == 1) and torch.all(kc[1] == 0)


@pytest.mark.parametrize("nctas", ["1", "3"])
@pytest.mark.parametrize("KV,hd,variant", [(1, 128, "rope"), (8, 128, "window"), (2, 64, "alibi"), (1, 64, "rope")])
def test_few_ctas_long_pieces(art, monkeypatch, nctas, KV, hd, variant):
    """The tensor-core decode gives every CTA an equal run of key tiles; a fixed small grid
    (a test hook) makes each CTA run many tiles of a sequence and cross sequence boundaries
    on small inputs, as the full-size workloads do."""
    monkeypatch.setenv("ATTN_TEST_DECODE_CTAS", nctas)
    B, H, Lmax = 3, 32 if KV <= 2 else 8, 900
    lens = [900, 1, 517]
    q, kc, vc, sl, qp = small_case(B, H, KV, hd, Lmax, 300 + KV + hd + int(nctas), torch.bfloat16, lens)
    base = 10000.0 if variant == "rope" else 0.0
    window = 300 if variant == "window" else 0
    out, lse = run_decode(art, q, kc, vc, sl, qp, base, window=window, alibi=variant == "alibi")
    assert art.attn_sync_status() == 0
    slopes = A.alibi_slopes(H) if variant == "alibi" else None
    ro, rl = A.decode(q, kc, vc, lens, lens, rope_base=base, window=window, slopes=slopes)
    assert_close(out, ro, torch.bfloat16, f"decode {nctas} CTAs KV={KV} hd={hd} {variant}")
    assert_lse_close(lse, rl, torch.bfloat16, "lse")


def test_many_units_use_the_plan_kernel(art):
    """More than 1024 (sequence, key/value head) units: a one-CTA kernel counts the tiles
    before the decode instead of every CTA counting them itself."""
    B, H, KV, hd, Lmax = 130, 8, 8, 64, 300
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(0, Lmax + 1, size=B)]
    lens[3] = 0
    q, kc, vc, sl, qp = small_case(B, H, KV, hd, Lmax, 77, torch.bfloat16, lens)
    out, lse = run_decode(art, q, kc, vc, sl, qp, 10000.0)
    assert art.attn_sync_status() == 0
    ro, rl = A.decode(q, kc, vc, lens, lens, rope_base=10000.0)
    assert_close(out, ro, torch.bfloat16, "decode, 1040 units")
    assert_lse_close(lse, rl, torch.bfloat16, "lse")
