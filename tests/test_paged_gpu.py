"""Paged KV cache on the GPU: decode through block tables and paged cache writes vs the oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


def paged_case(B, H, KV, hd, page_size, max_blocks, lens, seed):
    """A shuffled page pool: sequence b's blocks are distinct random pages; pages no sequence
    reaches hold NaN (so reading one would show), and table entries past a sequence are -1."""
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    need = [(L + page_size - 1) // page_size for L in lens]
    num_pages = sum(need) + 5
    order = rng.permutation(num_pages)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    at = 0
    for b in range(B):
        table[b, :need[b]] = order[at:at + need[b]]
        at += need[b]
    kp = workloads.normal((num_pages, page_size, KV, hd), seed, BF, g)
    vp = workloads.normal((num_pages, page_size, KV, hd), seed, BF, g)
    used = set(int(x) for x in table.ravel() if x >= 0)
    for page in range(num_pages):
        if page not in used:
            kp[page] = float("nan")
            vp[page] = float("nan")
    for b in range(B):  # rows past the length in a sequence's last page: finite but loud
        L = lens[b]
        if L % page_size:
            last = table[b, L // page_size]
            kp[last, L % page_size:] = 1e4
            vp[last, L % page_size:] = 1e4
    q = workloads.normal((B, H, hd), seed, BF, g)
    sl = torch.tensor(lens, dtype=torch.int32)
    return q, kp, vp, torch.from_numpy(table), sl


@pytest.mark.parametrize("page_size", [16, 64, 128])
@pytest.mark.parametrize("KV,flags", [(8, dict()), (1, dict(window=300)), (2, dict(alibi=True))])
def test_paged_decode_matches_oracle(art, page_size, KV, flags):
    B, H, hd, max_blocks = 5, 32, 128, 4096 // page_size
    lens = [1, 130, 2047, 4096, 777]
    q, kp, vp, table, sl = paged_case(B, H, KV, hd, page_size, max_blocks, lens, seed=page_size + KV)
    base = 0.0 if flags.get("alibi") else 10000.0
    window = flags.get("window", 0)
    slopes = art.alibi_slopes(H) if flags.get("alibi") else None
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = art.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda(), sl.cuda(), lse=lse,
                                rope_base=base, window=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.decode_paged(q, kp, vp, table.numpy(), sl.numpy(), sl.numpy(), page_size=page_size,
                                  rope_base=base, window=window,
                                  slopes=None if slopes is None else np.array(slopes))
    assert_close(out, ref, BF, f"paged decode ps{page_size} KV{KV} {flags}")
    assert_lse_close(lse, ref_lse, BF, "paged decode lse")


def test_paged_writes_then_decode_equal_the_contiguous_cache(art):
    """The same tokens written through attn_kv_write_paged (in two chunks) and through
    attn_kv_write give the same decode."""
    B, H, KV, hd, ps, Lmax, base = 3, 16, 2, 64, 32, 512, 10000.0
    g = torch.Generator().manual_seed(3)
    lens = [200, 512, 33]
    k = workloads.normal((B, Lmax, KV, hd), 3, BF, g).cuda()
    v = workloads.normal((B, Lmax, KV, hd), 3, BF, g).cuda()
    q = workloads.normal((B, H, hd), 3, BF, g).cuda()
    rng = np.random.default_rng(3)
    max_blocks = Lmax // ps
    table = torch.from_numpy(rng.permutation(B * max_blocks).reshape(B, max_blocks).astype(np.int32)).cuda()
    kp = torch.zeros(B * max_blocks, ps, KV, hd, dtype=BF, device="cuda")
    vp = torch.zeros_like(kp)
    kc = torch.zeros(B, Lmax, KV, hd, dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    for c0, c1 in [(0, 100), (100, Lmax)]:
        pos = torch.full((B,), c0, dtype=torch.int32, device="cuda")
        art.attn_kv_write_paged(k[:, c0:c1].contiguous(), v[:, c0:c1].contiguous(), kp, vp, table, pos,
                                rope_base=base)
        art.attn_kv_write(k[:, c0:c1].contiguous(), v[:, c0:c1].contiguous(), kc, vc, pos, rope_base=base)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    paged = art.attn_decode_paged(q, kp, vp, table, sl, sl, rope_base=base)
    flat = art.attn_decode(q, kc, vc, sl, sl, rope_base=base)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    assert torch.equal(paged, flat), "same rows, same tiles: the two layouts decode identically"
    ref, _ = A.decode(q.cpu(), kc.cpu(), vc.cpu(), sl.cpu().numpy(), sl.cpu().numpy(), rope_base=base)
    assert_close(paged, ref, BF, "paged decode after paged writes")


@pytest.mark.parametrize("page_size,KV,flags", [(16, 2, dict(alibi=True)), (128, 1, dict(window=300))])
def test_paged_decode_few_ctas(art, monkeypatch, page_size, KV, flags):
    """A fixed grid of 2 CTAs (a test hook): each CTA walks many paged tiles across sequences."""
    monkeypatch.setenv("ATTN_TEST_DECODE_CTAS", "2")
    B, H, hd, max_blocks = 5, 32, 128, 4096 // page_size
    lens = [1, 130, 2047, 4096, 777]
    q, kp, vp, table, sl = paged_case(B, H, KV, hd, page_size, max_blocks, lens, seed=7 + page_size + KV)
    base = 0.0 if flags.get("alibi") else 10000.0
    window = flags.get("window", 0)
    slopes = art.alibi_slopes(H) if flags.get("alibi") else None
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = art.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda(), sl.cuda(), lse=lse,
                                rope_base=base, window=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.decode_paged(q, kp, vp, table.numpy(), sl.numpy(), sl.numpy(), page_size=page_size,
                                  rope_base=base, window=window,
                                  slopes=None if slopes is None else np.array(slopes))
    assert_close(out, ref, BF, f"paged decode, 2 CTAs, ps{page_size} KV{KV} {flags}")
    assert_lse_close(lse, ref_lse, BF, "paged decode lse")
