"""Latent-attention decode on the GPU (the key up-projection folded into the query) vs the
oracle's unfolded definition."""
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


@pytest.mark.parametrize("dc", [64, 128])
@pytest.mark.parametrize("flags", [dict(), dict(window=500), dict(alibi=True)])
def test_latent_decode_matches_unfolded_oracle(art, dc, flags):
    B, H, hd, Lmax = 6, 32, 128, 3000
    g = torch.Generator().manual_seed(dc + len(flags))
    q = workloads.normal((B, H, hd), 0, BF, g)
    c = workloads.normal((B, Lmax, dc), 0, BF, g)
    W_uk = (torch.randn(H, dc, hd, generator=g) / np.sqrt(dc)).to(BF)
    W_uv = (torch.randn(H, dc, hd, generator=g) / np.sqrt(dc)).to(BF)
    lens = [1, 129, 2048, 3000, 0, 777]
    sl = torch.tensor(lens, dtype=torch.int32)
    for b, L in enumerate(lens):
        c[b, L:] = 0  # slots past the length are never weighted
    window = flags.get("window", 0)
    slopes = art.alibi_slopes(H) if flags.get("alibi") else None
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = art.attn_decode_latent(q.cuda(), c.cuda(), W_uk.cuda(), W_uv.cuda(), sl.cuda(), sl.cuda(), lse=lse,
                                 window=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.latent_decode(q, c, W_uk, W_uv, sl.numpy(), sl.numpy(), window=window,
                                   slopes=None if slopes is None else np.array(slopes))
    assert_close(out, ref, BF, f"latent dc{dc} {flags}")
    assert_lse_close(lse, ref_lse, BF, "latent lse")
    assert torch.count_nonzero(out[4]) == 0  # empty cache


def test_latent_decode_few_ctas(art, monkeypatch):
    """A fixed grid of 3 CTAs (a test hook): each CTA's run of latent tiles crosses sequences."""
    monkeypatch.setenv("ATTN_TEST_DECODE_CTAS", "3")
    B, H, hd, dc, Lmax = 4, 32, 128, 128, 1500
    g = torch.Generator().manual_seed(41)
    q = workloads.normal((B, H, hd), 0, BF, g)
    c = workloads.normal((B, Lmax, dc), 0, BF, g)
    W_uk = (torch.randn(H, dc, hd, generator=g) / np.sqrt(dc)).to(BF)
    W_uv = (torch.randn(H, dc, hd, generator=g) / np.sqrt(dc)).to(BF)
    lens = [1500, 3, 0, 901]
    sl = torch.tensor(lens, dtype=torch.int32)
    for b, L in enumerate(lens):
        c[b, L:] = 0
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = art.attn_decode_latent(q.cuda(), c.cuda(), W_uk.cuda(), W_uv.cuda(), sl.cuda(), sl.cuda(), lse=lse)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, ref_lse = A.latent_decode(q, c, W_uk, W_uv, sl.numpy(), sl.numpy())
    assert_close(out, ref, BF, "latent, 3 CTAs")
    assert_lse_close(lse, ref_lse, BF, "latent lse")
    assert torch.count_nonzero(out[2]) == 0  # empty cache
