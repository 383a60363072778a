"""The fused pre-norm attention sub-layer on the GPU (RMSNorm, QKV GEMM with RoPE and cache
writes in its epilogue, attention, Wo GEMM with the residual) vs the oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close, to_np

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


CASES = [
    # B, T, d, H, KV, flags
    (2, 256, 512, 8, 2, dict(rope_base=1e4, cache=True, pos0=100)),
    (1, 300, 1024, 8, 8, dict(rope_base=5e5)),
    (2, 200, 512, 8, 4, dict(alibi=True, cache=True, pos0=0)),
    (1, 390, 1024, 8, 2, dict(rope_base=1e4, window=96, pos0=7)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}d{c[2]}H{c[3]}KV{c[4]}")
def test_fused_block_matches_oracle(art, case):
    B, T, d, H, KV, flags = case
    hd = d // H
    g = torch.Generator().manual_seed(T + d)
    # RMSNorm makes the sub-layer independent of x's scale; a quarter-scale x and a half-scale
    # Wo keep the output (x + attention) near unit scale, where the bf16 bars are stated
    x = (0.25 * torch.randn(B, T, d, generator=g)).to(BF)
    gamma = (1.0 + 0.1 * torch.randn(d, generator=g)).to(BF)
    Wqkv = (torch.randn(d, (H + 2 * KV) * hd, generator=g) / np.sqrt(d)).to(BF)
    Wo = (torch.randn(H * hd, d, generator=g) / (2 * np.sqrt(H * hd))).to(BF)
    base = flags.get("rope_base", 0.0)
    pos0 = flags.get("pos0", 0)
    window = flags.get("window", 0)
    slopes = art.alibi_slopes(H) if flags.get("alibi") else None
    kc = vc = None
    Lmax = pos0 + T + 64
    if flags.get("cache"):
        kc = torch.zeros(B, Lmax, KV, hd, dtype=BF, device="cuda")
        vc = torch.zeros_like(kc)
    out = art.attn_block_fused(x.cuda(), gamma.cuda(), Wqkv.cuda(), Wo.cuda(), kcache=kc, vcache=vc, H=H,
                               KV=KV, pos0=pos0, rope_base=base, window=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    ref, rk, rv = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, pos0=pos0, rope_base=base, window=window,
                                slopes=None if slopes is None else np.array(slopes))
    assert_close(out, ref, BF, f"fused block {case}")
    if kc is not None:
        assert_close(kc[:, pos0:pos0 + T], rk, BF, "cache keys")
        assert_close(vc[:, pos0:pos0 + T], rv, BF, "cache values")
        assert torch.count_nonzero(kc[:, :pos0]) == 0 and torch.count_nonzero(kc[:, pos0 + T:]) == 0
