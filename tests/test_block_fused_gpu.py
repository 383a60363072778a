"""The fused pre-norm attention sub-layer on the GPU (RMSNorm, QKV GEMM with RoPE and cache
writes in its epilogue, attention, Wo GEMM with the residual) vs the oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close, assert_close_stored, to_np

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


def test_fused_block_at_bench_size(art):
    """The bench's fused sub-layer (x [2,4096,4096], gamma = 1, Wqkv = [Wq|Wk|Wv], caches
    [2,4096,8,128]) against the oracle on 1,024 sampled rows per sequence, and its cache rows."""
    from tests.test_block_gpu import sampled_rows
    bw = workloads.GQA_BLOCK
    x, W = workloads.block_inputs(bw)
    Wqkv = torch.cat([W["Wq"], W["Wk"], W["Wv"]], dim=1).contiguous()
    gamma = torch.ones(bw.d, dtype=BF)
    kc = torch.zeros(bw.B, bw.T, bw.KV, bw.hd, dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    out = art.attn_block_fused(x.cuda(), gamma.cuda(), Wqkv.cuda(), W["Wo"].cuda(), kcache=kc, vcache=vc,
                               H=bw.H, KV=bw.KV, rope_base=bw.rope_base, causal=bw.causal, window=bw.window)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    rows = sampled_rows(bw.T, 62)
    ref, rk, rv = A.block_fused(x, gamma, Wqkv, W["Wo"], H=bw.H, KV=bw.KV, rope_base=bw.rope_base,
                                causal=bw.causal, window=bw.window, rows=rows)
    assert_close(out[:, torch.from_numpy(rows).cuda()], ref, BF, "bench-size fused block")
    assert_close_stored(kc, rk, BF, "bench-size cache keys")
    assert_close_stored(vc, rv, BF, "bench-size cache values")


def test_fused_block_rows_near_eps(art):
    """Rows whose mean square is about eps (x ~ 1e-3 N(0,1), eps = 1e-6): where eps enters
    RMSNorm shows in the output (under the root it damps these rows by about 1/sqrt(2))."""
    B, T, d, H, KV = 1, 256, 512, 8, 2
    hd = d // H
    g = torch.Generator().manual_seed(77)
    x = (1e-3 * torch.randn(B, T, d, generator=g)).to(BF)
    gamma = (1.0 + 0.1 * torch.randn(d, generator=g)).to(BF)
    Wqkv = (torch.randn(d, (H + 2 * KV) * hd, generator=g) / np.sqrt(d)).to(BF)
    Wo = (torch.randn(H * hd, d, generator=g) / (2 * np.sqrt(H * hd))).to(BF)
    out = art.attn_block_fused(x.cuda(), gamma.cuda(), Wqkv.cuda(), Wo.cuda(), H=H, KV=KV, rope_base=1e4)
    torch.cuda.synchronize()
    ref, _, _ = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, rope_base=1e4)
    assert_close(out, ref, BF, "fused block, rows near eps")
    wrong, _, _ = A.block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, rope_base=1e4, eps=0.0)
    assert np.abs(wrong - ref).max() > 0.05   # the case does tell the readings apart


def test_prefolded_weights_give_the_same_output(art):
    """gamma folded into Wqkv once by the caller (fold_rmsnorm_gamma, then gamma=None) gives the
    same bits as folding on every call; the folded weights equal gamma[k] W[k][n] rounded to bf16."""
    B, T, d, H, KV = 2, 256, 512, 8, 2
    hd = d // H
    g = torch.Generator().manual_seed(11)
    x = (0.25 * torch.randn(B, T, d, generator=g)).to(BF).cuda()
    gamma = (1.0 + 0.1 * torch.randn(d, generator=g)).to(BF).cuda()
    Wqkv = (torch.randn(d, (H + 2 * KV) * hd, generator=g) / np.sqrt(d)).to(BF).cuda()
    Wo = (torch.randn(H * hd, d, generator=g) / (2 * np.sqrt(H * hd))).to(BF).cuda()
    Wg = art.fold_rmsnorm_gamma(gamma, Wqkv)
    torch.cuda.synchronize()
    expect = (gamma.double().cpu()[:, None] * Wqkv.double().cpu()).to(BF)
    assert torch.equal(Wg.cpu(), expect)
    a = art.attn_block_fused(x, gamma, Wqkv, Wo, H=H, KV=KV, rope_base=1e4)
    b = art.attn_block_fused(x, None, Wg, Wo, H=H, KV=KV, rope_base=1e4)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    assert torch.equal(a, b)
