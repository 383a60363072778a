"""Block parity on the GPU: projections + attention + output projection vs the oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


def run_block(art, w, x, pos0, **kw):
    return art.attn_block(x.cuda(), w["Wq"].cuda(), w["Wk"].cuda(), w["Wv"].cuda(),
                          w["Wo"].cuda(), pos0=pos0, **kw)


@pytest.mark.parametrize("pos0", [0, 100])
def test_tiny_block_fp32(art, pos0):
    """The lab's worked example on the GPU, fp32, within 1e-5 of the fp64 oracle."""
    cfg = workloads.TINY_BLOCK
    w = {n: torch.from_numpy(a) for n, a in workloads.tiny_block_inputs(cfg.seed).items()}
    out = run_block(art, w, w["x"][None], pos0, H=cfg.H, KV=cfg.KV, rope_base=cfg.rope_base)
    ref = A.block(w["x"][None], w["Wq"], w["Wk"], w["Wv"], w["Wo"], H=cfg.H, KV=cfg.KV,
                  pos0=pos0, rope_base=cfg.rope_base)
    assert_close(out, ref, torch.float32, f"tiny block pos0={pos0}")


def test_tiny_block_lab_properties_on_gpu(art):
    """Property 1 bit-exact on the GPU; Property 2 within the fp32 bar."""
    cfg = workloads.TINY_BLOCK
    w = {n: torch.from_numpy(a) for n, a in workloads.tiny_block_inputs(cfg.seed).items()}
    kw = dict(H=cfg.H, KV=cfg.KV, rope_base=cfg.rope_base)
    out = run_block(art, w, w["x"][None], 0, **kw)
    x2 = w["x"].clone()
    x2[-1] += 1.0
    out2 = run_block(art, w, x2[None], 0, **kw)
    assert torch.equal(out[0, :-1], out2[0, :-1])
    out3 = run_block(art, w, w["x"][None], 100, **kw)
    assert (out3 - out).abs().max().item() <= 1e-5


@pytest.mark.parametrize("shape", [(2, 256, 512, 8, 2), (1, 300, 256, 4, 4), (1, 1024, 2048, 16, 4),
                                   (1, 200, 1040, 8, 8), (1, 300, 320, 5, 5)])
def test_bf16_block(art, shape):
    B, T, d, H, KV = shape
    hd = d // H
    g = torch.Generator().manual_seed(31)
    x = workloads.normal((B, T, d), 0, torch.bfloat16, g)
    W = {n: (torch.randn(*s, generator=g) / np.sqrt(d)).to(torch.bfloat16)
         for n, s in (("Wq", (d, H * hd)), ("Wk", (d, KV * hd)), ("Wv", (d, KV * hd)),
                      ("Wo", (H * hd, d)))}
    out = run_block(art, W, x, 0, H=H, KV=KV, rope_base=10000.0)
    ref = A.block(x, W["Wq"], W["Wk"], W["Wv"], W["Wo"], H=H, KV=KV, rope_base=10000.0)
    assert_close(out, ref, torch.bfloat16, f"bf16 block {shape}")


@pytest.mark.parametrize("clusters", [None, 3, 6, 7])
@pytest.mark.parametrize("shape", [(1, 300, 256, 4, 4), (1, 300, 320, 5, 5), (2, 512, 1024, 8, 2)])
def test_block_projections_on_cta_pairs_equal_one_sm(art, shape, clusters, monkeypatch):
    """The projection GEMM on CTA pairs (256-row tiles, each SM staging half of the weights'
    columns) gives the same bits as on one SM per 128-row tile. The shapes have a last row
    tile whose second half lies past M (300 rows) and column tiles whose second half lies
    partly or wholly past N (QKV 960 and Wo 320 columns). A fixed number of pairs (a test
    hook) gives several rounds and, where the last round would keep at most half of the pairs
    busy, a last round of half-width items (e.g. 320 columns on 3 pairs: the second row pair's
    last tile cut into columns 256-383 and 384-511, the latter wholly past N; QKV 960 columns
    on 6 pairs: 768-895 and 896-1023, partly past N; QKV 1536 columns on 7 pairs)."""
    if clusters is not None:
        monkeypatch.setenv("ATTN_TEST_GEMM_CLUSTERS", str(clusters))
    B, T, d, H, KV = shape
    hd = d // H
    g = torch.Generator().manual_seed(37)
    x = workloads.normal((B, T, d), 0, torch.bfloat16, g)
    W = {n: (torch.randn(*s, generator=g) / np.sqrt(d)).to(torch.bfloat16)
         for n, s in (("Wq", (d, H * hd)), ("Wk", (d, KV * hd)), ("Wv", (d, KV * hd)),
                      ("Wo", (H * hd, d)))}
    pair = run_block(art, W, x, 0, H=H, KV=KV, rope_base=10000.0)
    torch.cuda.synchronize()
    monkeypatch.delenv("ATTN_TEST_GEMM_CLUSTERS", raising=False)
    monkeypatch.setenv("ATTN_TEST_GEMM_SINGLE", "1")
    one = run_block(art, W, x, 0, H=H, KV=KV, rope_base=10000.0)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    assert torch.equal(pair, one)


def sampled_rows(T: int, seed: int) -> np.ndarray:
    """The first and last 256 query rows and 512 others drawn at random (seeded)."""
    rng = np.random.default_rng(seed)
    middle = rng.choice(np.arange(256, T - 256), size=512, replace=False)
    return np.unique(np.concatenate([np.arange(256), middle, np.arange(T - 256, T)]))


def test_bf16_block_at_bench_size(art):
    """The bench's block (x [2,4096,4096], d 4096, H 32, KV 8, hd 128, RoPE 5e5, causal) in the
    launch configuration the bench times, against the oracle on 1,024 sampled rows per sequence."""
    bw = workloads.GQA_BLOCK
    x, W = workloads.block_inputs(bw)
    out = art.attn_block(x.cuda(), W["Wq"].cuda(), W["Wk"].cuda(), W["Wv"].cuda(), W["Wo"].cuda(),
                         H=bw.H, KV=bw.KV, rope_base=bw.rope_base, causal=bw.causal, window=bw.window)
    torch.cuda.synchronize()
    assert art.attn_sync_status() == 0
    rows = sampled_rows(bw.T, 61)
    ref = A.block(x, W["Wq"], W["Wk"], W["Wv"], W["Wo"], H=bw.H, KV=bw.KV, rope_base=bw.rope_base,
                  causal=bw.causal, window=bw.window, rows=rows)
    assert_close(out[:, torch.from_numpy(rows).cuda()], ref, torch.bfloat16, "bench-size block")
