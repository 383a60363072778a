"""Prefill parity on the GPU: the CUDA path through the C ABI against the fp64 oracle.

Small cases span several tiles and a ragged tail and are compared element by element;
the named full-size workloads are compared in full (or, for the 16k-token window case,
on a fixed row sample the oracle computes row by row). Causality is checked bit for bit.
"""
import zlib

import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._gpu_util import TOL, assert_close, assert_lse_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def art():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import alibi_rope_tile_b200 as m
    m.lib()
    return m


def run(art, q, k, v, w, with_lse=True, turn_keys_first=True):
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    B, T, H, hd = q.shape
    lse = torch.empty(B, H, T, dtype=torch.float32, device="cuda") if with_lse else None
    slopes = art.alibi_slopes(H) if w.alibi else None
    out = art.attn_prefill(dq, dk, dv, lse=lse, pos0=w.pos0, rope_base=w.rope_base,
                           causal=w.causal, window=w.window, alibi_slopes=slopes,
                           turn_keys_first=turn_keys_first)
    torch.cuda.synchronize()
    art.attn_sync_status()
    return out, lse


def oracle(q, k, v, w, rows=None):
    slopes = A.alibi_slopes(q.shape[2]) if w.alibi else None
    return A.attention(q, k, v, pos0=w.pos0, rope_base=w.rope_base, causal=w.causal,
                       window=w.window, slopes=slopes, rows=rows)


FLAGS = {
    "rope": dict(rope_base=10000.0),
    "rope5e5_pos0": dict(rope_base=500000.0, pos0=100),
    "alibi": dict(rope_base=0.0, alibi=True),
    "rope_window": dict(rope_base=10000.0, window=37),
    "rope_alibi_window": dict(rope_base=10000.0, window=130, alibi=True),
    "full_rope": dict(rope_base=10000.0, causal=False),
}
SHAPES = [(1, 1, 4, 2, 64), (2, 200, 4, 2, 64), (1, 333, 8, 2, 128), (1, 257, 4, 1, 128),
          (2, 130, 4, 4, 128), (1, 97, 6, 3, 32), (2, 45, 4, 2, 8)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("flags", sorted(FLAGS))
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}T{}H{}KV{}hd{}".format(*s))
def test_small(art, shape, flags, dtype):
    B, T, H, KV, hd = shape
    w = workloads.small_prefill(B, T, H, KV, hd, seed=zlib.crc32(repr((shape, flags)).encode()) % 1000, **FLAGS[flags])
    q, k, v = workloads.prefill_inputs(w, dtype)
    out, lse = run(art, q, k, v, w)
    ro, rl = oracle(q, k, v, w)
    assert_close(out, ro, dtype, f"out {w.name} {flags}")
    assert_lse_close(lse, rl, dtype, f"lse {w.name} {flags}")


@pytest.mark.parametrize("wname", ["mha_prefill_bf16_B4_T1024_H16_hd64_rope",
                                   "mha_prefill_bf16_B4_T1024_H16_hd64_alibi",
                                   "gqa_prefill_bf16_B2_T4096_H32_KV8_hd128"])
def test_named_workload_full(art, wname):
    w = workloads.PREFILLS[wname]
    q, k, v = workloads.prefill_inputs(w)
    out, lse = run(art, q, k, v, w)
    ro, rl = oracle(q, k, v, w)
    assert_close(out, ro, torch.bfloat16, w.name)
    assert_lse_close(lse, rl, torch.bfloat16, w.name)


# bf16 with hd 64 or 128 and RoPE runs two ways: a key rotation pass into the workspace, then
# the persistent attention kernel on turned keys (the default), or the keys turned inside the
# attention kernel as its tiles land (no workspace). Both must match the oracle.
ROPE_FLAGS = sorted(f for f in FLAGS if FLAGS[f].get("rope_base", 0) > 0)
SHAPES_128 = [s for s in SHAPES if s[4] in (64, 128)]


@pytest.mark.parametrize("flags", ROPE_FLAGS)
@pytest.mark.parametrize("shape", SHAPES_128, ids=lambda s: "B{}T{}H{}KV{}hd{}".format(*s))
def test_small_keys_turned_in_kernel(art, shape, flags):
    B, T, H, KV, hd = shape
    w = workloads.small_prefill(B, T, H, KV, hd, seed=zlib.crc32(repr((shape, flags)).encode()) % 1000, **FLAGS[flags])
    q, k, v = workloads.prefill_inputs(w, torch.bfloat16)
    out, lse = run(art, q, k, v, w, turn_keys_first=False)
    ro, rl = oracle(q, k, v, w)
    assert_close(out, ro, torch.bfloat16, f"out {w.name} {flags} (keys turned in the kernel)")
    assert_lse_close(lse, rl, torch.bfloat16, f"lse {w.name} {flags} (keys turned in the kernel)")


# More units (128 query rows of one head) than SMs, with a ragged last block: every CTA of the
# persistent kernel walks several units (the snake order, the query-buffer and statistics
# hand-overs), with windows that cut the key range of later units.
MULTI_UNIT = [
    ((3, 1000, 16, 4, 128), dict(rope_base=1e4)),
    ((2, 1100, 16, 2, 128), dict(rope_base=5e5, pos0=9, window=300, alibi=True)),
    ((4, 777, 16, 16, 64), dict(rope_base=1e4, alibi=True)),
    ((2, 650, 32, 8, 64), dict(rope_base=0.0, causal=False)),
]


@pytest.mark.parametrize("shape,flags", MULTI_UNIT, ids=lambda c: str(c) if isinstance(c, tuple) else "")
def test_multi_unit_ragged(art, shape, flags):
    B, T, H, KV, hd = shape
    w = workloads.small_prefill(B, T, H, KV, hd, seed=zlib.crc32(repr(shape).encode()) % 1000, **flags)
    q, k, v = workloads.prefill_inputs(w)
    out, lse = run(art, q, k, v, w)
    ro, rl = oracle(q, k, v, w)
    assert_close(out, ro, torch.bfloat16, f"out {w.name}")
    assert_lse_close(lse, rl, torch.bfloat16, f"lse {w.name}")


def test_gqa_workload_keys_turned_in_kernel(art):
    w = workloads.GQA
    q, k, v = workloads.prefill_inputs(w)
    out, lse = run(art, q, k, v, w, turn_keys_first=False)
    ro, rl = oracle(q, k, v, w)
    assert_close(out, ro, torch.bfloat16, w.name + " (keys turned in the kernel)")
    assert_lse_close(lse, rl, torch.bfloat16, w.name + " (keys turned in the kernel)")


def test_rotation_pass_workspace(art):
    """The rotation pass writes exactly B*T*KV*hd bf16 values into a caller's workspace and
    leaves the bytes after them alone; a larger, reused workspace gives the same output."""
    w = workloads.small_prefill(2, 333, 8, 2, 128, seed=21, rope_base=10000.0, pos0=7)
    q, k, v = workloads.prefill_inputs(w)
    need = art.attn_prefill_workspace_size(2, 333, 2, 128, 10000.0)
    assert need == 2 * 333 * 2 * 128 * 2
    ws = torch.full((need + 4096,), 0x5A, dtype=torch.uint8, device="cuda")
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    o1 = art.attn_prefill(dq, dk, dv, pos0=7, rope_base=10000.0, workspace=ws)
    o2 = art.attn_prefill(dq, dk, dv, pos0=7, rope_base=10000.0, workspace=ws)
    torch.cuda.synchronize()
    art.attn_sync_status()
    assert torch.equal(o1, o2)
    assert bool((ws[need:] == 0x5A).all())
    # the workspace holds the keys turned at positions pos0 + t: compare with the oracle's turn
    # (fp32 arithmetic, about 1e-6 of the pair's size, then one rounding to bf16 within
    # 2^-9 of the value)
    kr = ws[:need].view(torch.bfloat16).view(2, 333, 2, 128).cpu().double().numpy()
    ref = A.rope(k.permute(0, 2, 1, 3), np.arange(7, 7 + 333), 10000.0).transpose(0, 2, 1, 3)
    assert np.all(np.abs(kr - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4)
    ro, _ = oracle(q, k, v, w)
    assert_close(o1, ro, torch.bfloat16, "out with a reused workspace")


def long_rows(T=16384, W=4096, seed=3):
    rows = set(range(256)) | set(range(T - 256, T))
    for c in range(W, T, W):
        rows |= set(range(c - 64, c + 64))
    rng = np.random.default_rng(seed)
    rows |= set(rng.choice(T, 512, replace=False).tolist())
    return np.array(sorted(rows))


def test_long_window_sampled_rows(art):
    w = workloads.LONG_WINDOW
    q, k, v = workloads.prefill_inputs(w)
    out, lse = run(art, q, k, v, w)
    rows = long_rows()
    ro, rl = oracle(q, k, v, w, rows=rows)
    assert_close(out[:, rows], ro, torch.bfloat16, w.name + " sampled rows")
    assert_lse_close(lse[:, :, rows], rl, torch.bfloat16, w.name + " sampled rows")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("shape,flags", [((1, 1000, 8, 2, 128), dict(rope_base=500000.0)),
                                          ((2, 513, 4, 4, 64), dict(rope_base=0.0, alibi=True)),
                                          ((1, 700, 4, 2, 128), dict(rope_base=1e4, window=300))])
def test_causality_bit_exact(art, shape, flags, dtype):
    """Changing the last token (q, k and v) leaves every earlier output row bit-identical."""
    B, T, H, KV, hd = shape
    w = workloads.small_prefill(B, T, H, KV, hd, seed=7, **flags)
    q, k, v = workloads.prefill_inputs(w, dtype)
    out, _ = run(art, q, k, v, w, with_lse=False)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, -1] += 1.0
    k2[:, -1] -= 2.0
    v2[:, -1] *= 3.0
    out2, _ = run(art, q2, k2, v2, w, with_lse=False)
    assert torch.equal(out[:, :-1], out2[:, :-1])
    assert not torch.equal(out[:, -1], out2[:, -1])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("hd", [64, 128])
def test_window_one_is_value(art, hd, dtype):
    """Closed form: a window of one key returns each row's own value, exactly."""
    w = workloads.small_prefill(2, 300, 8, 2, hd, seed=9, rope_base=10000.0, window=1)
    q, k, v = workloads.prefill_inputs(w, dtype)
    out, _ = run(art, q, k, v, w, with_lse=False)
    assert torch.equal(out.cpu(), v.repeat_interleave(4, dim=2))


def test_relative_positions_gpu(art):
    """Shifting every position by 100 changes the GPU result only within rounding."""
    w0 = workloads.small_prefill(1, 512, 8, 2, 128, seed=11, rope_base=10000.0)
    w1 = workloads.small_prefill(1, 512, 8, 2, 128, seed=11, rope_base=10000.0, pos0=100)
    q, k, v = workloads.prefill_inputs(w0)
    o0, _ = run(art, q, k, v, w0)
    o1, _ = run(art, q, k, v, w1)
    d = (o0.float() - o1.float()).abs()
    assert d.max().item() <= TOL[torch.bfloat16]["max_abs"]
    assert d.mean().item() <= TOL[torch.bfloat16]["mean_abs"]


def test_matches_torch_sdpa_crosscheck(art):
    """Extra sanity check (not the oracle): agrees with torch SDPA on a no-rope causal case."""
    w = workloads.small_prefill(2, 256, 8, 2, 128, seed=13)
    q, k, v = workloads.prefill_inputs(w)
    out, _ = run(art, q, k, v, w, with_lse=False)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.cuda().transpose(1, 2).float(), k.cuda().transpose(1, 2).float(),
        v.cuda().transpose(1, 2).float(), is_causal=True, enable_gqa=True).transpose(1, 2)
    assert (out.float() - ref).abs().max().item() < 2e-2
