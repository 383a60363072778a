"""attn_prefill_host: the prefill on host buffers, cut into slices whose copies overlap the
attention. Every output row must equal the device prefill's bit for bit (each slice runs the
same kernels on the same rows), whatever the slicing, and match the fp64 oracle."""
import zlib

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


def device_run(art, q, k, v, w):
    B, T, H, hd = q.shape
    lse = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
    slopes = art.alibi_slopes(H) if w.alibi else None
    out = art.attn_prefill(q.cuda(), k.cuda(), v.cuda(), lse=lse, pos0=w.pos0, rope_base=w.rope_base,
                           causal=w.causal, window=w.window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


def host_run(art, q, k, v, w, pinned=True):
    B, T, H, hd = q.shape
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out = torch.empty(q.shape, dtype=q.dtype, pin_memory=pinned)
    lse = torch.empty(B, H, T, dtype=torch.float32, pin_memory=pinned)
    slopes = art.alibi_slopes(H) if w.alibi else None
    art.attn_prefill_host(q, k, v, out, lse, pos0=w.pos0, rope_base=w.rope_base, causal=w.causal,
                          window=w.window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    art.attn_sync_status()
    return out, lse


# slicing: B < 4 cuts key/value-head groups (ng = 4, 2, 1 here), B >= 4 runs of sequences
CASES = [
    ((2, 300, 16, 8, 128), dict(rope_base=1e4)),
    ((1, 257, 8, 2, 128), dict(rope_base=5e5, pos0=11, window=100)),
    ((3, 130, 8, 1, 128), dict(rope_base=1e4)),
    ((5, 200, 4, 2, 64), dict(rope_base=0.0, alibi=True)),
    ((1, 90, 12, 4, 64), dict(rope_base=1e4, alibi=True)),
    ((18, 40, 4, 4, 128), dict(rope_base=1e4, causal=False)),
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("shape,flags", CASES, ids=lambda c: str(c) if isinstance(c, tuple) else "")
def test_host_prefill_equals_device_prefill(art, shape, flags, dtype):
    B, T, H, KV, hd = shape
    w = workloads.small_prefill(B, T, H, KV, hd, seed=zlib.crc32(repr(shape).encode()) % 1000, **flags)
    q, k, v = workloads.prefill_inputs(w, dtype)
    do, dl = device_run(art, q, k, v, w)
    ho, hl = host_run(art, q, k, v, w)
    assert torch.equal(ho, do), "host-buffer prefill differs from the device prefill"
    assert torch.equal(hl, dl)


def test_host_prefill_matches_oracle_and_pageable_memory(art):
    w = workloads.small_prefill(2, 333, 8, 2, 128, seed=5, rope_base=1e4, alibi=True)
    q, k, v = workloads.prefill_inputs(w)
    ho, hl = host_run(art, q, k, v, w, pinned=False)
    ro, rl = A.attention(q, k, v, pos0=w.pos0, rope_base=w.rope_base, causal=w.causal, window=w.window,
                         slopes=A.alibi_slopes(8))
    assert_close(ho, ro, torch.bfloat16, "host prefill (pageable)")
    assert_lse_close(hl, rl, torch.bfloat16, "host prefill lse (pageable)")


def test_host_prefill_gqa_workload(art):
    w = workloads.GQA
    q, k, v = workloads.prefill_inputs(w)
    do, dl = device_run(art, q, k, v, w)
    ho, hl = host_run(art, q, k, v, w)
    assert torch.equal(ho, do) and torch.equal(hl, dl)


def test_host_prefill_back_to_back_calls_share_a_workspace(art):
    """Two calls on one stream with one workspace: the second's copies wait for the first's."""
    w1 = workloads.small_prefill(2, 200, 8, 2, 128, seed=1, rope_base=1e4)
    w2 = workloads.small_prefill(2, 200, 8, 2, 128, seed=2, rope_base=1e4)
    q1, k1, v1 = (t.pin_memory() for t in workloads.prefill_inputs(w1))
    q2, k2, v2 = (t.pin_memory() for t in workloads.prefill_inputs(w2))
    ws = torch.empty(art.attn_prefill_host_workspace_size(2, 200, 8, 2, 128, 1e4), dtype=torch.uint8, device="cuda")
    o1 = art.attn_prefill_host(q1, k1, v1, rope_base=1e4, workspace=ws)
    o2 = art.attn_prefill_host(q2, k2, v2, rope_base=1e4, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, device_run(art, q1, k1, v1, w1)[0])
    assert torch.equal(o2, device_run(art, q2, k2, v2, w2)[0])


def test_host_prefill_from_two_threads(art):
    """Two host threads, each with its own stream and workspace, call attn_prefill_host at
    once (the calls share the device's copy streams; their enqueueing is serialised): every
    result equals the device prefill's."""
    import threading
    shapes = [(2, 260, 8, 2, 128, 1e4), (1, 300, 16, 4, 64, 5e5)]
    cases = []
    for i, (B, T, H, KV, hd, base) in enumerate(shapes):
        w = workloads.small_prefill(B, T, H, KV, hd, seed=50 + i, rope_base=base)
        q, k, v = workloads.prefill_inputs(w)
        cases.append((w, q.pin_memory(), k.pin_memory(), v.pin_memory()))
    results = [[None] * 3 for _ in cases]
    errors = []

    def worker(i):
        try:
            w, q, k, v = cases[i]
            s = torch.cuda.Stream()
            ws = torch.empty(art.attn_prefill_host_workspace_size(w.B, w.T, w.H, w.KV, w.hd, w.rope_base),
                             dtype=torch.uint8, device="cuda")
            for r in range(3):
                out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
                art.attn_prefill_host(q, k, v, out, rope_base=w.rope_base, workspace=ws, stream=s)
                s.synchronize()
                results[i][r] = out
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    art.attn_sync_status()
    for i, (w, q, k, v) in enumerate(cases):
        ref, _ = device_run(art, q, k, v, w)
        for r in range(3):
            assert torch.equal(results[i][r], ref)
