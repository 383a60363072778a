"""The allocation-free decode entry point against the regular one (GPU).

attn_decode_noalloc serves callers that must not allocate device memory: its split
partials live in a fixed scratch array inside the library instead of a workspace the
caller passes. It runs the same kernels as attn_decode on the same inputs, only with other
scratch memory, so the test calls it through the C ABI twice in a row (the array keeps the
previous call's contents; the second call has other lengths) and requires out and lse to
be bit-identical to attn_decode with a workspace; the first call is also checked against
the fp64 oracle at the bf16 bars. It also checks that sizes beyond the array's maximum are
refused before anything runs. It sits in a file of its own that pytest collects last, and
passes alone in a fresh process as well as after the other tests.
"""
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


def _case(seed, B, H, KV, hd, Lmax, lo, hi):
    w = workloads.Decode(f"noalloc_case_{seed}", B=B, H=H, KV=KV, hd=hd, Lmax=Lmax, len_lo=lo,
                         len_hi=hi, seed=seed)
    q, kc, vc, sl, qp = workloads.decode_inputs(w)
    return [t.cuda() for t in (q, kc, vc, sl, qp)]


@pytest.mark.parametrize("KV", [8, 1])
def test_noalloc_matches_workspace_decode_twice(art, KV):
    B, H, hd, Lmax = 16, 32, 128, 4096
    for call, seed in enumerate((41, 42)):   # two calls in a row on the shared array
        q, kc, vc, sl, qp = _case(seed + KV, B, H, KV, hd, Lmax, 1, Lmax)
        ref_lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
        ref = art.attn_decode(q, kc, vc, sl, qp, lse=ref_lse, rope_base=10000.0)
        out = torch.empty_like(q)
        lse = torch.empty_like(ref_lse)
        art.attn_decode_noalloc(q, kc, vc, sl, qp, out, lse, rope_base=10000.0)
        torch.cuda.synchronize()
        art.attn_sync_status()
        assert torch.isfinite(out.float()).all()
        assert torch.equal(out, ref), f"call {call}: out differs from attn_decode"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from attn_decode"
        if call == 0:
            o_ref, l_ref = A.decode(q.cpu(), kc.cpu(), vc.cpu(), sl.tolist(), qp.tolist(), rope_base=10000.0)
            assert_close(out, o_ref, torch.bfloat16, "noalloc vs oracle")
            assert_lse_close(lse, l_ref, torch.bfloat16, "noalloc lse vs oracle")


def test_noalloc_refuses_sizes_beyond_its_scratch(art):
    import ctypes
    B, H, KV, hd, Lmax = 64, 32, 8, 128, 65536
    assert art.attn_decode_workspace_size(B, H, KV, hd, Lmax) > (8 << 20)
    q = torch.zeros(B, H, hd, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 7.0)
    kc = torch.zeros(B, 128, KV, hd, dtype=torch.bfloat16, device="cuda")  # never read
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = art.lib().attn_decode_noalloc(q.data_ptr(), kc.data_ptr(), kc.data_ptr(), sl.data_ptr(),
                                       sl.data_ptr(), out.data_ptr(), None, B, H, KV, hd, Lmax,
                                       10000.0, 0, None, 1, None)
    assert st == -3
    msg = ctypes.create_string_buffer(512)
    art.lib().attn_last_error(msg, 512)
    assert b"maximum" in msg.value
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)   # refused before anything ran
