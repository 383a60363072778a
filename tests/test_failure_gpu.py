"""Failure detection on the GPU without a GPU fault.

A test hook makes every CTA of the tensor-core decode kernel wait on an mbarrier that
nothing signals, with a 2 ms bound. Each CTA must give up, record ATTN_ERR_TIMEOUT in the
device status word, let its own copies and MMAs finish, free its tensor memory and exit;
the host reads the status with attn_sync_status, and the context stays usable: the next
call gives the oracle's result.
"""
import os

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


def _case():
    w = workloads.Decode("timeout_case", B=2, H=8, KV=2, hd=128, Lmax=512, len_lo=100, len_hi=512,
                         seed=77)
    q, kc, vc, sl, qp = workloads.decode_inputs(w)
    return w, q, kc, vc, sl, qp


def test_decode_wait_times_out_and_context_survives(art):
    w, q, kc, vc, sl, qp = _case()
    dq, dkc, dvc, dsl, dqp = q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), qp.cuda()
    art.attn_sync_status()                       # start clean
    os.environ["ATTN_TEST_DECODE_STALL_NS"] = "2000000"
    try:
        art.attn_decode(dq, dkc, dvc, dsl, dqp, rope_base=w.rope_base)
    finally:
        del os.environ["ATTN_TEST_DECODE_STALL_NS"]
    with pytest.raises(art.AttnError) as e:
        art.attn_sync_status()
    assert e.value.status == -5                  # ATTN_ERR_TIMEOUT
    art.attn_sync_status()                       # the word was cleared
    out = art.attn_decode(dq, dkc, dvc, dsl, dqp, rope_base=w.rope_base)
    torch.cuda.synchronize()
    art.attn_sync_status()
    ref, _ = A.decode(q, kc, vc, sl.tolist(), qp.tolist(), rope_base=w.rope_base)
    assert_close(out, ref, torch.bfloat16, "decode after a timed-out call")
