"""The bounded on-chip waits of the fused forward, made to run out.

Every wait of the fused kernel for another role of its CTA (an operand copy,
an MMA, an epilogue warp) has a limit; one that runs out flags
HAD_ERR_TIMEOUT, lets the copies and MMAs already in flight complete, frees
the CTA's tensor memory and returns.  Here the limit is set to one
microsecond, far below the time the first operand copy takes, so the waits
give up; the call must report the timeout, and a normal call on the same
device afterwards must still give the exact result (its CTAs could allocate
tensor memory, so the aborted ones freed theirs).
"""
import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _inputs(B, H, n, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, n, d, generator=g).to(torch.bfloat16) for _ in range(3))
    return (q.cuda(), k.cuda(), v.cuda(), synth.per_head_sigma(q).cuda(),
            synth.per_head_sigma(k).cuda())


@pytest.mark.parametrize("d", [64, 128])
def test_wait_limit_runs_out_then_the_device_is_usable(d):
    from sparse_attention_sigma_b200 import had
    B, H, n, N = 1, 2, 300, 40
    q, k, v, sq, sk = _inputs(B, H, n, d, 91 + d)
    tau = 1 / math.sqrt(d)
    ref = had.had_attention_fwd(q, k, v, sq, sk, N, tau)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    prev = had.had_set_wait_limit_ns(1000)
    try:
        had.had_attention_fwd(q, k, v, sq, sk, N, tau, dev_status=status)
        torch.cuda.synchronize()
    finally:
        had.had_set_wait_limit_ns(prev)
    assert status.item() & (1 << had.HAD_ERR_TIMEOUT)
    status.zero_()
    again = had.had_attention_fwd(q, k, v, sq, sk, N, tau, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(again, ref)
