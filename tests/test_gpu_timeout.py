"""The failure path of the bounded waits, run on the GPU without faulting it.

Every wait inside the kernels gives up after a time limit, records where, raises
the CTA's abort flag and lets the kernel end with its copies drained and its
tensor memory freed ("Attenzione: softmax online, riscalamento e memoria",
section 5, asks for explicit conventions instead of silent failure; here a lost
arrival becomes an error status instead of a hang).  The test hook shortens the
limit to 1 ms and has the forward kernel's producer withhold its first V copy
(the copy is never issued, so nothing lands later), on the smallest shape: one
work item of one key block, one CTA.  No trap, no fault, no endless loop.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import compare

pytestmark = pytest.mark.gpu

# wait-site codes of the tensor-core forward kernel (the kernel's WaitSite enum)
SITE_VFULL, SITE_OFINAL = 6, 9


def test_a_withheld_copy_times_out_and_the_next_call_is_clean(cuda_device):
    from online_softmax_12_b200 import attn

    g = torch.Generator().manual_seed(7)
    q, k, v = (torch.randn(1, 1, 64, 128, generator=g).to(torch.bfloat16) for _ in range(3))
    qd, kd, vd = (t.to(cuda_device) for t in (q, k, v))
    assert attn.check_status() == attn.OK          # start from a clear status word
    attn.testing_set(1_000_000, attn.TEST_DROP_FIRST_V)
    try:
        attn.attn_fwd(qd, kd, vd, 128 ** -0.5, False)
        torch.cuda.synchronize()                    # the kernel ended: the wait gave up
        detail = attn.status_detail()
    finally:
        attn.testing_set(0, 0)
    assert attn.check_status() == attn.ERR_TIMEOUT, attn.last_error()
    assert detail[0] & 0x1                          # the timeout flag
    site, warp = detail[1] & 0xFF, (detail[1] >> 8) & 0xFF
    assert detail[1] & 0x80000000
    # the MMA issuer (warp 8) waiting for the withheld V tile starts first; the softmax
    # warps of the only query tile (warps 0-3) wait for the finished output just after it
    assert (site, warp) == (SITE_VFULL, 8) or (site == SITE_OFINAL and warp < 4), (site, warp)
    assert detail[2] == 0                           # CTA 0
    assert attn.check_status() == attn.OK           # the read cleared it

    # the same call again on the same device: normal status and parity
    o, lse = attn.attn_fwd(qd, kd, vd, 128 ** -0.5, False, out_f32=True)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 128 ** -0.5, False)
    compare(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "bf16")
    assert np.all(np.isfinite(o.cpu().numpy()))
