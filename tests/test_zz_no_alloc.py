"""attn_decode_paged_static: the paged decode for callers that cannot allocate
device memory (a host callback, an allocator's own code path, a plugin whose
framework owns every allocation).  It keeps the split-KV partial states in the
library's fixed 32 MiB device array instead of a caller workspace.

Checked through the C ABI against the regular attn_decode_paged, with the
bf16 tolerance every decode test uses, on two calls in a row (the second call
reuses the array the first one left behind).  This file sorts last so that a
run stopping at the first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from online_softmax_12_b200 import inputs
from parity import TOL

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_call(attn, x, q, o, lse, split_tokens=0):
    S, H, d = q.shape
    P, page, H_kv, _ = x["k_pages"].shape
    return attn._lib.attn_decode_paged_static(
        _p(q), _p(x["k_pages"]), _p(x["v_pages"]), _p(x["block_table"]), _p(x["seq_lens"]), S, H, H_kv, d, page,
        x["block_table"].shape[1], P, x["max_seq_len"], split_tokens, float(x["scale"]), _p(o), _p(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b, la, lb):
    tol = TOL["bf16"]
    assert np.max(np.abs(a - b)) <= tol["o"]
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(la))
    assert np.all(np.abs(la[fin] - lb[fin]) <= tol["lse"] * np.maximum(np.abs(lb[fin]), 1.0))


@pytest.mark.parametrize("name", ["bf16_paged_decode_8seq_h32_kv8_d128_p16", "bf16_paged_decode_64seq_h32_kv8_d128_p16"])
def test_static_scratch_decode_matches_workspace_decode(name, cuda_device):
    from online_softmax_12_b200 import attn

    sh = {**inputs.SMALL_DECODE, **inputs.DECODE_WORKLOADS}[name]
    host = inputs.make_decode_inputs(sh)
    x = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    S, H, d = x["q"].shape
    queries = [x["q"], (x["q"].float() * -0.5).to(torch.bfloat16)]   # two different calls in a row
    for q in queries:
        o_ref, lse_ref = attn.attn_decode_paged(q, x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"],
                                                x["max_seq_len"], x["scale"])
        o = torch.full_like(q, float("nan"))
        lse = torch.full((S, H), float("nan"), dtype=torch.float32, device=cuda_device)
        st = _static_call(attn, x, q, o, lse)
        assert st == attn.OK, attn.last_error()
        torch.cuda.synchronize()
        assert attn.check_status() == attn.OK
        _close(o.float().cpu().numpy(), o_ref.float().cpu().numpy(), lse.cpu().numpy(), lse_ref.cpu().numpy())


def test_static_scratch_rejects_requests_beyond_its_size(cuda_device):
    from online_softmax_12_b200 import attn

    x = inputs.make_decode_inputs(inputs.SMALL_DECODE["bf16_paged_decode_8seq_h32_kv8_d128_p16"])
    x = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    q = x["q"]
    o = torch.zeros_like(q)
    lse = torch.zeros(q.shape[0], q.shape[1], dtype=torch.float32, device=cuda_device)
    # one-token splits over the whole block table (44 pages of 16 tokens): 8 x 32 x 704 partial
    # states of 4 + 128 fp32, about 95 MB
    big = dict(x)
    big["max_seq_len"] = x["block_table"].shape[1] * x["k_pages"].shape[1]
    need = attn.decode_workspace_bytes(q.shape[0], q.shape[1], x["k_pages"].shape[2], q.shape[2],
                                       big["max_seq_len"], 1)
    assert need > 32 << 20
    st = _static_call(attn, big, q, o, lse, split_tokens=1)
    assert st == attn.ERR_INVALID_ARG
    assert "32" in attn.last_error() or "scratch" in attn.last_error()
    torch.cuda.synchronize()
    assert torch.all(o == 0)   # nothing was launched
