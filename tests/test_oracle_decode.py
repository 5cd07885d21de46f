"""Pins of the oracle's paged decode (one query token per sequence through a
block table of fixed-size pages, as in the paged KV cache of "Kernel di
attenzione rapida e fusione degli operatori", section "Attenzione di tipo
FlashAttention e attenzione paginata")."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_12_b200 import inputs


def _small():
    return inputs.make_decode_inputs(inputs.SMALL_DECODE["bf16_paged_decode_8seq_h32_kv8_d128_p16"])


def test_paged_decode_equals_contiguous_definition():
    """The gather through the block table must reproduce attention over the
    tokens in their logical order (which the generator also keeps, before it
    scatters them into pages).  Both runs do the same arithmetic in the same
    order, so the results are bit-identical."""
    x = _small()
    o, lse = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"])
    start = 0
    for s, n in enumerate(x["seq_lens"].tolist()):
        kt = x["k_tok"][start:start + n].permute(1, 0, 2)[None].contiguous()   # [1, H_kv, n, d]
        vt = x["v_tok"][start:start + n].permute(1, 0, 2)[None].contiguous()
        q = x["q"][s][None, :, None, :].contiguous()                             # [1, H, 1, d]
        o_c, lse_c = oracle.attn_fwd(q, kt, vt, x["scale"])
        assert np.array_equal(o[s], o_c[0, :, 0, :])
        assert np.array_equal(lse[s], lse_c[0, :, 0])
        start += n
    assert np.all(np.isfinite(o)), "a NaN means a page or slot outside the sequence was read"


def test_paged_decode_matches_torch_sdpa_after_independent_gather():
    x = _small()
    o, lse = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"])
    ps = x["page_size"]
    H = x["q"].shape[1]
    for s, n in enumerate(x["seq_lens"].tolist()):
        t = torch.arange(n)
        pages = x["block_table"][s, t // ps].long()
        kt = x["k_pages"][pages, t % ps].double()          # [n, H_kv, d]
        vt = x["v_pages"][pages, t % ps].double()
        q = x["q"][s].double()                              # [H, d]
        H_kv = kt.shape[1]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[None, :, None, :], kt.permute(1, 0, 2)[None], vt.permute(1, 0, 2)[None], scale=x["scale"],
            enable_gqa=True)[0, :, 0, :]
        assert np.max(np.abs(o[s] - ref.numpy())) <= 1e-12
        sc = torch.einsum("hd,nhd->hn", q, kt.repeat_interleave(H // H_kv, 1)) * x["scale"]
        assert np.max(np.abs(lse[s] - torch.logsumexp(sc, -1).numpy())) <= 1e-12


def test_dominant_token_is_gathered_bit_exactly():
    """Make one logical position's key dominate by 800 (exp(-800) == 0 in
    float64): the output must be exactly that token's value row, found
    through the block table."""
    x = _small()
    ps = x["page_size"]
    q = torch.zeros_like(x["q"])
    q[:, :, 0] = 1.0
    k_pages = torch.zeros_like(x["k_pages"])
    for s, n in enumerate(x["seq_lens"].tolist()):
        for p in sorted({0, n - 1, min(ps, n - 1), n // 2}):
            kp = k_pages.clone()
            kp[x["block_table"][s, p // ps].long(), p % ps, :, 0] = 800.0
            o, lse = oracle.decode_paged(q[s:s + 1], kp, x["v_pages"], x["block_table"][s:s + 1],
                                         x["seq_lens"][s:s + 1], 1.0)
            want = x["v_pages"][x["block_table"][s, p // ps].long(), p % ps]     # [H_kv, d]
            H, H_kv = q.shape[1], want.shape[0]
            assert np.array_equal(o[0], want.double().repeat_interleave(H // H_kv, 0).numpy())
            assert np.all(lse[0] == 800.0)


def test_empty_sequence_and_bad_page_ids():
    x = _small()
    lens = x["seq_lens"].clone()
    lens[0] = 0
    o, lse = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], lens, x["scale"])
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    bt = x["block_table"].clone()
    bt[1, 0] = x["num_pages"]
    with pytest.raises(ValueError):
        oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], bt, x["seq_lens"], x["scale"])
    lens2 = x["seq_lens"].clone()
    lens2[2] = x["max_pages_per_seq"] * x["page_size"] + 1
    with pytest.raises(ValueError):
        oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], lens2, x["scale"])
