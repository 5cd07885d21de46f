"""Pins of the oracle's paged prefill: a block of query tokens per sequence (the
sequence's last positions) against its keys and values gathered through a block
table, as in the paged KV cache of "Kernel di attenzione rapida e fusione degli
operatori", section "Attenzione di tipo FlashAttention e attenzione paginata"."""
import numpy as np
import pytest
import torch

import oracle
from online_softmax_12_b200 import inputs

SMALL = inputs.PagedPrefillShape(num_seqs=4, H=8, H_kv=2, d=64, n_q=40, len_lo=40, len_hi=300, seed_index=7)


def _contig(x, s):
    """Sequence s's keys and values in logical order, from the generator's token
    arrays (no block table involved): [1, H_kv, len, d]."""
    lens = x["seq_lens"].tolist()
    start = sum(lens[:s])
    n = lens[s]
    kt = x["k_tok"][start:start + n].permute(1, 0, 2)[None].contiguous()
    vt = x["v_tok"][start:start + n].permute(1, 0, 2)[None].contiguous()
    return kt, vt


@pytest.mark.parametrize("causal", [True, False])
def test_paged_prefill_equals_contiguous_definition(causal):
    """The gather through the block table reproduces attention over the tokens in
    their logical order: the queries are the last n_q positions, so with causal
    masking query i keeps keys t <= i + len - n_q (bottom-right alignment of the
    dense oracle).  Same arithmetic in the same order: bit-identical."""
    x = inputs.make_paged_prefill_inputs(SMALL)
    o, lse = oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"],
                                  causal)
    for s in range(SMALL.num_seqs):
        kt, vt = _contig(x, s)
        o_c, lse_c = oracle.attn_fwd(x["q"][s][None], kt, vt, x["scale"], causal)
        assert np.array_equal(o[s], o_c[0])
        assert np.array_equal(lse[s], lse_c[0])
    assert np.all(np.isfinite(o)), "a NaN means a page or slot outside the sequence was read"


def test_paged_prefill_matches_torch_sdpa_after_independent_gather():
    """torch's float64 attention on keys gathered page by page with plain indexing."""
    x = inputs.make_paged_prefill_inputs(SMALL)
    o, lse = oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"])
    ps = x["page_size"]
    G = SMALL.H // SMALL.H_kv
    for s, n in enumerate(x["seq_lens"].tolist()):
        t = torch.arange(n)
        pages = x["block_table"][s, t // ps].long()
        k = x["k_pages"][pages, t % ps].double().permute(1, 0, 2).repeat_interleave(G, 0)   # [H, n, d]
        v = x["v_pages"][pages, t % ps].double().permute(1, 0, 2).repeat_interleave(G, 0)
        q = x["q"][s].double()                                                             # [H, n_q, d]
        i = torch.arange(SMALL.n_q)[:, None]
        keep = t[None, :] <= i + n - SMALL.n_q
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=x["scale"])
        sc = torch.einsum("hqd,hkd->hqk", q, k) * x["scale"]
        lse_ref = torch.logsumexp(sc.masked_fill(~keep, float("-inf")), dim=-1)
        assert np.allclose(o[s], ref.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[s], lse_ref.numpy(), rtol=0, atol=1e-12)


def test_whole_sequence_as_the_block_is_plain_causal_attention():
    """n_q = len: the block is the whole sequence and the result is ordinary causal attention."""
    sh = inputs.PagedPrefillShape(num_seqs=2, H=4, H_kv=4, d=64, n_q=33, len_lo=33, len_hi=33, seed_index=8)
    x = inputs.make_paged_prefill_inputs(sh)
    o, lse = oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"])
    for s in range(2):
        kt, vt = _contig(x, s)
        o_c, lse_c = oracle.attn_fwd(x["q"][s][None], kt, vt, x["scale"], True)
        assert np.array_equal(o[s], o_c[0])
        # causal row 0 keeps one key: O is that value row exactly, LSE its scaled score
        assert np.array_equal(o[s, :, 0], vt[0, :, 0].double().numpy().repeat(1, 0))


def test_bad_page_id_is_rejected():
    x = inputs.make_paged_prefill_inputs(SMALL)
    bt = x["block_table"].clone()
    bt[1, 0] = x["num_pages"] + 3
    with pytest.raises(ValueError):
        oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], bt, x["seq_lens"], x["scale"])
