"""Parity of the paged prefill (a block of query tokens per sequence against its
paged KV cache, through the tcgen05 prefill kernel with a page-gathering
producer) with the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from online_softmax_12_b200 import inputs
from parity import compare

pytestmark = pytest.mark.gpu


def _attn():
    from online_softmax_12_b200 import attn

    return attn


def _run(x, dev, causal=None, block_table=None, seq_lens=None, out_f32=False):
    attn = _attn()
    c = x["causal"] if causal is None else causal
    o, lse = attn.attn_prefill_paged(x["q"].to(dev), x["k_pages"].to(dev), x["v_pages"].to(dev),
                                     (x["block_table"] if block_table is None else block_table).to(dev),
                                     (x["seq_lens"] if seq_lens is None else seq_lens).to(dev), x["scale"], c,
                                     out_f32=out_f32)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _ref(x, causal=None):
    c = x["causal"] if causal is None else causal
    return oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"], c)


CASES = {
    # ragged query block (200 = 128 + 72), lengths from the block itself to several key blocks
    "d128_gqa4_nq200": inputs.PagedPrefillShape(4, 8, 2, 128, 200, 200, 700, seed_index=11),
    "d64_gqa2_nq130": inputs.PagedPrefillShape(3, 4, 2, 64, 130, 130, 520, seed_index=12),
    # the block is the whole sequence (plain causal prefill), lengths not multiples of 16
    "d128_whole_333": inputs.PagedPrefillShape(2, 4, 4, 128, 333, 333, 333, seed_index=13),
    # short sequences: one partly filled key block, one query row
    "d128_nq1_short": inputs.PagedPrefillShape(5, 8, 1, 128, 1, 1, 60, seed_index=14),
    # long sequences, many key blocks and pages, 8 query heads per kv head
    "d128_gqa8_long": inputs.PagedPrefillShape(2, 16, 2, 128, 256, 1500, 3000, seed_index=15),
}


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("causal", [True, False])
def test_paged_prefill_matches_oracle(name, causal, cuda_device):
    x = inputs.make_paged_prefill_inputs(CASES[name])
    o_ref, lse_ref = _ref(x, causal)
    # the arithmetic, on the fp32 output, against the literal bound
    o32, lse32 = _run(x, cuda_device, causal, out_f32=True)
    assert _attn().check_status() == 0
    assert np.all(np.isfinite(o32)), "NaN from a slot past a sequence's end or a spare page"
    print(name, causal, "fp32 out", compare(o32, lse32, o_ref, lse_ref, "bf16"))
    o, lse = _run(x, cuda_device, causal)
    assert _attn().check_status() == 0
    # the bf16 output is the fp32 output rounded to nearest
    assert np.array_equal(lse, lse32)
    assert np.array_equal(o, torch.from_numpy(o32).to(torch.bfloat16).float().numpy())
    print(name, causal, "bf16 out", compare(o, lse, o_ref, lse_ref, "bf16", bf16_output=True))


def test_lengths_shorter_than_the_query_block_give_empty_rows(cuda_device):
    """seq_lens[s] < n_q: causal rows before the first key keep nothing (O = 0, LSE = -inf)."""
    x = inputs.make_paged_prefill_inputs(CASES["d64_gqa2_nq130"])
    lens = x["seq_lens"].clone()
    lens[1] = 100          # queries 0..29 of sequence 1 see no key
    lens[2] = 0            # an empty sequence
    o, lse = _run(x, cuda_device, True, seq_lens=lens)
    assert _attn().check_status() == 0
    o_ref, lse_ref = oracle.prefill_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], lens, x["scale"], True)
    compare(o, lse, o_ref, lse_ref, "bf16", bf16_output=True)
    o32, lse32 = _run(x, cuda_device, True, seq_lens=lens, out_f32=True)
    compare(o32, lse32, o_ref, lse_ref, "bf16")
    assert np.all(np.isneginf(lse[1, :, :30])) and np.all(o[1, :, :30] == 0)
    assert np.all(np.isneginf(lse[2])) and np.all(o[2] == 0)


def test_bad_page_id_is_reported(cuda_device):
    attn = _attn()
    x = inputs.make_paged_prefill_inputs(CASES["d128_gqa4_nq200"])
    bt = x["block_table"].clone()
    bt[0, 1] = x["num_pages"] + 7
    _run(x, cuda_device, True, block_table=bt)
    assert attn.check_status() == attn.ERR_INVALID_ARG
    assert attn.check_status() == attn.OK


def test_deterministic(cuda_device):
    x = inputs.make_paged_prefill_inputs(CASES["d128_gqa4_nq200"])
    a = _run(x, cuda_device)
    b = _run(x, cuda_device)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_matches_the_dense_kernel_on_the_same_tokens(cuda_device):
    """The same queries and keys through attn_fwd (contiguous K and V, the last n_q
    positions as queries) and through the paged path: the kernels do the same
    arithmetic in the same order, so the outputs agree bit for bit."""
    attn = _attn()
    sh = CASES["d128_whole_333"]
    x = inputs.make_paged_prefill_inputs(sh)
    o_p, lse_p = _run(x, cuda_device, True)
    start = 0
    for s, n in enumerate(x["seq_lens"].tolist()):
        kt = x["k_tok"][start:start + n].permute(1, 0, 2)[None].contiguous().to(cuda_device)
        vt = x["v_tok"][start:start + n].permute(1, 0, 2)[None].contiguous().to(cuda_device)
        o_d, lse_d = attn.attn_fwd(x["q"][s][None].to(cuda_device), kt, vt, x["scale"], True)
        torch.cuda.synchronize()
        assert np.array_equal(o_d[0].float().cpu().numpy(), o_p[s])
        assert np.array_equal(lse_d[0].cpu().numpy(), lse_p[s])
        start += n


def test_full_size_workload(cuda_device):
    """The benchmark's paged-prefill workload (8 sequences of 4096..16384 tokens, the
    newest 2048 as causal queries) in its launch configuration: every row of query
    heads 0 and 31 of every sequence, plus sampled rows of the other heads, against
    the oracle on keys gathered densely through the block table; bf16 and fp32 output."""
    sh = inputs.PAGED_PREFILL_WORKLOADS["bf16_paged_prefill_8seq_chunk2048_h32_kv8_d128_p16"]
    x = inputs.make_paged_prefill_inputs(sh)
    o, lse = _run(x, cuda_device, True)
    assert _attn().check_status() == 0
    assert np.all(np.isfinite(o))
    o32, lse32 = _run(x, cuda_device, True, out_f32=True)
    assert _attn().check_status() == 0
    rng = np.random.default_rng(3)
    ps = x["page_size"]
    for s in range(sh.num_seqs):
        n = int(x["seq_lens"][s])
        t = torch.arange(n)
        pages = x["block_table"][s, t // ps].long()
        k = x["k_pages"][pages, t % ps].permute(1, 0, 2)[None].contiguous()   # [1, H_kv, n, d]
        v = x["v_pages"][pages, t % ps].permute(1, 0, 2)[None].contiguous()
        rows = np.unique(np.concatenate([np.arange(sh.n_q), np.arange((sh.H - 1) * sh.n_q, sh.H * sh.n_q),
                                         rng.choice(sh.H * sh.n_q, size=48, replace=False)]))
        o_ref, lse_ref = oracle.attn_rows(x["q"][s][None], k, v, x["scale"], True, rows=rows)
        h, i = rows // sh.n_q, rows % sh.n_q
        compare(o[s][h, i], lse[s][h, i], o_ref, lse_ref, "bf16", bf16_output=True)
        compare(o32[s][h, i], lse32[s][h, i], o_ref, lse_ref, "bf16")
