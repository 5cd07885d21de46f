"""Parity of the paged split-KV decode and merge kernels with the float64 oracle,
and bit-exact page/slot gathering through the block table."""
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


def _to(x, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _decode(x, dev, split_tokens=0, q=None, k_pages=None, seq_lens=None, block_table=None):
    attn = _attn()
    g = _to(x, dev)
    o, lse = attn.attn_decode_paged(
        (q if q is not None else x["q"]).to(dev), (k_pages if k_pages is not None else x["k_pages"]).to(dev),
        g["v_pages"], (block_table if block_table is not None else x["block_table"]).to(dev),
        (seq_lens if seq_lens is not None else x["seq_lens"]).to(dev), x["max_seq_len"], x["scale"],
        split_tokens=split_tokens)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _small():
    return inputs.make_decode_inputs(inputs.SMALL_DECODE["bf16_paged_decode_8seq_h32_kv8_d128_p16"])


ONE_LAUNCH = -1   # ATTN_DECODE_ONE_LAUNCH: clusters of CTAs merge their partials on chip


@pytest.mark.parametrize("split_tokens", [0, 16, 48, 100, 128, 700, ONE_LAUNCH])
def test_small_decode_matches_oracle(split_tokens, cuda_device):
    """Split sizes from one token page to the whole sequence: the merge of
    "Attenzione: softmax online, riscalamento e memoria", section 4, over 1 to
    ~44 partial states per head; and the single launch, whose cluster of 8 CTAs
    merges its 8 partial states through distributed shared memory."""
    x = _small()
    o, lse = _decode(x, cuda_device, split_tokens)
    assert _attn().check_status() == 0
    o_ref, lse_ref = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"],
                                         x["scale"])
    compare(o, lse, o_ref, lse_ref, "bf16")


def test_dominant_token_is_gathered_bit_exactly(cuda_device):
    """Make one logical position's key dominate every other score by far more
    than 127 in base 2: every other weight is exactly 0 after ex2, so the output
    must be that token's value row, bit for bit, wherever the block table put it.
    Positions: first and last token, every page boundary around them, the middle."""
    x = _small()
    ps = x["page_size"]
    H = x["q"].shape[1]
    H_kv = x["k_pages"].shape[2]
    G = H // H_kv
    q = x["q"].clone()
    # one query head per kv group carries the probe; the dominant key is alpha * q for that head
    for s, n in enumerate(x["seq_lens"].tolist()):
        positions = sorted({0, n - 1, n // 2} | {p for p in range(0, n, ps)} | {p - 1 for p in range(ps, n, ps)})
        for split in (0, 16, ONE_LAUNCH):
            for pos in positions[:: max(1, len(positions) // 12)]:
                kp = x["k_pages"].clone()
                page = int(x["block_table"][s, pos // ps])
                for g in range(H_kv):
                    kp[page, pos % ps, g] = (q[s, g * G].float() * 20).to(torch.bfloat16)
                o, lse = _decode(x, cuda_device, split, k_pages=kp, q=q)
                want = x["v_pages"][page, pos % ps].float().numpy()   # [H_kv, d]
                for g in range(H_kv):
                    assert np.array_equal(o[s, g * G], want[g]), (s, pos, g)


def test_zero_query_averages_exactly_the_sequence(cuda_device):
    """q = 0 gives uniform weights: O is the mean of V over exactly len_s tokens.
    A NaN would mean a slot past the end or a spare page was read."""
    x = _small()
    q = torch.zeros_like(x["q"])
    o_ref, lse_ref = oracle.decode_paged(q, x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], x["scale"])
    for split in (0, ONE_LAUNCH):
        o, lse = _decode(x, cuda_device, split, q=q)
        assert np.all(np.isfinite(o))
        compare(o, lse, o_ref, lse_ref, "bf16")
        assert np.allclose(lse, np.log(x["seq_lens"].numpy().astype(np.float64))[:, None], atol=1e-5)


def test_empty_sequence_and_bad_table_entries(cuda_device):
    attn = _attn()
    x = _small()
    lens = x["seq_lens"].clone()
    lens[3] = 0
    lens[5] = 3          # fewer pages than the cluster has CTAs: most shares are empty
    for split in (0, ONE_LAUNCH):
        o, lse = _decode(x, cuda_device, split, seq_lens=lens)
        assert attn.check_status() == attn.OK
        assert np.all(o[3] == 0) and np.all(np.isneginf(lse[3]))
        o_ref, lse_ref = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], lens, x["scale"])
        compare(o, lse, o_ref, lse_ref, "bf16")
    # a page id outside the pool is skipped (never dereferenced) and reported
    bt = x["block_table"].clone()
    bt[2, 0] = x["num_pages"] + 5
    bt[5, 1] = -3
    o, lse = _decode(x, cuda_device, 0, block_table=bt)
    assert attn.check_status() == attn.ERR_INVALID_ARG
    assert np.all(np.isfinite(o))
    assert attn.check_status() == attn.OK  # the word was cleared


@pytest.mark.parametrize("split", [0, ONE_LAUNCH])
def test_deterministic(split, cuda_device):
    x = _small()
    a = _decode(x, cuda_device, split)
    b = _decode(x, cuda_device, split)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("split_tokens", [0, 16, 128, ONE_LAUNCH])
def test_reference_moves_every_block(split_tokens, cuda_device):
    """Scores that rise along each sequence: every 128 tokens lift every head's maximum by
    more than the rescale threshold (8 in base 2), so the split kernel rescales its running
    state block after block and the merge combines partials whose maxima differ by far more
    than that; every element against the oracle (the premise is checked on the inputs)."""
    sh = inputs.DecodeShape(8, 32, 8, 128, 16, 300, 700, seed_index=43)
    x = inputs.make_rising_decode_inputs(sh, 0.08)
    q, kt, G = x["q"].double(), x["k_tok"].double(), sh.H // sh.H_kv
    moved, start = [], 0
    for s, n in enumerate(x["seq_lens"].tolist()):
        sc = x["scale"] * torch.einsum("hd,tgd->htg", q[s], kt[start:start + n])
        start += n
        sc = torch.stack([sc[h, :, h // G] for h in range(sh.H)])
        run = sc[:, :128].amax(1)
        for j0 in range(128, n - 127, 128):
            bm = sc[:, j0:j0 + 128].amax(1)
            moved.append(((bm - run) / np.log(2.0) > 8.0).double().mean().item())
            run = torch.maximum(run, bm)
    assert np.mean(moved) > 0.9, np.mean(moved)
    o_ref, lse_ref = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"],
                                         x["scale"])
    o, lse = _decode(x, cuda_device, split_tokens)
    assert _attn().check_status() == 0
    print(split_tokens, compare(o, lse, o_ref, lse_ref, "bf16"))


def test_full_size_decode_every_sequence(cuda_device):
    """The benchmark's decode workload at full size (64 sequences of 512..8192
    tokens), in the benchmark's launch configuration and in the other decode path;
    every element of every sequence's output and log-sum-exp against the oracle."""
    sh = inputs.DECODE_WORKLOADS["bf16_paged_decode_64seq_h32_kv8_d128_p16"]
    x = inputs.make_decode_inputs(sh)
    o_ref, lse_ref = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"],
                                         x["scale"])
    for split in (0, 1024, ONE_LAUNCH):
        o, lse = _decode(x, cuda_device, split)
        assert _attn().check_status() == 0
        assert np.all(np.isfinite(o))
        info = compare(o, lse, o_ref, lse_ref, "bf16")
        print(split, info)


@pytest.mark.parametrize("page_size, d, G", [(8, 128, 4), (32, 64, 2), (16, 64, 8), (16, 128, 1)])
def test_page_sizes_head_dims_and_group_sizes(page_size, d, G, cuda_device):
    """16-token pages take the tensor-core kernel, other page sizes the CUDA-core
    kernel; both against the oracle, for d = 64 / 128 and 1 to 8 query heads per kv head."""
    sh = inputs.DecodeShape(6, 2 * G, 2, d, page_size, 1, 300, seed_index=4)
    x = inputs.make_decode_inputs(sh)
    for split in (0, 48):
        o, lse = _decode(x, cuda_device, split)
        assert _attn().check_status() == 0
        o_ref, lse_ref = oracle.decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"],
                                             x["scale"])
        compare(o, lse, o_ref, lse_ref, "bf16", bf16_output=True)
