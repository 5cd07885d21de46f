"""The seeded generators: determinism, shapes, and the structure the workloads ask for."""
import torch

from online_softmax_12_b200 import inputs


def test_forward_inputs_are_deterministic_and_shaped():
    sh = inputs.SMALL_FWD["bf16_keymask_b2_h2_n777_d64_qstd4"]
    a = inputs.make_fwd_inputs(sh)
    b = inputs.make_fwd_inputs(sh)
    for key in ("q", "k", "v", "key_mask"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (2, 2, 777, 64) and a["q"].dtype == torch.bfloat16
    assert a["k"].shape == (2, 2, 777, 64)
    kept = a["key_mask"].sum(1)
    assert torch.equal(kept, a["kept"]) and int(kept.min()) >= 1
    # the mask is a contiguous prefix
    for bi in range(2):
        L = int(kept[bi])
        assert a["key_mask"][bi, :L].all() and not a["key_mask"][bi, L:].any()
    # Q has standard deviation 4
    assert 3.8 < a["q"].float().std() < 4.2


def test_decode_inputs_structure():
    sh = inputs.SMALL_DECODE["bf16_paged_decode_8seq_h32_kv8_d128_p16"]
    x = inputs.make_decode_inputs(sh)
    ps = x["page_size"]
    lens = x["seq_lens"]
    used = ((lens + ps - 1) // ps)
    assert x["num_pages"] == int(used.sum()) + sh.spare_pages
    # every page in use belongs to exactly one (sequence, logical page)
    owned = torch.cat([x["block_table"][s, : int(used[s])] for s in range(sh.num_seqs)])
    assert owned.unique().numel() == owned.numel()
    assert int(owned.min()) >= 0 and int(owned.max()) < x["num_pages"]
    # slots past each sequence's end are NaN, slots inside are finite
    for s in range(sh.num_seqs):
        n = int(lens[s])
        last = x["block_table"][s, (n - 1) // ps].long()
        tail = x["k_pages"][last, (n - 1) % ps + 1:]
        assert torch.isnan(tail.float()).all()
        assert torch.isfinite(x["k_pages"][last, (n - 1) % ps].float()).all()


def test_shard_range_partitions():
    for n in (0, 1, 7, 64):
        for w in (1, 2, 3, 8):
            spans = [inputs.shard_range(n, r, w) for r in range(w)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(w - 1))


def test_backward_inputs_extend_the_forward_recipe():
    from online_softmax_12_b200 import inputs

    sh = inputs.SMALL_BWD["bf16_bwd_causal_gqa_h8_kv2_n300_d128"]
    x = inputs.make_bwd_inputs(sh)
    f = inputs.make_fwd_inputs(sh)
    for n in ("q", "k", "v"):
        assert torch.equal(x[n], f[n])
    assert x["do"].dtype == torch.bfloat16 and tuple(x["do"].shape) == (sh.B, sh.H, sh.n_q, sh.d)
    g = torch.Generator().manual_seed(x["seed"] + inputs.DO_SEED_OFFSET)
    want = torch.randn(sh.B, sh.H, sh.n_q, sh.d, generator=g).to(torch.bfloat16)
    assert torch.equal(x["do"], want)
    assert torch.equal(inputs.make_bwd_inputs(sh)["do"], x["do"])
    # the key mask of a masked workload is drawn by the forward recipe, unchanged
    shm = inputs.SMALL_BWD["bf16_bwd_keymask_b2_h2_n333_d64_qstd4"]
    assert torch.equal(inputs.make_bwd_inputs(shm)["key_mask"], inputs.make_fwd_inputs(shm)["key_mask"])


def test_rising_score_inputs_structure():
    """Keys along one direction with a linearly rising coordinate: the projection of K on the
    direction of the mean query rises along the sequence; deterministic; FP8 copies decode
    to blocks with one descale each."""
    a = inputs.make_rising_score_inputs(300, 64, "bf16", 8.0, seed_index=99)
    b = inputs.make_rising_score_inputs(300, 64, "bf16", 8.0, seed_index=99)
    assert all(torch.equal(a[n], b[n]) for n in ("q", "k", "v"))
    assert a["q"].shape == (1, 2, 300, 64) and a["q"].dtype == torch.bfloat16 and not a["causal"]
    u = a["q"].float().mean(dim=(0, 1, 2))
    u = u / u.norm()
    proj = a["k"].float()[0, 0] @ u
    assert float(proj[-20:].mean()) > 7.0 and float(proj[:20].mean()) < -7.0
    assert bool((proj[1:] - proj[:-1]).mean() > 0)
    f = inputs.make_rising_score_inputs(300, 128, "fp8", 8.0, seed_index=99)
    assert f["q"].dtype == torch.uint8 and f["descale"]["k"].shape == (1, 2, 3)


def test_rising_decode_inputs_structure():
    """The rising-score decode batch keeps the decode recipe's lengths, pool and block table
    (same generator order for the lengths), and its keys rise along each sequence."""
    sh = inputs.DecodeShape(4, 8, 2, 64, 16, 100, 300, seed_index=98)
    x = inputs.make_rising_decode_inputs(sh, 0.08)
    y = inputs.make_decode_inputs(sh)
    assert torch.equal(x["seq_lens"], y["seq_lens"])
    lens = x["seq_lens"]
    used = (lens + 15) // 16
    assert x["num_pages"] == int(used.sum()) + sh.spare_pages
    u = x["q"].float().mean(dim=(0, 1))
    u = u / u.norm()
    n0 = int(lens[0])
    proj = x["k_tok"][:n0, 0].float() @ u
    assert float(proj[-10:].mean() - proj[:10].mean()) > 0.08 * (n0 - 10) * 0.8
