"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these tests needs a GPU.  Each pin is chosen so that a plausible
mistake in the oracle (a dropped term, a wrong sign or index, a transposed
operand, a wrong mask alignment) fails at least one of them.
"""
import json
import math
import os
import random

import numpy as np
import pytest
import torch

import oracle
from oracle import streaming
from conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------------------------
# Worked example: "Attenzione: softmax online, riscalamento e memoria", section 3
# --------------------------------------------------------------------------------------------

def _example_as_attention(ex, dtype=torch.float64):
    """Encode the printed scores in a d=2 attention problem: q = (1, 0), k_j = (s_j, 0), scale 1."""
    s = ex["scores"]
    q = torch.tensor([[[[1.0, 0.0]]]], dtype=dtype)
    k = torch.tensor([[[[sj, 0.0] for sj in s]]], dtype=dtype)
    v = torch.tensor([[ex["values"]]], dtype=dtype)
    return q, k, v


def test_worked_example_definition():
    ex = _golden("worked_example.json")
    q, k, v = _example_as_attention(ex)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0)
    tol = 0.5 * 10.0 ** -ex["printed_digits"] + 1e-15
    assert np.all(np.abs(o[0, 0, 0] - np.array(ex["final_o"])) <= tol)
    l_printed = ex["steps"][-1]["l"]
    m_printed = ex["steps"][-1]["m"]
    # lse = m + ln l; the printed l carries 9 digits, so ln l is known to 0.5e-9 / l
    assert abs(lse[0, 0, 0] - (m_printed + math.log(l_printed))) <= tol / l_printed + 1e-12


def test_worked_example_every_step_of_the_recurrence():
    ex = _golden("worked_example.json")
    trace = []
    streaming.stream_row(ex["scores"], ex["values"], trace=trace)
    tol = 0.5 * 10.0 ** -ex["printed_digits"] + 1e-15
    assert len(trace) == len(ex["steps"])
    for (m, l, o), row in zip(trace, ex["steps"]):
        assert m == row["m"]
        assert abs(l - row["l"]) <= tol
        assert all(abs(a - b) <= tol for a, b in zip(o, row["o"]))


def test_worked_example_wrong_rescale_is_caught():
    """The mistake the page warns about (rescale l, not u) gives its printed
    wrong value, and the pin above rejects it."""
    ex = _golden("worked_example.json")
    tol = 0.5 * 10.0 ** -ex["printed_digits"] + 1e-15
    wrong = streaming.output(streaming.stream_row(ex["scores"], ex["values"], wrong_rescale=True))
    assert abs(wrong[0] - ex["wrong_rescale_o1"]) <= tol
    assert abs(wrong[1] - ex["final_o"][1]) <= tol        # the second component hides the bug
    assert abs(wrong[0] - ex["final_o"][0]) > 0.1          # ... the first exposes it


def test_worked_example_merge_orders():
    ex = _golden("worked_example.json")
    s, v = ex["scores"], ex["values"]
    tol = 0.5 * 10.0 ** -ex["printed_digits"] + 1e-15
    for cut in (1, 2):
        a = streaming.stream_row(s[:cut], v[:cut])
        b = streaming.stream_row(s[cut:], v[cut:])
        for st in (streaming.merge(a, b), streaming.merge(b, a)):
            assert all(abs(x - y) <= tol for x, y in zip(streaming.output(st), ex["final_o"]))


def test_naive_exponential_overflows_on_the_example():
    """Section 3: exp(1000) overflows a double, which is why the maximum is subtracted."""
    with pytest.raises(OverflowError):
        math.exp(1000.0)


# --------------------------------------------------------------------------------------------
# Blocked vs materialised: section 4 experiment, re-run with our own generator
# --------------------------------------------------------------------------------------------

def test_blocked_equals_materialised():
    spec = _golden("blocked_vs_materialised.json")
    rng = np.random.default_rng(spec["seed"])
    worst = 0.0
    n_cmp = 0
    for a in spec["amplitudes"]:
        scores = rng.uniform(-a, a, spec["n_keys"]).tolist()
        values = rng.uniform(-spec["value_range"], spec["value_range"], (spec["n_keys"], spec["d_v"])).tolist()
        ref = streaming.materialised_row(scores, values)
        # the definition in C agrees with the materialised Python row
        q = torch.tensor([[[[1.0, 0.0, 0.0, 0.0]]]], dtype=torch.float64)
        k = torch.zeros(1, 1, spec["n_keys"], 4, dtype=torch.float64)
        k[0, 0, :, 0] = torch.tensor(scores, dtype=torch.float64)
        o, _ = oracle.attn_fwd(q, k, torch.tensor([[values]], dtype=torch.float64), scale=1.0)
        assert np.max(np.abs(o[0, 0, 0] - np.array(ref))) <= 1e-14
        for block in spec["blocks"]:
            got = streaming.blocked_row(scores, values, block)
            worst = max(worst, max(abs(x - y) for x, y in zip(got, ref)))
            n_cmp += 1
    assert n_cmp == 12
    # the page reports ~6.66e-16 for its draws; ours differ, the order of magnitude may not
    assert worst <= 1e-14


# --------------------------------------------------------------------------------------------
# Brute force on tiny inputs (textbook softmax without the max shift)
# --------------------------------------------------------------------------------------------

def _brute(q, k, v, scale, causal, mask):
    B, H, n_q, d = q.shape
    _, H_kv, n_kv, _ = k.shape
    o = np.zeros((B, H, n_q, d))
    lse = np.full((B, H, n_q), -math.inf)
    for b in range(B):
        for h in range(H):
            g = h // (H // H_kv)
            for i in range(n_q):
                ex = []
                for j in range(n_kv):
                    if mask is not None and not mask[b][j]:
                        continue
                    if causal and j > i + n_kv - n_q:
                        continue
                    s = scale * math.fsum(float(q[b, h, i, m]) * float(k[b, g, j, m]) for m in range(d))
                    ex.append((math.exp(s), j))
                if not ex:
                    continue
                z = math.fsum(e for e, _ in ex)
                for m in range(d):
                    o[b, h, i, m] = math.fsum(e * float(v[b, g, j, m]) for e, j in ex) / z
                lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("trial", range(12))
def test_bruteforce_tiny(trial):
    rnd = random.Random(1000 + trial)
    B = rnd.choice([1, 2])
    H_kv = rnd.choice([1, 2])
    H = H_kv * rnd.choice([1, 3])
    n_q = rnd.choice([1, 3, 5, 8])
    n_kv = rnd.choice([1, 4, 7, 8])
    d = rnd.choice([1, 3, 5])
    causal = rnd.random() < 0.5
    g = torch.Generator().manual_seed(trial)
    q = torch.randn(B, H, n_q, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, H_kv, n_kv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, H_kv, n_kv, d, generator=g, dtype=torch.float64)
    mask = None
    if rnd.random() < 0.5:
        mask = (torch.rand(B, n_kv, generator=g) < 0.7).to(torch.uint8)
    scale = rnd.choice([1.0, 0.5, 1 / math.sqrt(max(d, 1))])
    o, lse = oracle.attn_fwd(q, k, v, scale, causal, mask)
    ob, lb = _brute(q.numpy(), k.numpy(), v.numpy(), scale, causal, None if mask is None else mask.numpy())
    assert np.allclose(o, ob, rtol=1e-13, atol=1e-13)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.allclose(lse[fin], lb[fin], rtol=1e-13, atol=1e-13)
    assert np.all(o[~fin] == 0.0)


def test_bf16_and_f32_inputs_are_widened_exactly():
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, 2, 5, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, 6, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 6, 8, generator=g).to(torch.bfloat16)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.3)
    o2, l2 = oracle.attn_fwd(q.double(), k.double(), v.double(), 0.3)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = oracle.attn_fwd(q.float(), k.float(), v.float(), 0.3)
    assert np.array_equal(o1, o3) and np.array_equal(l1, l3)


# --------------------------------------------------------------------------------------------
# Library special case: torch's float64 CPU attention
# --------------------------------------------------------------------------------------------

def _torch_ref(q, k, v, scale, causal, mask):
    B, H, n_q, d = q.shape
    n_kv = k.shape[2]
    allow = torch.ones(B, 1, n_q, n_kv, dtype=torch.bool)
    if causal:
        i = torch.arange(n_q)[:, None]
        j = torch.arange(n_kv)[None, :]
        allow = allow & (j <= i + (n_kv - n_q))
    if mask is not None:
        allow = allow & mask.bool()[:, None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allow, scale=scale, enable_gqa=True)
    rep = H // k.shape[1]
    s = torch.einsum("bhid,bhjd->bhij", q, k.repeat_interleave(rep, dim=1)) * scale
    lse = torch.logsumexp(s.masked_fill(~allow, -math.inf), dim=-1)
    return o, lse


@pytest.mark.parametrize("case", [
    dict(B=1, H=1, H_kv=1, n_q=256, n_kv=256, d=64, causal=False, mask=False),     # the fp32 workload's shape
    dict(B=2, H=4, H_kv=4, n_q=130, n_kv=130, d=32, causal=True, mask=False),
    dict(B=1, H=8, H_kv=2, n_q=97, n_kv=97, d=16, causal=True, mask=False),        # GQA, 4 query heads per KV head
    dict(B=2, H=2, H_kv=2, n_q=150, n_kv=150, d=16, causal=False, mask=True),      # key padding
    dict(B=1, H=4, H_kv=1, n_q=33, n_kv=80, d=8, causal=True, mask=True),          # n_q < n_kv, bottom-right causal
])
def test_matches_torch_float64_sdpa(case):
    g = torch.Generator().manual_seed(11)
    q = torch.randn(case["B"], case["H"], case["n_q"], case["d"], generator=g, dtype=torch.float64) * 2
    k = torch.randn(case["B"], case["H_kv"], case["n_kv"], case["d"], generator=g, dtype=torch.float64)
    v = torch.randn(case["B"], case["H_kv"], case["n_kv"], case["d"], generator=g, dtype=torch.float64)
    mask = None
    if case["mask"]:
        kept = torch.randint(1, case["n_kv"] + 1, (case["B"],), generator=g)
        mask = (torch.arange(case["n_kv"])[None] < kept[:, None]).to(torch.uint8)
    scale = 1 / math.sqrt(case["d"])
    o, lse = oracle.attn_fwd(q, k, v, scale, case["causal"], mask)
    o_t, lse_t = _torch_ref(q, k, v, scale, case["causal"], mask)
    assert np.max(np.abs(o - o_t.numpy())) <= 1e-12
    assert np.max(np.abs(lse - lse_t.numpy())) <= 1e-12


# --------------------------------------------------------------------------------------------
# Invariants and closed forms
# --------------------------------------------------------------------------------------------

def _random_case(seed, B=2, H=4, H_kv=2, n=40, d=8, std=3.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, n, d, generator=g, dtype=torch.float64) * std
    k = torch.randn(B, H_kv, n, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, H_kv, n, d, generator=g, dtype=torch.float64)
    return q, k, v


def test_output_is_convex_combination_and_normaliser_in_range():
    """Section 1: weights positive and summing to one, so each output
    coordinate lies between the smallest and largest kept value; 1 <= l <= |K|."""
    q, k, v = _random_case(3)
    o, lse = oracle.attn_fwd(q, k, v, 0.4, causal=True)
    B, H, n, d = q.shape
    rep = H // k.shape[1]
    kk, vv = k.repeat_interleave(rep, 1), v.repeat_interleave(rep, 1)
    for i in range(n):
        vi = vv[:, :, : i + 1, :].numpy()
        assert np.all(o[:, :, i, :] >= vi.min(axis=2) - 1e-12)
        assert np.all(o[:, :, i, :] <= vi.max(axis=2) + 1e-12)
        s = (torch.einsum("bhd,bhjd->bhj", q[:, :, i, :], kk[:, :, : i + 1, :]) * 0.4).numpy()
        l = np.exp(lse[:, :, i] - s.max(axis=2))
        assert np.all(l >= 1 - 1e-12) and np.all(l <= i + 1 + 1e-9)


def test_zero_query_gives_uniform_weights():
    q, k, v = _random_case(4)
    q.zero_()
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=True)
    rep = q.shape[1] // k.shape[1]
    vv = v.repeat_interleave(rep, 1).numpy()
    n = q.shape[2]
    for i in range(n):
        assert np.allclose(o[:, :, i, :], vv[:, :, : i + 1, :].mean(axis=2), rtol=0, atol=1e-14)
        assert np.allclose(lse[:, :, i], math.log(i + 1), rtol=0, atol=1e-14)


def test_single_kept_key_is_exact():
    """Causal row 0 keeps one key: o = v_0 and lse = s_00 exactly."""
    q, k, v = _random_case(5)
    o, lse = oracle.attn_fwd(q, k, v, 0.7, causal=True)
    rep = q.shape[1] // k.shape[1]
    vv = v.repeat_interleave(rep, 1)
    kk = k.repeat_interleave(rep, 1)
    assert np.array_equal(o[:, :, 0, :], vv[:, :, 0, :].numpy())
    s00 = 0.7 * np.array([[math.fsum((q[b, h, 0] * kk[b, h, 0]).tolist()) for h in range(q.shape[1])]
                          for b in range(q.shape[0])])
    assert np.allclose(lse[:, :, 0], s00, rtol=0, atol=1e-12)


def test_shift_invariance():
    """Adding the same constant to every score of a row leaves o unchanged and
    shifts lse by that constant (section 1).  The shift enters through an extra
    coordinate: q gets c, every key gets 1."""
    q, k, v = _random_case(6, d=6)
    c = 37.25
    q2 = torch.cat([q, torch.full(q.shape[:-1] + (1,), c, dtype=q.dtype)], -1)
    k2 = torch.cat([k, torch.ones(k.shape[:-1] + (1,), dtype=k.dtype)], -1)
    v2 = torch.cat([v, torch.zeros(v.shape[:-1] + (1,), dtype=v.dtype)], -1)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=True)
    o2, lse2 = oracle.attn_fwd(q2, k2, v2, 0.5, causal=True)
    assert np.allclose(o2[..., :-1], o, rtol=0, atol=1e-13)
    assert np.allclose(lse2 - lse, 0.5 * c, rtol=0, atol=1e-11)


def test_dominant_key_selects_its_value_exactly():
    """With one score 800 above the others, exp(-800) underflows to 0 in
    float64, so the output is that key's value to the last bit."""
    g = torch.Generator().manual_seed(8)
    d, n = 4, 9
    v = torch.randn(1, 1, n, d, generator=g, dtype=torch.float64)
    for hot in range(n):
        k = torch.zeros(1, 1, n, d, dtype=torch.float64)
        k[0, 0, :, 0] = torch.randn(n, generator=g, dtype=torch.float64)
        k[0, 0, hot, 0] = 900.0
        q = torch.tensor([[[[1.0, 0, 0, 0]]]], dtype=torch.float64)
        o, lse = oracle.attn_fwd(q, k, v, 1.0)
        assert np.array_equal(o[0, 0, 0], v[0, 0, hot].numpy())
        assert lse[0, 0, 0] == 900.0


def test_fully_masked_row_convention():
    q, k, v = _random_case(9, B=2, H=2, H_kv=2, n=5, d=4)
    mask = torch.ones(2, 5, dtype=torch.uint8)
    mask[1] = 0
    o, lse = oracle.attn_fwd(q, k, v, 1.0, key_mask=mask)
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(lse[0]))
    # n_q > n_kv with causal alignment at the bottom right: the first rows see nothing
    q2 = torch.randn(1, 1, 6, 4, dtype=torch.float64)
    o2, lse2 = oracle.attn_fwd(q2, k[:1, :1, :4], v[:1, :1, :4], 1.0, causal=True)
    assert np.all(np.isneginf(lse2[0, 0, :2])) and np.all(np.isfinite(lse2[0, 0, 2:]))


def test_selected_rows_match_full_run():
    q, k, v = _random_case(10)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal=True)
    rows = [0, 5, 41, 79, 159, 320 - 1]
    o_r, lse_r = oracle.attn_rows(q, k, v, 0.3, True, None, rows)
    assert np.array_equal(o_r, o.reshape(-1, q.shape[-1])[rows])
    assert np.array_equal(lse_r, lse.reshape(-1)[rows])


def test_invalid_arguments_are_rejected():
    q, k, v = _random_case(11, H=3, H_kv=2)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, 1.0)
    with pytest.raises(ValueError):
        oracle.attn_rows(*_random_case(12), 1.0, rows=[10 ** 9])
