"""Parity of the block-scaled FP8 E4M3 forward (tcgen05 kind::f8f6f4) with the float64
oracle on the decoded inputs.

Tolerance (derived; the pages fix none for FP8).  The inputs are exact (the oracle
uses the same block-decoded values) and fp32 accumulates; the one rounding that
matters is P to E4M3.  ``oracle.fp8_error_bound`` gives, per element, the most that
rounding can move O under the kernel's rounding model (weights measured 2^8 above
the running maximum, times the V block's factor, rounded to nearest E4M3, O
normalised by the sum of the rounded weights):
sum_k E_k |v_kc - O_c| / (sum P - sum E) with E_k half an E4M3 ulp of weight k (2^-4
relative, 2^-10 absolute in the subnormal range).  The bar adds 1e-5 of the weights'
spread of V (the fp32 exponent arithmetic and ex2.approx), 1e-6 of max|v| (fp32
accumulation), and half a bf16 ulp for a bf16 output.  The LSE comes from the
unrounded weights: the bf16 bound 1e-3 relative.  The bar is tight enough that a
single block given the wrong descale fails it (tested below).
"""
import numpy as np
import pytest
import torch

import oracle
from online_softmax_12_b200 import inputs
from parity import half_ulp_bf16

pytestmark = pytest.mark.gpu


def _attn():
    from online_softmax_12_b200 import attn

    return attn


def _run(x, dev, out_f32=False):
    attn = _attn()
    d = {n: t.to(dev) for n, t in x["descale"].items()}
    km = x["key_mask"].to(dev) if x.get("key_mask") is not None else None
    o, lse = attn.attn_fwd_fp8(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), d["q"], d["k"], d["v"], x["scale"],
                               x["causal"], km, out_f32=out_f32)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _decoded(x, descale=None):
    d = x["descale"] if descale is None else descale
    return tuple(oracle.decode_e4m3_blocks(x[n], d[n]) for n in ("q", "k", "v"))


def _ref_and_bar(x, rows=None, descale=None):
    """(o_ref, lse_ref, bar) for the given rows (flat ids; None = all), shaped [rows, d]."""
    d = x["descale"] if descale is None else descale
    q, k, v = _decoded(x, d)
    o_ref, lse_ref = oracle.attn_rows(q, k, v, x["scale"], x["causal"], x.get("key_mask"), rows)
    bound, spread = oracle.fp8_error_bound(q, k, v, d["v"], x["scale"], x["causal"], x.get("key_mask"), rows)
    bar = bound + 1e-5 * spread + 1e-6 * float(np.max(np.abs(v)))
    return o_ref, lse_ref, bar


def _check(o, lse, o_ref, lse_ref, bar, bf16_out):
    """o, lse: [rows, d], [rows].  Raises AssertionError outside the bar."""
    bound = bar + (half_ulp_bf16(o_ref) if bf16_out else 0.0)
    err = np.abs(o - o_ref)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(err <= bound), f"max excess {float(np.max(err - bound)):.3e}, {int(np.sum(err > bound))} elements"
    fin = ~empty
    d = np.abs(lse[fin] - lse_ref[fin])
    assert np.all(d <= 1e-3 * np.maximum(np.abs(lse_ref[fin]), 1.0)), float(np.max(d))
    return float(np.max(err)), float(np.max(err / np.maximum(bound, 1e-30)))


CASES = {
    "causal_gqa_n777": inputs.FwdShape(1, 4, 2, 777, 777, 128, "fp8", True, seed_index=31),
    "noncausal_b2_n300_nkv1000": inputs.FwdShape(2, 2, 2, 300, 1000, 128, "fp8", False, seed_index=32),
    "keymask_b2_n600_qstd4": inputs.FwdShape(2, 2, 1, 600, 600, 128, "fp8", False, q_std=4.0, prefix_mask=True,
                                             seed_index=33),
    # bottom-right causal alignment with fewer and with more queries than keys (the latter leaves
    # 700 rows per head with no key: O = 0, LSE = -inf)
    "causal_b2_nq300_nkv1000": inputs.FwdShape(2, 4, 2, 300, 1000, 128, "fp8", True, seed_index=34),
    "causal_nq1000_nkv300": inputs.FwdShape(1, 4, 2, 1000, 300, 128, "fp8", True, seed_index=35),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_forward_matches_oracle(name, cuda_device):
    sh = CASES[name]
    x = inputs.make_fwd_inputs(sh)
    o_ref, lse_ref, bar = _ref_and_bar(x)
    o, lse = _run(x, cuda_device, out_f32=True)
    print(name, "fp32 out (max err, max err / bar)", _check(o.reshape(-1, sh.d), lse.reshape(-1), o_ref, lse_ref,
                                                            bar, False))
    o, lse = _run(x, cuda_device)
    print(name, "bf16 out", _check(o.reshape(-1, sh.d), lse.reshape(-1), o_ref, lse_ref, bar, True))


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_fp8_bar_fails_a_single_mis_scaled_block(which, cuda_device):
    """The GPU output with the true descales, checked against an oracle in which one block's
    descale is doubled (the mistake planted on the CPU side): the bar must reject it."""
    sh = CASES["causal_gqa_n777"]
    x = inputs.make_fwd_inputs(sh)
    o, lse = _run(x, cuda_device, out_f32=True)
    wrong = {n: t.clone() for n, t in x["descale"].items()}
    wrong[which][0, 0, 2] *= 2.0            # rows or keys 256..383 of head 0
    o_ref, lse_ref, bar = _ref_and_bar(x, descale=wrong)
    with pytest.raises(AssertionError):
        _check(o.reshape(-1, sh.d), lse.reshape(-1), o_ref, lse_ref, bar, False)


def test_fp8_one_kept_key_gives_its_value(cuda_device):
    """Causal row 0 keeps one key: its weight is the only one, so O is that value row
    (its block's descale times the decoded bytes) to fp32 rounding."""
    x = inputs.make_fwd_inputs(CASES["causal_gqa_n777"])
    o, lse = _run(x, cuda_device, out_f32=True)
    v0 = oracle.decode_e4m3_blocks(x["v"], x["descale"]["v"])[0, :, 0, :]          # [H_kv, d]
    G = 2
    for h in range(4):
        assert np.allclose(o[0, h, 0], v0[h // G], rtol=1e-6, atol=0)


def test_fp8_bad_descale_is_reported(cuda_device):
    attn = _attn()
    x = inputs.make_fwd_inputs(CASES["causal_gqa_n777"])
    x["descale"] = {n: t.clone() for n, t in x["descale"].items()}
    x["descale"]["k"][0, 1, 3] = 0.0
    d = {n: t.to(cuda_device) for n, t in x["descale"].items()}
    attn.attn_fwd_fp8(x["q"].to(cuda_device), x["k"].to(cuda_device), x["v"].to(cuda_device), d["q"], d["k"], d["v"],
                      x["scale"], True)
    assert attn.check_status() == attn.ERR_INVALID_ARG
    assert attn.check_status() == attn.OK


def test_fp8_deterministic(cuda_device):
    x = inputs.make_fwd_inputs(CASES["causal_gqa_n777"])
    a = _run(x, cuda_device)
    b = _run(x, cuda_device)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp8_reference_moves_every_block(cuda_device):
    """Scores that rise along the keys: each key block holds a new maximum for every row, so
    the FP8 kernel (reference at every new maximum) rescales O in every block after the first.
    Every element against the oracle at the derived bar, fp32 and bf16 output."""
    x = inputs.make_rising_score_inputs(777, 128, "fp8", 8.0, seed_index=42)
    q, k, _ = _decoded(x)
    s = x["scale"] * np.einsum("bhid,bhjd->bhij", q, k)
    run, moved = s[..., :128].max(-1), []
    for j0 in range(128, s.shape[-1] - 127, 128):
        bm = s[..., j0:j0 + 128].max(-1)
        moved.append(bm > run)
        run = np.maximum(run, bm)
    assert float(np.mean(moved)) > 0.9
    o_ref, lse_ref, bar = _ref_and_bar(x)
    o, lse = _run(x, cuda_device, out_f32=True)
    print("fp32 out", _check(o.reshape(-1, 128), lse.reshape(-1), o_ref, lse_ref, bar, False))
    o, lse = _run(x, cuda_device)
    print("bf16 out", _check(o.reshape(-1, 128), lse.reshape(-1), o_ref, lse_ref, bar, True))


def test_fp8_full_size_sampled_rows(cuda_device):
    """The FP8 benchmark workload (causal GQA, n = 16384) in its launch configuration:
    every row of query heads 0 and 31 in their first 512 and last 256 positions, plus
    sampled rows, against the oracle at the derived bar; bf16 and fp32 output."""
    sh = inputs.FP8_WORKLOADS["fp8_causal_gqa_h32_kv8_n16384_d128"]
    x = inputs.make_fwd_inputs(sh)
    o, lse = _run(x, cuda_device)
    o32, lse32 = _run(x, cuda_device, out_f32=True)
    assert np.all(np.isfinite(o))
    rng = np.random.default_rng(5)
    n = sh.n_q
    rows = np.unique(np.concatenate([np.arange(512), np.arange(n - 256, n),
                                     np.arange(31 * n, 31 * n + 512), np.arange(32 * n - 256, 32 * n),
                                     rng.choice(sh.H * n, size=128, replace=False)]))
    o_ref, lse_ref, bar = _ref_and_bar(x, rows)
    print("bf16 out", _check(o.reshape(-1, sh.d)[rows], lse.reshape(-1)[rows], o_ref, lse_ref, bar, True))
    print("fp32 out", _check(o32.reshape(-1, sh.d)[rows], lse32.reshape(-1)[rows], o_ref, lse_ref, bar, False))
