"""Parity of the FP8 E4M3 forward (tcgen05 kind::f8f6f4) with the float64 oracle on
the decoded inputs.

Tolerance (derived; the pages fix none for FP8): the inputs are exact (the oracle
uses the same decoded values), fp32 accumulates, and P is rounded to E4M3 with a
relative error |e_j| <= 2^-4 per weight.  With O normalised by the sum of the
rounded weights, O_gpu - O = sum_j w_j (e_j - e_mean) (v_j - O) / (1 + e_mean), so
|dO| <= 2^-3 / (1 - 2^-4) * max_j |v_j - O| <= 0.134 * (max|v| + max|O|) per
element (weights below E4M3's subnormal range are rounded to 0; they carry less
than 2^-17 of the row's largest weight each).  On top comes half a bf16 ulp for a
bf16 output.  The LSE comes from the unrounded weights: the bf16 bound 1e-3
relative.  The mean error is also checked (random data: the errors of many
weights average out), which catches a systematic fault the loose bound would not.
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
    d = x["descale"]
    km = x["key_mask"].to(dev) if x.get("key_mask") is not None else None
    o, lse = attn.attn_fwd_fp8(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), d["q"], d["k"], d["v"], x["scale"],
                               x["causal"], km, out_f32=out_f32)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _ref(x):
    d = x["descale"]
    return oracle.attn_fwd_fp8(x["q"], x["k"], x["v"], d["q"], d["k"], d["v"], x["scale"], x["causal"],
                               x.get("key_mask"))


def _check(o, lse, o_ref, lse_ref, x, bf16_out):
    vmax = float(np.max(np.abs(oracle.e4m3_to_f64(x["v"]) * x["descale"]["v"])))
    bound = 0.134 * (vmax + np.abs(o_ref)) + (half_ulp_bf16(o_ref) if bf16_out else 0.0)
    err = np.abs(o - o_ref)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(err <= bound), float(np.max(err - bound))
    fin = ~empty
    assert float(np.mean(err[fin])) <= 5e-3, float(np.mean(err[fin]))
    d = np.abs(lse[fin] - lse_ref[fin])
    assert np.all(d <= 1e-3 * np.maximum(np.abs(lse_ref[fin]), 1.0)), float(np.max(d))
    return float(np.max(err)), float(np.mean(err[fin]))


CASES = {
    "causal_gqa_n777": inputs.FwdShape(1, 4, 2, 777, 777, 128, "fp8", True, seed_index=31),
    "noncausal_b2_n300_nkv1000": inputs.FwdShape(2, 2, 2, 300, 1000, 128, "fp8", False, seed_index=32),
    "keymask_b2_n600_qstd4": inputs.FwdShape(2, 2, 1, 600, 600, 128, "fp8", False, q_std=4.0, prefix_mask=True,
                                             seed_index=33),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_forward_matches_oracle(name, cuda_device):
    x = inputs.make_fwd_inputs(CASES[name])
    o_ref, lse_ref = _ref(x)
    o, lse = _run(x, cuda_device, out_f32=True)
    print(name, "fp32 out", _check(o, lse, o_ref, lse_ref, x, False))
    o, lse = _run(x, cuda_device)
    print(name, "bf16 out", _check(o, lse, o_ref, lse_ref, x, True))


def test_fp8_one_kept_key_gives_its_value(cuda_device):
    """Causal row 0 keeps one key: its weight is the only one, so O is that value row,
    exactly (times v_descale, then rounded to bf16)."""
    x = inputs.make_fwd_inputs(CASES["causal_gqa_n777"])
    o, lse = _run(x, cuda_device, out_f32=True)
    v0 = oracle.e4m3_to_f64(x["v"])[0, :, 0, :] * x["descale"]["v"]          # [H_kv, d]
    G = 2
    for h in range(4):
        assert np.allclose(o[0, h, 0], v0[h // G], rtol=1e-6, atol=0)


def test_fp8_deterministic(cuda_device):
    x = inputs.make_fwd_inputs(CASES["causal_gqa_n777"])
    a = _run(x, cuda_device)
    b = _run(x, cuda_device)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp8_full_size_sampled_rows(cuda_device):
    """The FP8 benchmark workload (causal GQA, n = 16384) in its launch configuration;
    sampled rows against the oracle."""
    sh = inputs.FP8_WORKLOADS["fp8_causal_gqa_h32_kv8_n16384_d128"]
    x = inputs.make_fwd_inputs(sh)
    o, lse = _run(x, cuda_device)
    assert np.all(np.isfinite(o))
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(sh.H * sh.n_q, size=96, replace=False))
    d = x["descale"]
    o_ref, lse_ref = oracle.attn_fwd_fp8(x["q"], x["k"], x["v"], d["q"], d["k"], d["v"], x["scale"], True,
                                         rows=rows)
    h, i = rows // sh.n_q, rows % sh.n_q
    _check(o[0][h, i], lse[0][h, i], o_ref, lse_ref, x, True)
