"""Pins of the oracle's FP8 E4M3 path: the bit-pattern decoder and attention on
decoded inputs (the FP8 forward's reference; the method itself is the same
definition, "Sviluppo AI ed Algebra Lineare", FP8 section, with inputs stored in
E4M3 and one scale per tensor)."""
import numpy as np
import torch

import oracle
from online_softmax_12_b200 import inputs


def test_e4m3_decoder_matches_the_format_definition():
    bits = np.arange(256)
    got = oracle.e4m3_to_f64(bits)
    # the format's landmarks: zero, the smallest subnormal 2^-9, the largest subnormal
    # 7/8 * 2^-6, one, the largest finite 448 (0x7E), NaN at 0x7F and 0xFF, and the sign bit
    assert got[0x00] == 0.0 and got[0x80] == 0.0
    assert got[0x01] == 2.0 ** -9 and got[0x07] == 7 / 8 * 2.0 ** -6
    assert got[0x08] == 2.0 ** -6 and got[0x38] == 1.0
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert np.array_equal(got[0x81:0xFF], -got[0x01:0x7F])
    # ... and every pattern agrees with torch's float8_e4m3fn conversion
    ref = torch.tensor(bits, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_fp8_attention_is_the_definition_on_decoded_inputs():
    sh = inputs.FwdShape(1, 2, 1, 40, 56, 64, "fp8", True, seed_index=21)
    x = inputs.make_fwd_inputs(sh)
    d = x["descale"]
    o, lse = oracle.attn_fwd_fp8(x["q"], x["k"], x["v"], d["q"], d["k"], d["v"], x["scale"], True)
    q = torch.tensor(oracle.e4m3_to_f64(x["q"]) * d["q"])
    k = torch.tensor(oracle.e4m3_to_f64(x["k"]) * d["k"]).repeat_interleave(2, 1)
    v = torch.tensor(oracle.e4m3_to_f64(x["v"]) * d["v"]).repeat_interleave(2, 1)
    keep = torch.arange(56)[None, :] <= torch.arange(40)[:, None] + 16
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=x["scale"])
    assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    # quantisation kept the tensors' ranges: the largest magnitude sits at 448 * descale
    for n in ("q", "k", "v"):
        dec = oracle.e4m3_to_f64(x[n])
        assert np.all(np.isfinite(dec)) and np.max(np.abs(dec)) == 448.0
