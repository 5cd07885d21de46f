"""Pins of the oracle's FP8 E4M3 path: the bit-pattern decoder, the block-scaled
decode ("Sviluppo AI ed Algebra Lineare", FP8 section, "Quantizzazione a Blocchi e
Scaling Algebrico": each block X of rows is stored as X_fp8 = round(X / s_X) with
s_X = max|X| / 448, and X = s_X X_fp8), attention on decoded inputs, and the
per-element error bound of rounding the weights to E4M3 (the FP8 parity bar)."""
import math

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


def test_block_decode_is_value_times_its_blocks_scale():
    g = torch.Generator().manual_seed(3)
    bits = torch.randint(0, 0x7E, (2, 3, 300, 8), generator=g, dtype=torch.int32).to(torch.uint8)
    dec = torch.tensor(bits.numpy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()   # torch's decode
    s = np.full((2, 3, 3), 0.25)
    assert np.array_equal(oracle.decode_e4m3_blocks(bits, s), dec * 0.25)
    assert np.array_equal(oracle.decode_e4m3_blocks(bits, 0.25), dec * 0.25)       # a scalar: every block
    s2 = s.copy()
    s2[1, 2, 1] = 3.0                       # rows 128..255 of batch 1, head 2
    got = oracle.decode_e4m3_blocks(bits, s2)
    diff = got != dec * 0.25
    assert np.array_equal(np.argwhere(diff.any(axis=3))[:, :2], np.tile([1, 2], (diff.any(axis=3).sum(), 1)))
    assert diff[1, 2, 128:256].any() and not diff[1, 2, :128].any() and not diff[1, 2, 256:].any()
    assert np.array_equal(got[1, 2, 128:256], dec[1, 2, 128:256] * 3.0)


def test_block_quantiser_round_trip():
    """inputs.quantize_e4m3_blocks: each block's largest magnitude encodes as 448 exactly,
    and every element decodes within half an E4M3 ulp (2^-4 relative, 2^-10 * s below
    the normal range) of its fp32 value."""
    g = torch.Generator().manual_seed(4)
    x = torch.randn(2, 2, 300, 64, generator=g) * torch.tensor([1.0, 7.0])[None, :, None, None]
    x[0, 0, 128:256] = 0.0                  # an all-zero block keeps descale 1
    bits, s = inputs.quantize_e4m3_blocks(x)
    assert s.shape == (2, 2, 3) and float(s[0, 0, 1]) == 1.0
    dec = oracle.decode_e4m3_blocks(bits, s)
    xs = x.double().numpy()
    srow = np.repeat(s.double().numpy(), 128, axis=2)[:, :, :300, None]
    assert np.all(np.abs(dec - xs) <= 2.0 ** -4 * np.abs(xs) + 2.0 ** -10 * srow + 1e-300)
    for b in range(2):
        for h in range(2):
            for j in range(3):
                blk = dec[b, h, 128 * j:128 * (j + 1)]
                if float(s[b, h, j]) != 1.0 or np.any(blk):
                    assert np.max(np.abs(blk)) == 448.0 * float(s[b, h, j])


def test_fp8_attention_is_the_definition_on_decoded_inputs():
    sh = inputs.FwdShape(1, 2, 1, 140, 300, 64, "fp8", True, seed_index=21)
    x = inputs.make_fwd_inputs(sh)
    d = x["descale"]
    assert d["q"].shape == (1, 2, 2) and d["k"].shape == (1, 1, 3)
    o, lse = oracle.attn_fwd_fp8(x["q"], x["k"], x["v"], d["q"], d["k"], d["v"], x["scale"], True)
    q = torch.tensor(oracle.decode_e4m3_blocks(x["q"], d["q"]))
    k = torch.tensor(oracle.decode_e4m3_blocks(x["k"], d["k"])).repeat_interleave(2, 1)
    v = torch.tensor(oracle.decode_e4m3_blocks(x["v"], d["v"])).repeat_interleave(2, 1)
    keep = torch.arange(300)[None, :] <= torch.arange(140)[:, None] + 160
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=x["scale"])
    assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def _simulate_fp8_rounding(x, v, keep, ratio_of_key, block=128):
    """The FP8 weight-rounding model on one row, simulated with torch's E4M3 rounding: blocks
    in order, a running maximum m_j that follows every new maximum, weights 2^(8 + x - m_j)
    times the key's V-block ratio rounded to nearest E4M3, O and l rescaled when m_j moves,
    l summing the rounded weights divided back by their ratio."""
    m = -math.inf
    acc = np.zeros(v.shape[1])
    l = 0.0
    for j0 in range(0, x.size, block):
        sl = slice(j0, j0 + block)
        kk = keep[sl]
        if not kk.any():
            continue
        m_new = max(m, float(x[sl][kk].max()))
        if m != -math.inf:
            acc *= 2.0 ** (m - m_new)
            l *= 2.0 ** (m - m_new)
        m = m_new
        r = ratio_of_key[sl][kk]
        w = torch.tensor(2.0 ** (8.0 + x[sl][kk] - m) * r).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        acc += (w / r) @ v[sl][kk]
        l += float((w / r).sum())
    return acc / l


def test_fp8_bound_holds_for_simulated_rounding_and_is_attained():
    """The bound is never exceeded by the simulated rounding (random rows, several blocks,
    unequal V-block ratios, score ranges that reach E4M3's subnormals), one kept key gives 0,
    and a two-key row built on a rounding tie reaches more than 0.9 of it (so an inflated
    bound fails)."""
    rng = np.random.default_rng(8)
    B, H, n, d = 1, 2, 300, 16
    for spread_scale in (1.0, 6.0):
        q = rng.standard_normal((B, H, n, d)) * spread_scale
        k = rng.standard_normal((B, H, n, d))
        v = rng.standard_normal((B, H, n, d))
        sv = rng.uniform(0.3, 1.0, (B, H, 3))
        scale = 1 / math.sqrt(d)
        bound, spread = oracle.fp8_error_bound(q, k, v, sv, scale, True)
        o, _ = oracle.attn_fwd(q, k, v, scale, True)
        ratio = np.repeat(sv / sv.max(axis=2, keepdims=True), 128, axis=2)[:, :, :n]
        worst = 0.0
        for h in range(H):
            for i in range(0, n, 7):
                x = scale / math.log(2.0) * (k[0, h] @ q[0, h, i])
                keep = np.arange(n) <= i
                o_sim = _simulate_fp8_rounding(x, v[0, h], keep, ratio[0, h])
                r = h * n + i
                err = np.abs(o_sim - o[0, h, i])
                assert np.all(err <= bound[r] * (1 + 1e-9) + 1e-13), (h, i, float(np.max(err - bound[r])))
                worst = max(worst, float(np.max(err / np.maximum(bound[r], 1e-300))))
        assert worst > 0.2, worst
    # one kept key (causal row 0): O is that value exactly, the bound is 0
    assert np.all(bound[0] == 0) and np.all(spread[0] == 0)
    # a tie: the second key's weight is 136 = 17 * 2^3, halfway between E4M3's 128 and 144
    qq = np.zeros((1, 1, 1, 2))
    qq[0, 0, 0, 0] = 1.0
    kk = np.zeros((1, 1, 2, 2))
    kk[0, 0, 1, 0] = math.log(136.0 / 256.0)          # scores 0 and ln(136/256), scale 1
    vv = np.zeros((1, 1, 2, 2))
    vv[0, 0, 0, 0], vv[0, 0, 1, 0] = -1.0, 1.0
    b2, _ = oracle.fp8_error_bound(qq, kk, vv, np.ones((1, 1, 1)), 1.0, False)
    o2, _ = oracle.attn_fwd(qq, kk, vv, 1.0, False)
    x2 = np.array([0.0, math.log2(136.0 / 256.0)])
    o_sim = _simulate_fp8_rounding(x2, vv[0, 0], np.array([True, True]), np.ones(2))
    ratio2 = abs(o_sim[0] - o2[0, 0, 0, 0]) / b2[0, 0]
    assert 0.9 <= ratio2 <= 1.0 + 1e-9, ratio2


def test_fp8_bound_subnormal_floor_scales_with_the_v_block_ratio():
    """A weight stored in E4M3's subnormal range (spacing 2^-9) from a V block of ratio 1/2:
    its stored value 2.5 * 2^-9 is a tie and rounds to 2 * 2^-9, an error of 2^-10 in the
    stored weight and 2^-9 once divided back by the ratio.  The bound's subnormal term
    2^-10 / r_j is attained; without the division by the ratio it would be exceeded."""
    n = 129
    qq = np.zeros((1, 1, 1, 2))
    qq[0, 0, 0, 0] = 1.0
    kk = np.zeros((1, 1, n, 2))
    p2 = 5 * 2.0 ** -9                                     # final-frame weight of key 128
    kk[0, 0, 128, 0] = math.log(p2 / 256.0)                # scale 1: score ln(P2 / 2^8)
    vv = np.zeros((1, 1, n, 2))
    vv[0, 0, 128, 0] = 1.0
    mask = np.zeros((1, n), dtype=np.uint8)
    mask[0, [0, 128]] = 1
    sv = np.array([[[1.0, 0.5]]])
    b, _ = oracle.fp8_error_bound(qq, kk, vv, sv, 1.0, False, mask)
    o, _ = oracle.attn_fwd(qq, kk, vv, 1.0, False, mask)
    x = np.zeros(n)
    x[128] = math.log2(p2 / 256.0)
    ratio = np.array([1.0] * 128 + [0.5])
    o_sim = _simulate_fp8_rounding(x, vv[0, 0], mask[0] != 0, ratio)
    err = abs(o_sim[0] - o[0, 0, 0, 0])
    assert 0.95 * b[0, 0] <= err <= b[0, 0] * (1 + 1e-9), (err, b[0, 0])
