"""Pins of the float64 backward oracle (``oracle.backward``), independent of it.

* central finite differences of the forward oracle (C, itself pinned to the
  pages' worked example, brute force and torch): every element of dQ, dK and
  dV on tiny shapes, causal, masked, GQA and n_q != n_kv;
* closed forms: one kept key (dQ = dK = 0, dV = dO), zero queries (uniform
  weights, covariance form), a fully masked row (no contribution);
* invariants at moderate size: every dS row sums to 0, so the keys' dK sum to
  0; every weight row sums to 1, so the keys' dV sum to the rows' dO;
* torch's float64 CPU autograd of scaled_dot_product_attention;
* the sampled full-length routine against the dense one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * std).numpy()


def _loss(q, k, v, do, scale, causal, mask):
    o, _ = oracle.attn_fwd(q, k, v, scale, causal, mask)
    return float((o * do).sum())


def _finite_diff(q, k, v, do, scale, causal, mask, eps=1e-6):
    grads = []
    for which in range(3):
        x = (q, k, v)[which]
        gx = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp = x.copy()
            xm = x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which] = xp
            args_m[which] = xm
            gx[idx] = (_loss(*args_p, do, scale, causal, mask) - _loss(*args_m, do, scale, causal, mask)) / (2 * eps)
        grads.append(gx)
    return grads


@pytest.mark.parametrize("B,H,H_kv,n_q,n_kv,d,causal,masked", [
    (1, 2, 1, 4, 4, 3, False, False),
    (1, 2, 2, 5, 5, 2, True, False),
    (2, 4, 2, 3, 5, 2, True, True),
    (1, 3, 1, 5, 3, 2, False, True),
    (1, 2, 1, 6, 4, 3, True, False),   # n_q > n_kv: the first rows keep no key
])
def test_finite_differences(B, H, H_kv, n_q, n_kv, d, causal, masked):
    seed = 100 + B * 7 + H * 3 + n_q * 11 + n_kv
    q = _rand((B, H, n_q, d), seed)
    k = _rand((B, H_kv, n_kv, d), seed + 1)
    v = _rand((B, H_kv, n_kv, d), seed + 2)
    do = _rand((B, H, n_q, d), seed + 3)
    mask = None
    if masked:
        mask = np.ones((B, n_kv), dtype=np.uint8)
        mask[0, 1] = 0
        if B > 1:
            mask[1, -1] = 0
    scale = 0.7
    dq, dk, dv = bwd.attn_bwd(q, k, v, do, scale, causal, mask)
    fq, fk, fv = _finite_diff(q, k, v, do, scale, causal, mask)
    for got, want in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-7)


def test_one_kept_key():
    # each row keeps exactly one key (causal, n_q = n_kv = 1 per batch row is too
    # small; use a key mask with one kept key)
    B, H, H_kv, n, d = 2, 4, 2, 6, 5
    q, k, v, do = _rand((B, H, n, d), 1), _rand((B, H_kv, n, d), 2), _rand((B, H_kv, n, d), 3), _rand((B, H, n, d), 4)
    mask = np.zeros((B, n), dtype=np.uint8)
    mask[0, 2] = 1
    mask[1, 5] = 1
    dq, dk, dv = bwd.attn_bwd(q, k, v, do, 0.5, False, mask)
    assert np.all(dq == 0) and np.all(dk == 0)
    for b, j in ((0, 2), (1, 5)):
        for g in range(H_kv):
            want = do[b, 2 * g:2 * g + 2].sum(axis=(0, 1))
            np.testing.assert_allclose(dv[b, g, j], want, rtol=1e-14, atol=1e-14)
        others = [i for i in range(n) if i != j]
        assert np.all(dv[b, :, others] == 0)


def test_zero_queries_uniform_weights():
    # q = 0: every kept key has weight 1/n, so
    #   dV_j = (1/n) sum_i dO_i,
    #   dQ_i = (scale/n) sum_j (dO_i . (v_j - vbar)) k_j   (covariance of the values and keys),
    #   dK_j = (scale/n) sum_i (dO_i . (v_j - vbar)) q_i = 0.
    B, H, n, d = 1, 2, 7, 4
    q = np.zeros((B, H, n, d))
    k, v, do = _rand((B, H, n, d), 11), _rand((B, H, n, d), 12), _rand((B, H, n, d), 13)
    scale = 1.3
    dq, dk, dv = bwd.attn_bwd(q, k, v, do, scale)
    for h in range(H):
        vbar = v[0, h].mean(axis=0)
        cov = (v[0, h] - vbar).T @ k[0, h] / n          # [d_v, d_k]
        np.testing.assert_allclose(dq[0, h], scale * do[0, h] @ cov, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dv[0, h], np.tile(do[0, h].sum(axis=0) / n, (n, 1)), rtol=1e-12, atol=1e-13)
    assert np.abs(dk).max() < 1e-14


def test_fully_masked_row_adds_nothing():
    B, H, n, d = 1, 1, 5, 3
    q, k, v, do = _rand((B, H, n, d), 21), _rand((B, H, n, d), 22), _rand((B, H, n, d), 23), _rand((B, H, n, d), 24)
    mask = np.zeros((B, n), dtype=np.uint8)
    dq, dk, dv = bwd.attn_bwd(q, k, v, do, 0.5, False, mask)
    assert np.all(dq == 0) and np.all(dk == 0) and np.all(dv == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_invariants(causal):
    B, H, H_kv, n, d = 2, 4, 2, 40, 16
    q, k, v, do = _rand((B, H, n, d), 31, 2.0), _rand((B, H_kv, n, d), 32), _rand((B, H_kv, n, d), 33), \
        _rand((B, H, n, d), 34)
    mask = np.ones((B, n), dtype=np.uint8)
    mask[1, 30:] = 0
    dq, dk, dv = bwd.attn_bwd(q, k, v, do, 1 / math.sqrt(d), causal, mask)
    assert np.abs(dk.sum(axis=2)).max() < 1e-12 * max(1.0, np.abs(dk).max()) * n
    for b in range(B):
        for g in range(H_kv):
            want = do[b, 2 * g:2 * g + 2].sum(axis=(0, 1))
            np.testing.assert_allclose(dv[b, g].sum(axis=0), want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal,masked,n_q,n_kv", [(False, False, 33, 33), (True, False, 29, 29),
                                                   (True, True, 17, 40), (False, True, 40, 17)])
def test_torch_autograd(causal, masked, n_q, n_kv):
    B, H, H_kv, d = 2, 6, 2, 8
    q = torch.from_numpy(_rand((B, H, n_q, d), 41)).requires_grad_()
    k = torch.from_numpy(_rand((B, H_kv, n_kv, d), 42)).requires_grad_()
    v = torch.from_numpy(_rand((B, H_kv, n_kv, d), 43)).requires_grad_()
    do = torch.from_numpy(_rand((B, H, n_q, d), 44))
    scale = 0.4
    keep = torch.ones(n_q, n_kv, dtype=torch.bool)
    if causal:
        keep = torch.ones(n_q, n_kv, dtype=torch.bool).tril(n_kv - n_q)
    keep = keep.expand(B, 1, n_q, n_kv).clone()
    mask = None
    if masked:
        mask = np.ones((B, n_kv), dtype=np.uint8)
        mask[0, 3] = 0
        mask[1, : n_kv // 3] = 0
        keep &= torch.from_numpy(mask != 0)[:, None, None, :]
    # keep only rows that keep at least one key (torch gives NaN for empty rows)
    rows_ok = keep.any(dim=-1)
    assert bool(rows_ok.all())
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=scale, enable_gqa=True)
    o.backward(do)
    dq, dk, dv = bwd.attn_bwd(q.detach(), k.detach(), v.detach(), do, scale, causal, mask)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_matches_dense(causal):
    B, H, H_kv, n, d = 2, 4, 2, 300, 16
    q, k, v, do = _rand((B, H, n, d), 51), _rand((B, H_kv, n, d), 52), _rand((B, H_kv, n, d), 53), \
        _rand((B, H, n, d), 54)
    mask = np.ones((B, n), dtype=np.uint8)
    mask[1, 250:] = 0
    scale = 0.25
    dq, dk, dv, sc = bwd.attn_bwd(q, k, v, do, scale, causal, mask, with_scale=True)
    keys = np.array([0, 1, 77, 128, 249, 299])
    rows = np.array([0, 5, 150, 299])
    for b, g in ((0, 1), (1, 0)):
        o, lse = bwd.group_forward(q, k, v, scale, causal, mask, b, g, 2, row_chunk=64)
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, mask)
        np.testing.assert_allclose(o, o_ref[b, 2 * g:2 * g + 2], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, lse_ref[b, 2 * g:2 * g + 2], rtol=1e-12, atol=1e-13)
        sk, sv, sq, ss = bwd.group_bwd_sampled(q, k, v, do, o, lse, scale, causal, mask, b, g, 2, keys, rows,
                                               row_chunk=64, with_scale=True)
        np.testing.assert_allclose(sk, dk[b, g, keys], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sv, dv[b, g, keys], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sq, dq[b, 2 * g:2 * g + 2][:, rows], rtol=1e-10, atol=1e-12)
        # the sampled error scales are the dense ones (themselves pinned above and below)
        np.testing.assert_allclose(ss["dk"], sc["dk"][b, g, keys], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(ss["dv"], sc["dv"][b, g, keys], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(ss["dq"], sc["dq"][b, 2 * g:2 * g + 2][:, rows], rtol=1e-10, atol=1e-12)


def test_error_scales_bound_a_perturbed_computation():
    # Perturb every weight and dS entry by a relative 2^-9 (random sign), as bf16
    # rounding of the MMA operands would: the gradients must move by at most
    # 2^-9 times the error scales.
    B, H, n, d = 1, 2, 50, 8
    q, k, v, do = _rand((B, H, n, d), 61, 2.0), _rand((B, H, n, d), 62), _rand((B, H, n, d), 63), \
        _rand((B, H, n, d), 64)
    scale = 1 / math.sqrt(d)
    dq, dk, dv, sc = bwd.attn_bwd(q, k, v, do, scale, True, None, with_scale=True)
    rng = np.random.default_rng(65)
    r = 2.0 ** -9
    keep = bwd._keep(n, n, True, None)
    for h in range(H):
        p = bwd._weights(scale * q[0, h] @ k[0, h].T, keep)
        dp = do[0, h] @ v[0, h].T
        row = (p * dp).sum(axis=1, keepdims=True)
        p_r = p * (1 + r * rng.choice([-1.0, 1.0], p.shape))
        ds_r = (p * (dp - row)) * (1 + r * rng.choice([-1.0, 1.0], p.shape))
        # plus float64 rounding of the two products compared (summed in different orders by a
        # multithreaded BLAS): 1e-12 of the magnitudes involved
        for got, ref, mag in ((p_r.T @ do[0, h], dv[0, h], sc["dv"][0, h]),
                              (scale * ds_r @ k[0, h], dq[0, h], sc["dq"][0, h]),
                              (scale * ds_r.T @ q[0, h], dk[0, h], sc["dk"][0, h])):
            np.testing.assert_array_less(np.abs(got - ref), r * mag + 1e-12 * (np.abs(ref) + mag) + 1e-15)


def _perturbed_grads(q, k, do, p, dp, o, scale, r, s_p, s_o, s_ds):
    """Gradients of one head from weights, O and dS that each carry a relative error r
    with the given signs (the model the error scales describe): P' = P (1 + r s_p),
    row' = dO . (O (1 + r s_o)), dS' = P' (dP - row') (1 + r s_ds)."""
    p_r = p * (1 + r * s_p)
    row_r = (do * (o * (1 + r * s_o))).sum(axis=1, keepdims=True)
    ds_r = p_r * (dp - row_r) * (1 + r * s_ds)
    return scale * ds_r @ k, scale * ds_r.T @ q, p_r.T @ do


def test_error_scales_are_attained_in_closed_form():
    """Upper pin of the error scales: one query row and two keys, built so that the
    row term sum_k P_k dP_k is exactly 0 (dO = e0, v1 = p2 e0, v2 = -p1 e0).  Then a
    relative error r in each weight, signed like dP_j times the sign of the multiplier,
    and an error r in each O element, signed against it, move each gradient element
    by r times its error scale (up to second-order terms), so a scale that is too large
    by any factor, or that drops a term, fails one of the equalities below."""
    scale, r = 0.5, 2.0 ** -20
    q = np.array([[0.7, -1.3]])                       # one query row, d = 2
    k = np.array([[1.1, 0.4], [0.3, 0.9]])            # same sign in every column
    s = scale * q @ k.T
    p = np.exp(s - s.max())
    p /= p.sum()
    v = np.array([[p[0, 1], 0.0], [-p[0, 0], 0.0]])
    do = np.array([[1.0, 0.0]])
    o = p @ v
    dp = do @ v.T
    assert abs(float((p * dp).sum())) < 1e-15         # the row term vanishes
    Q, K, V, DO = (x[None, None] for x in (q, k, v, do))
    dq, dk, dv, sc = bwd.attn_bwd(Q, K, V, DO, scale, False, None, with_scale=True)
    dq, dk, dv = dq[0, 0], dk[0, 0], dv[0, 0]
    # dq[0, c]: weight errors signed sign(dP_j) sign(k_jc) (the same for both keys),
    # the row term moved against that sign through O
    for c in range(2):
        sg = np.sign(k[:, c])
        assert sg[0] == sg[1]
        s_p = np.sign(dp) * sg[None, :]
        s_o = -sg[0] * np.sign(do * o)
        got_q, _, _ = _perturbed_grads(q, k, do, p, dp, o, scale, r, s_p, s_o, np.zeros_like(p))
        ratio = abs(got_q[0, c] - dq[0, c]) / (r * sc["dq"][0, 0, 0, c])
        assert 0.99 <= ratio <= 1.0 + 1e-6, ("dq", c, ratio)
    # dk[j, c]: one query row, so signs by sign(q_c)
    for c in range(2):
        sq = np.sign(q[0, c])
        s_p = np.sign(dp) * sq
        s_o = -sq * np.sign(do * o)
        _, got_k, _ = _perturbed_grads(q, k, do, p, dp, o, scale, r, s_p, s_o, np.zeros_like(p))
        for j in range(2):
            ratio = abs(got_k[j, c] - dk[j, c]) / (r * sc["dk"][0, 0, j, c])
            assert 0.99 <= ratio <= 1.0 + 1e-6, ("dk", j, c, ratio)
    # dv[j, 0]: weight errors signed like dO (only the weights enter dV)
    s_p = np.ones_like(p) * np.sign(do[0, 0])
    _, _, got_v = _perturbed_grads(q, k, do, p, dp, o, scale, r, s_p, np.zeros_like(o), np.zeros_like(p))
    for j in range(2):
        ratio = abs(got_v[j, 0] - dv[j, 0]) / (r * sc["dv"][0, 0, j, 0])
        assert 0.99 <= ratio <= 1.0 + 1e-6, ("dv", j, ratio)


def test_error_scales_are_reached_by_random_perturbations():
    """The worst element of random-sign perturbations (weights, O and dS each off by a
    relative 2^-9) reaches a sizeable fraction of the error scale: above 0.3 for each
    gradient.  A scale inflated by a factor 4 or more fails here; the bound itself (at
    most 2 for this model, where the weight and dS errors compound) is checked too."""
    B, H, n, d = 1, 2, 40, 8
    q, k, v, do = _rand((B, H, n, d), 71, 2.0), _rand((B, H, n, d), 72), _rand((B, H, n, d), 73), \
        _rand((B, H, n, d), 74)
    scale = 1 / math.sqrt(d)
    dq, dk, dv, sc = bwd.attn_bwd(q, k, v, do, scale, True, None, with_scale=True)
    rng = np.random.default_rng(75)
    r = 2.0 ** -9
    keep = bwd._keep(n, n, True, None)
    worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for h in range(H):
        p = bwd._weights(scale * q[0, h] @ k[0, h].T, keep)
        dp = do[0, h] @ v[0, h].T
        o = p @ v[0, h]
        for _ in range(20):
            s_p, s_ds = (rng.choice([-1.0, 1.0], p.shape) for _ in range(2))
            s_o = rng.choice([-1.0, 1.0], o.shape)
            got = _perturbed_grads(q[0, h], k[0, h], do[0, h], p, dp, o, scale, r, s_p, s_o, s_ds)
            for name, g, ref in zip(("dq", "dk", "dv"), got, (dq[0, h], dk[0, h], dv[0, h])):
                mag = sc[name][0, h]
                nz = mag > 0
                ratio = np.abs(g - ref)[nz] / (r * mag[nz])
                worst[name] = max(worst[name], float(ratio.max()))
    for name, w in worst.items():
        assert 0.3 <= w <= 2.0 + 1e-6, (name, w)


def test_error_scale_row_term_is_attained():
    """The row term |sum_k P_k dP_k| of the scales, which the closed form above leaves at 0:
    with dP_1 = 1 > 0 > row (dP_2 = -3 and P_2 large enough), key 1 has |dP_1 - row| =
    |dP_1| + |row|, and errors signed along dP_1 - row in its weight and against it in O
    move dk_1 by r times its scale.  A scale without the row term, or with it doubled,
    fails."""
    scale, r = 1.0, 2.0 ** -20
    q = np.array([[1.0, 0.5]])
    k = np.array([[0.2, -0.4], [0.9, 0.3]])
    s = scale * q @ k.T
    p = np.exp(s - s.max())
    p /= p.sum()
    v = np.array([[1.0, 0.0], [-3.0, 0.0]])
    do = np.array([[1.0, 0.0]])
    o = p @ v
    dp = do @ v.T
    row = float((p * dp).sum())
    assert dp[0, 0] > 0 > row and abs(row) > 0.5
    Q, K, V, DO = (x[None, None] for x in (q, k, v, do))
    _, dk, _, sc = bwd.attn_bwd(Q, K, V, DO, scale, False, None, with_scale=True)
    for c in range(2):
        sq = np.sign(q[0, c])
        s_p = np.sign(dp - row) * sq
        s_o = -sq * np.sign(do * o)
        _, got_k, _ = _perturbed_grads(q, k, do, p, dp, o, scale, r, s_p, s_o, np.zeros_like(p))
        ratio = abs(got_k[0, c] - dk[0, 0, 0, c]) / (r * sc["dk"][0, 0, 0, c])
        assert 0.99 <= ratio <= 1.0 + 1e-6, (c, ratio)
