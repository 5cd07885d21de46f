"""Float64 gradients of exact attention (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline and
reference legs may import this module.  It shares no code with the CUDA library.

What it computes
----------------
The chat page ("Sviluppo AI ed Algebra Lineare", section "Ricalcolo nel Backward Pass
(Recomputation)") states the backward pass's contract: only the row statistics
of the forward pass are kept, and the score and weight blocks are recomputed
from Q, K and V.  It prints no gradient formulas.  This module therefore takes
the plain reading: the gradients of L = sum(dO * O) with respect to Q, K and V,
where O is the forward definition of ``oracle.attn_rows`` (kept keys only, GQA
head g = h // (H / H_kv), bottom-right causal alignment).  The chain rule gives,
for one query head and the keys its row keeps:

    s_ij  = scale * q_i . k_j            (excluded keys: no entry)
    P_ij  = softmax_j(s_ij)
    dV_j += sum_i P_ij dO_i
    dP_ij = dO_i . v_j
    dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)
    dQ_i  = scale * sum_j dS_ij k_j
    dK_j += scale * sum_i dS_ij q_i

summed over the query heads of each kv head for dK and dV.  A row that keeps no
key has no weights: it adds nothing to any gradient and its dQ row is 0.

Everything is materialised per (batch, head) in float64 from the exact values of
the inputs (bf16 widened exactly).  ``tests/test_oracle_bwd.py`` pins it to
central finite differences of the forward oracle, closed forms, invariants and
torch's float64 CPU autograd.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    import torch

    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _keep_rows(i0, i1, n_q, n_kv, causal, mask_row):
    """[i1 - i0, n_kv] bool: key j is kept for query row i (rows i0..i1-1)."""
    keep = np.ones((i1 - i0, n_kv), dtype=bool)
    if causal:
        i = np.arange(i0, i1)[:, None]
        j = np.arange(n_kv)[None, :]
        keep &= j <= i + (n_kv - n_q)
    if mask_row is not None:
        keep &= (mask_row != 0)[None, :]
    return keep


def _keep(n_q, n_kv, causal, mask_row):
    """[n_q, n_kv] bool: key j is kept for query row i."""
    return _keep_rows(0, n_q, n_q, n_kv, causal, mask_row)


def _weights(s, keep):
    """Row softmax over the kept entries; rows with no kept entry are all 0."""
    s = np.where(keep, s, -np.inf)
    mu = s.max(axis=1, keepdims=True)
    has = np.isfinite(mu)
    w = np.where(keep, np.exp(s - np.where(has, mu, 0.0)), 0.0)
    l = w.sum(axis=1, keepdims=True)
    return np.where(has, w / np.where(has, l, 1.0), 0.0)


def attn_bwd(q, k, v, do, scale, causal=False, key_mask=None, with_scale=False):
    """Gradients (dq [B, H, n_q, d], dk, dv [B, H_kv, n_kv, d]) in float64.

    q, do: [B, H, n_q, d]; k, v: [B, H_kv, n_kv, d]; key_mask: [B, n_kv]
    (nonzero = keep) or None.  With ``with_scale`` it also returns the error
    scales of ``error_scales`` (a dict) computed from the same weights.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    mask = None if key_mask is None else np.asarray(_f64(key_mask))
    B, H, n_q, d = q.shape
    H_kv, n_kv = k.shape[1], k.shape[2]
    group = H // H_kv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    sc = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v)} if with_scale else None
    for b in range(B):
        keep = _keep(n_q, n_kv, causal, None if mask is None else mask[b])
        for h in range(H):
            g = h // group
            p = _weights(scale * q[b, h] @ k[b, g].T, keep)
            dp = do[b, h] @ v[b, g].T
            row = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - row)
            dq[b, h] = scale * ds @ k[b, g]
            dk[b, g] += scale * ds.T @ q[b, h]
            dv[b, g] += p.T @ do[b, h]
            if with_scale:
                o = p @ v[b, g]
                _accumulate_scales(sc, b, h, g, p, dp, row, o, q[b, h], k[b, g], do[b, h], scale)
    if with_scale:
        return dq, dk, dv, sc
    return dq, dk, dv


def _accumulate_scales(sc, b, h, g, p, dp, row, o, qh, kg, doh, scale):
    # Size of each gradient element's terms, with every factor replaced by its
    # magnitude: a relative error e in each weight, each dS entry and each O element
    # moves the element by at most e times this.
    dD = (np.abs(doh) * np.abs(o)).sum(axis=1, keepdims=True)   # |dO_i| . |O_i|
    e_ds = p * (np.abs(dp) + np.abs(row) + dD)
    sc["dv"][b, g] += p.T @ np.abs(doh)
    sc["dk"][b, g] += scale * e_ds.T @ np.abs(qh)
    sc["dq"][b, h] = scale * e_ds @ np.abs(kg)


def error_scales(q, k, v, do, scale, causal=False, key_mask=None):
    """Magnitude sums that bound how far rounding can move each gradient element.

    dv: sum_i P_ij |dO_i|; dk: scale * sum_i e_ij |q_i|; dq: scale * sum_j e_ij |k_j|,
    with e_ij = P_ij (|dP_ij| + |sum_k P_ik dP_ik| + |dO_i| . |O_i|).  A computation
    whose weights, dS entries and O inputs each carry relative error at most r is
    within r times these of the exact gradients (up to fp32 accumulation).
    """
    return attn_bwd(q, k, v, do, scale, causal, key_mask, with_scale=True)[3]


def group_forward(q, k, v, scale, causal, key_mask, b, g, group, row_chunk=1024):
    """Float64 O [group, n_q, d] and LSE [group, n_q] of the query heads of kv head g
    in batch row b, computed in row chunks so that full-length rows fit in memory."""
    q, k, v = _f64(q[b, g * group:(g + 1) * group]), _f64(k[b, g]), _f64(v[b, g])
    mask_row = None if key_mask is None else np.asarray(_f64(key_mask[b]))
    n_q, d = q.shape[1], q.shape[2]
    n_kv = k.shape[0]
    o = np.zeros((group, n_q, d))
    lse = np.full((group, n_q), -np.inf)
    for i0 in range(0, n_q, row_chunk):
        i1 = min(n_q, i0 + row_chunk)
        keep = _keep_rows(i0, i1, n_q, n_kv, causal, mask_row)
        for t in range(group):
            s = np.where(keep, scale * q[t, i0:i1] @ k.T, -np.inf)
            mu = s.max(axis=1, keepdims=True)
            has = np.isfinite(mu)[:, 0]
            w = np.where(keep, np.exp(s - np.where(has[:, None], mu, 0.0)), 0.0)
            l = w.sum(axis=1)
            o[t, i0:i1][has] = (w[has] @ v) / l[has][:, None]
            lse[t, i0:i1][has] = mu[has, 0] + np.log(l[has])
    return o, lse


def group_bwd_sampled(q, k, v, do, o, lse, scale, causal, key_mask, b, g, group, key_rows, query_rows,
                      row_chunk=1024, with_scale=False):
    """Gradients of one kv head's group at full length, on samples.

    o, lse: the group's float64 forward (``group_forward``), used for the weights
    P_ij = exp(s_ij - LSE_i) and the row terms sum_k P_ik dP_ik = dO_i . O_i, which
    equal the definition's.  Returns (dk [len(key_rows), d], dv [len(key_rows), d],
    dq [group, len(query_rows), d]); with ``with_scale`` also the error scales of
    ``error_scales`` for the same elements, as a dict with keys dk, dv, dq.
    """
    qg, kg, vg, dog = (_f64(x) for x in (q[b, g * group:(g + 1) * group], k[b, g], v[b, g],
                                          do[b, g * group:(g + 1) * group]))
    mask_row = None if key_mask is None else np.asarray(_f64(key_mask[b]))
    n_q, d = qg.shape[1], qg.shape[2]
    n_kv = kg.shape[0]
    key_rows = np.asarray(key_rows)
    query_rows = np.asarray(query_rows)
    row = (dog * o).sum(axis=2)                                       # [group, n_q]
    d_mag = (np.abs(dog) * np.abs(o)).sum(axis=2)                     # |dO_i| . |O_i|
    dk = np.zeros((key_rows.size, d))
    dv = np.zeros((key_rows.size, d))
    sc = {"dk": np.zeros_like(dk), "dv": np.zeros_like(dv)} if with_scale else None
    for i0 in range(0, n_q, row_chunk):
        i1 = min(n_q, i0 + row_chunk)
        keep = _keep_rows(i0, i1, n_q, n_kv, causal, mask_row)[:, key_rows]
        for t in range(group):
            s = scale * qg[t, i0:i1] @ kg[key_rows].T
            lt = lse[t, i0:i1][:, None]
            p = np.where(keep & np.isfinite(lt), np.exp(s - np.where(np.isfinite(lt), lt, 0.0)), 0.0)
            dp = dog[t, i0:i1] @ vg[key_rows].T
            ds = p * (dp - row[t, i0:i1][:, None])
            dk += scale * ds.T @ qg[t, i0:i1]
            dv += p.T @ dog[t, i0:i1]
            if with_scale:
                e_ds = p * (np.abs(dp) + np.abs(row[t, i0:i1])[:, None] + d_mag[t, i0:i1][:, None])
                sc["dk"] += scale * e_ds.T @ np.abs(qg[t, i0:i1])
                sc["dv"] += p.T @ np.abs(dog[t, i0:i1])
    dq = np.zeros((group, query_rows.size, d))
    if with_scale:
        sc["dq"] = np.zeros_like(dq)
    keep_q = np.stack([_keep_rows(i, i + 1, n_q, n_kv, causal, mask_row)[0] for i in query_rows])
    for t in range(group):
        s = scale * qg[t, query_rows] @ kg.T
        lt = lse[t, query_rows][:, None]
        p = np.where(keep_q & np.isfinite(lt), np.exp(s - np.where(np.isfinite(lt), lt, 0.0)), 0.0)
        dp = dog[t, query_rows] @ vg.T
        ds = p * (dp - row[t, query_rows][:, None])
        dq[t] = scale * ds @ kg
        if with_scale:
            e_ds = p * (np.abs(dp) + np.abs(row[t, query_rows])[:, None] + d_mag[t, query_rows][:, None])
            sc["dq"][t] = scale * e_ds @ np.abs(kg)
    if with_scale:
        return dk, dv, dq, sc
    return dk, dv, dq
