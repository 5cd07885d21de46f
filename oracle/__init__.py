"""Float64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline and reference legs may import anything here.  The
oracle shares no code with the CUDA library and never imports it; the only
module both sides use is the seeded input generator, which holds none of the
attention arithmetic.

Contents
--------
* ``attn_rows`` / ``attn_fwd``: the plain definition of scaled dot-product
  attention, row by row, in float64 (C, ``attn_oracle.c``): materialised score
  row, two-pass max-subtracted softmax, weighted sum of values, and the
  log-sum-exp of the scaled scores.
* ``decode_paged``: the same definition for one query token per sequence, with
  keys and values gathered through a block table of fixed-size pages.
* ``prefill_paged``: the same for a block of query tokens per sequence (the last
  positions of the sequence, causal or not) through the block table.
* ``attn_fwd_fp8``: the definition on FP8 E4M3 inputs (decoded from their bit
  patterns by ``e4m3_to_f64`` and multiplied by one descale per 128-row block,
  ``decode_e4m3_blocks``), and ``fp8_error_bound``, the per-element bound that
  rounding the weights to E4M3 allows (the FP8 parity bar).
* ``backward``: gradients dQ, dK, dV of the definition (chain rule, float64,
  numpy), the error scales the GPU tolerance is built from, and a sampled
  full-length routine for one kv head's group.
* ``streaming``: the scalar running (m, l, u) recurrence and the disjoint-block
  merge of "Attenzione: softmax online, riscalamento e memoria" (sections 2-4),
  used as an independent cross-check of the definition.

Every function here is pinned by ``tests/test_oracle_*.py`` against values the
pages print, closed forms, invariants, a pure-Python brute force and torch's
float64 CPU attention.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_DT = {"f64": 0, "f32": 1, "bf16": 2}
_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        c_void_p, c_int, c_double, c_int64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.oracle_attn_rows.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int, c_int, c_int,
                                         c_int, c_int, c_int, c_double, c_int, c_void_p, c_int64, c_void_p,
                                         c_void_p, c_int]
        lib.oracle_attn_rows.restype = c_int
        lib.oracle_decode_paged.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                            c_int, c_int, c_int, c_int, c_int, c_double, c_void_p, c_void_p, c_int]
        lib.oracle_decode_paged.restype = c_int
        lib.oracle_prefill_paged.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                             c_int, c_int, c_int, c_int, c_int, c_int, c_double, c_int, c_void_p,
                                             c_void_p, c_int]
        lib.oracle_prefill_paged.restype = c_int
        lib.oracle_default_threads.restype = c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _as_host_array(x):
    """Return (contiguous numpy array, dtype tag) without changing any value.

    bf16 tensors are passed as their raw 16-bit patterns; the C side widens
    them exactly to float64.
    """
    import torch

    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), "bf16"
        if x.dtype == torch.float32:
            return x.numpy(), "f32"
        if x.dtype == torch.float64:
            return x.numpy(), "f64"
        raise TypeError(f"unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, "f64"
    if x.dtype == np.float32:
        return x, "f32"
    raise TypeError(f"unsupported dtype {x.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


def attn_rows(q, k, v, scale, causal=False, key_mask=None, rows=None, threads=0):
    """Float64 attention for selected rows.

    q: [B, H, n_q, d]; k, v: [B, H_kv, n_kv, d] (torch or numpy; f64, f32 or bf16,
    all three the same dtype).  key_mask: [B, n_kv] (nonzero = keep) or None.
    rows: iterable of flat ids (b*H + h)*n_q + i, or None for every row.
    Returns (o [n_rows, d] float64, lse [n_rows] float64).
    """
    qa, tq = _as_host_array(q)
    ka, tk = _as_host_array(k)
    va, tv = _as_host_array(v)
    if not (tq == tk == tv):
        raise TypeError("q, k, v must share a dtype")
    B, H, n_q, d = qa.shape
    Bk, H_kv, n_kv, dk = ka.shape
    if Bk != B or dk != d or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    mask = None
    if key_mask is not None:
        mask = np.ascontiguousarray(np.asarray(key_mask.cpu() if hasattr(key_mask, "cpu") else key_mask)
                                    ).astype(np.uint8)
        if mask.shape != (B, n_kv):
            raise ValueError("key_mask must be [B, n_kv]")
    if rows is None:
        rows_a, n_rows = None, B * H * n_q
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows = rows_a.size
    o = np.empty((n_rows, d), dtype=np.float64)
    lse = np.empty((n_rows,), dtype=np.float64)
    rc = _load().oracle_attn_rows(_ptr(qa), _ptr(ka), _ptr(va), _DT[tq], _ptr(mask), B, H, H_kv, n_q, n_kv, d,
                                  float(scale), int(bool(causal)), _ptr(rows_a), n_rows, _ptr(o), _ptr(lse),
                                  int(threads))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows failed with {rc}")
    return o, lse


def attn_fwd(q, k, v, scale, causal=False, key_mask=None, threads=0):
    """All rows; returns (o [B, H, n_q, d], lse [B, H, n_q]) in float64."""
    B, H, n_q, d = tuple(q.shape)
    o, lse = attn_rows(q, k, v, scale, causal, key_mask, None, threads)
    return o.reshape(B, H, n_q, d), lse.reshape(B, H, n_q)


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale, threads=0):
    """Float64 one-token decode through a block table.

    q: [S, H, d]; k_pages, v_pages: [num_pages, page_size, H_kv, d];
    block_table: [S, max_pages] int32; seq_lens: [S] int32.
    Returns (o [S, H, d], lse [S, H]) in float64.
    """
    qa, tq = _as_host_array(q)
    ka, tk = _as_host_array(k_pages)
    va, tv = _as_host_array(v_pages)
    if not (tq == tk == tv):
        raise TypeError("dtype mismatch")
    S, H, d = qa.shape
    num_pages, page_size, H_kv, dk = ka.shape
    bt = np.ascontiguousarray(np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table,
                                         dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens, dtype=np.int32))
    if dk != d or bt.shape[0] != S or sl.shape != (S,):
        raise ValueError("shape mismatch")
    o = np.empty((S * H, d), dtype=np.float64)
    lse = np.empty((S * H,), dtype=np.float64)
    rc = _load().oracle_decode_paged(_ptr(qa), _ptr(ka), _ptr(va), _DT[tq], _ptr(bt), _ptr(sl), S, H, H_kv, d,
                                     page_size, bt.shape[1], num_pages, float(scale), _ptr(o), _ptr(lse),
                                     int(threads))
    if rc != 0:
        raise ValueError(f"oracle_decode_paged failed with {rc}")
    return o.reshape(S, H, d), lse.reshape(S, H)


def prefill_paged(q, k_pages, v_pages, block_table, seq_lens, scale, causal=True, threads=0):
    """Float64 attention of n_q query tokens per sequence (the last n_q positions)
    through a block table.

    q: [S, H, n_q, d]; k_pages, v_pages: [num_pages, page_size, H_kv, d];
    block_table: [S, max_pages] int32; seq_lens: [S] int32 (each >= 0).
    Returns (o [S, H, n_q, d], lse [S, H, n_q]) in float64.
    """
    qa, tq = _as_host_array(q)
    ka, tk = _as_host_array(k_pages)
    va, tv = _as_host_array(v_pages)
    if not (tq == tk == tv):
        raise TypeError("dtype mismatch")
    S, H, n_q, d = qa.shape
    num_pages, page_size, H_kv, dk = ka.shape
    bt = np.ascontiguousarray(np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table,
                                         dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens, dtype=np.int32))
    if dk != d or bt.shape[0] != S or sl.shape != (S,):
        raise ValueError("shape mismatch")
    o = np.empty((S * H * n_q, d), dtype=np.float64)
    lse = np.empty((S * H * n_q,), dtype=np.float64)
    rc = _load().oracle_prefill_paged(_ptr(qa), _ptr(ka), _ptr(va), _DT[tq], _ptr(bt), _ptr(sl), S, H, H_kv, n_q, d,
                                      page_size, bt.shape[1], num_pages, float(scale), int(bool(causal)), _ptr(o),
                                      _ptr(lse), int(threads))
    if rc != 0:
        raise ValueError(f"oracle_prefill_paged failed with {rc}")
    return o.reshape(S, H, n_q, d), lse.reshape(S, H, n_q)


def e4m3_to_f64(bits):
    """Decode FP8 E4M3 (the variant without infinities) from its bit patterns.

    Layout: sign (1 bit), exponent (4 bits, bias 7), mantissa (3 bits).  Exponent 0
    holds subnormals 2^-6 * m / 8; exponent 1..15 holds 2^(e - 7) * (1 + m / 8),
    except S.1111.111, which is NaN (the format's only special value)."""
    b = np.asarray(bits.cpu() if hasattr(bits, "cpu") else bits).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & ((b & 0x7) == 7), np.nan, mag)
    return sign * mag


def decode_e4m3_blocks(bits, descale, block=128):
    """Float64 values of a block-scaled E4M3 tensor: element (b, h, i, c) is
    e4m3_to_f64(bits[b, h, i, c]) * descale[b, h, i // block] ("Sviluppo AI ed Algebra
    Lineare", FP8 section, "Quantizzazione a Blocchi e Scaling Algebrico": a block X is
    stored as X_fp8 with its scale s_X, and X = s_X * X_fp8).  bits: [B, heads, n, d];
    descale: [B, heads, ceil(n / block)] (a scalar applies to every block)."""
    x = e4m3_to_f64(bits)
    s = np.asarray(descale.cpu() if hasattr(descale, "cpu") else descale, dtype=np.float64)
    if s.ndim == 0:
        return x * float(s)
    B, Hh, n, _ = x.shape
    if s.shape != (B, Hh, -(-n // block)):
        raise ValueError(f"descale shape {s.shape} does not match {x.shape} in blocks of {block}")
    return x * np.repeat(s, block, axis=2)[:, :, :n, None]


def attn_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal=False, key_mask=None, rows=None,
                 threads=0):
    """Attention on block-scaled FP8 E4M3 inputs: every element is its decoded value
    times its block's descale (``decode_e4m3_blocks``; q8 [B, H, n_q, d], k8/v8
    [B, H_kv, n_kv, d] as uint8 bit patterns, descales [B, heads, ceil(n / 128)]), then
    the float64 definition of attn_rows.  Returns (o, lse) as attn_rows does (all rows
    shaped like attn_fwd when rows is None)."""
    q = decode_e4m3_blocks(q8, q_descale)
    k = decode_e4m3_blocks(k8, k_descale)
    v = decode_e4m3_blocks(v8, v_descale)
    o, lse = attn_rows(q, k, v, scale, causal, key_mask, rows, threads)
    if rows is None:
        B, H, n_q, d = q.shape
        return o.reshape(B, H, n_q, d), lse.reshape(B, H, n_q)
    return o, lse


def fp8_error_bound(q, k, v, v_descale, scale, causal=False, key_mask=None, rows=None, block=128,
                    row_chunk=16):
    """Per-element bound on how far rounding the weights to E4M3 can move O, for the FP8
    forward's arithmetic (the parity bar of the FP8 path; the pages give no FP8 tolerance).

    q [B, H, n_q, d], k, v [B, H_kv, n_kv, d]: the decoded float64 inputs; v_descale
    [B, H_kv, ceil(n_kv / block)]: V's block descales.  The rounding model (the FP8
    forward's documented arithmetic): each kept key's weight is measured 2^8 above a
    running row maximum m_j <= m (m the row's final maximum, base 2 units), multiplied by
    its V block's ratio r_j = v_descale[j] / max_j' v_descale[j'] (<= 1) and rounded to
    nearest E4M3; O is normalised by the sum of the rounded weights (each divided back by
    r_j).  In the final frame the weight is P_k = 2^(8 + x_k - m) (x_k the scaled score in
    base 2), and its rounding error is at most E_k = max(2^-4 P_k, min(P_k, 2^-10 / r_j))
    (half an E4M3 ulp relative for normal values; at most the value itself and 2^-10
    absolute below 2^-6), except for a key that holds the row maximum in a V block of
    ratio 1: its weight is 2^8 in the frame where it became the maximum, exact in E4M3
    (E_k = 0).  Since O' - O = sum_k dP_k (v_k - O) / sum_k P'_k,

        |O'_c - O_c| <= sum_k E_k |v_kc - O_c| / (sum_k P_k - sum_k E_k).

    Returns (bound [n_rows, d], spread [n_rows, d]) with spread = sum_k P_k |v_kc - O_c| /
    sum_k P_k (the weights' mean absolute deviation of V); rows with no kept key give 0.
    rows: flat row ids (b * H + h) * n_q + i, or None for all.
    """
    qf = np.asarray(q, dtype=np.float64)
    kf = np.asarray(k, dtype=np.float64)
    vf = np.asarray(v, dtype=np.float64)
    B, H, n_q, d = qf.shape
    H_kv, n_kv = kf.shape[1], kf.shape[2]
    group = H // H_kv
    sv = np.asarray(v_descale.cpu() if hasattr(v_descale, "cpu") else v_descale, dtype=np.float64)
    ratio = sv / sv.max(axis=2, keepdims=True)                          # [B, H_kv, n_blocks]
    ratio_key = np.repeat(ratio, block, axis=2)[:, :, :n_kv]             # r_j of each key's block
    floor_abs = 2.0 ** -10 / ratio_key
    mask = None if key_mask is None else np.asarray(key_mask.cpu() if hasattr(key_mask, "cpu") else key_mask)
    all_rows = np.arange(B * H * n_q) if rows is None else np.asarray(rows, dtype=np.int64)
    bound = np.zeros((all_rows.size, d))
    spread = np.zeros((all_rows.size, d))
    log2e = 1.0 / np.log(2.0)
    plane = all_rows // n_q                                   # b * H + h of every row
    for bh in np.unique(plane):
        b, h = int(bh) // H, int(bh) % H
        g = h // group
        idx_all = np.nonzero(plane == bh)[0]
        for c0 in range(0, idx_all.size, row_chunk):
            idx = idx_all[c0:c0 + row_chunk]
            i = all_rows[idx] % n_q
            # keys past the chunk's last causally kept one carry no weight: leave them out
            kmax = n_kv if not causal else max(0, min(n_kv, int(i.max()) + n_kv - n_q + 1))
            if kmax == 0:
                continue
            kk, vv = kf[b, g, :kmax], vf[b, g, :kmax]                    # views [kmax, d]
            x = scale * log2e * (qf[b, h, i] @ kk.T)                      # [r, kmax]
            keep = np.ones_like(x, dtype=bool)
            if causal:
                keep &= np.arange(kmax)[None, :] <= (i + n_kv - n_q)[:, None]
            if mask is not None:
                keep &= (mask[b, :kmax] != 0)[None, :]
            has = keep.any(axis=1)
            m = np.where(has, np.where(keep, x, -np.inf).max(axis=1), 0.0)
            p = np.where(keep, np.exp2(8.0 + np.where(keep, x, 0.0) - m[:, None]), 0.0)
            exact = keep & (x == m[:, None]) & (ratio_key[b, g, :kmax] == 1.0)[None, :]
            e = np.where(keep & ~exact, np.maximum(2.0 ** -4 * p, np.minimum(p, floor_abs[b, g, :kmax][None, :])),
                         0.0)
            l = p.sum(axis=1)
            o = (p @ vv) / np.where(has, l, 1.0)[:, None]
            dev_ = np.abs(vv[None, :, :] - o[:, None, :])                  # [r, kmax, d]
            num_e = np.matmul(e[:, None, :], dev_)[:, 0, :]
            num_p = np.matmul(p[:, None, :], dev_)[:, 0, :]
            bound[idx] = np.where(has[:, None], num_e / np.where(has, l - e.sum(axis=1), 1.0)[:, None], 0.0)
            spread[idx] = np.where(has[:, None], num_p / np.where(has, l, 1.0)[:, None], 0.0)
    return bound, spread


__all__ = ["attn_rows", "attn_fwd", "attn_fwd_fp8", "e4m3_to_f64", "decode_e4m3_blocks", "decode_paged",
           "prefill_paged", "fp8_error_bound",
           "default_threads", "streaming", "backward"]

from . import backward, streaming  # noqa: E402  (pure Python, no native code)
