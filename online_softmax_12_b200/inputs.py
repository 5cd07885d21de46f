"""Seeded synthetic inputs for exact attention (prefill/forward and paged decode).

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the float64 oracle can take
their inputs from it.  Everything is drawn on the CPU with a
``torch.Generator`` seeded per workload, so a workload name plus a seed fixes
every byte of the input.

Recipe (the workload shapes come from the attention configurations the
online-softmax pages are exercised on):

* Prefill/forward: Q, K, V i.i.d. N(0, sigma^2) drawn in fp32 in the order
  Q, K, V, then rounded to bf16 with round-to-nearest-even where the workload
  is bf16.  Layout Q, O: [B, H, n_q, d]; K, V: [B, H_kv, n_kv, d]; contiguous.
  A key-padding mask, where present, keeps a contiguous prefix of each batch
  row of length L_b ~ U{1..n_kv} (inclusive), drawn after V, stored as uint8
  [B, n_kv] with 1 = keep.
* Paged decode: per-sequence lengths ~ U{len_lo..len_hi} (inclusive) first,
  then Q [S, H, d], then the keys and values of all tokens in sequence order,
  then one random permutation of the page pool.  The pool holds
  sum_s ceil(len_s / page) pages plus ``spare_pages``; the permutation's
  entries are handed out in order to (seq 0, page 0), (seq 0, page 1), ...,
  (seq 1, page 0), ...  Spare pages, the slots past len_s in each last page,
  and block-table entries past a sequence's last page (which point at a spare
  page) are filled with NaN, so any read outside a sequence poisons its output
  instead of touching memory outside the pool.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

# Seed of the blocked-vs-materialised experiment on the online-softmax page
# ("Attenzione: softmax online e riscalamento", section 4); workload k uses
# SEED_BASE + k.
SEED_BASE = 20260924


@dataclass(frozen=True)
class FwdShape:
    B: int
    H: int
    H_kv: int
    n_q: int
    n_kv: int
    d: int
    dtype: str          # "f32", "bf16" or "fp8" (E4M3 with one scale per 128-row block)
    causal: bool
    q_std: float = 1.0
    scale: float | None = None   # None -> 1/sqrt(d)
    prefix_mask: bool = False
    seed_index: int = 0

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)


@dataclass(frozen=True)
class DecodeShape:
    num_seqs: int
    H: int
    H_kv: int
    d: int
    page_size: int
    len_lo: int
    len_hi: int
    spare_pages: int = 64
    scale: float | None = None
    seed_index: int = 0

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def max_pages_per_seq(self) -> int:
        return -(-self.len_hi // self.page_size)


# The five full-size workloads, named by what they are.
FWD_WORKLOADS: dict[str, FwdShape] = {
    "fp32_h1_n256_d64": FwdShape(1, 1, 1, 256, 256, 64, "f32", False, seed_index=1),
    "bf16_causal_b4_h16_n2048_d128": FwdShape(4, 16, 16, 2048, 2048, 128, "bf16", True, seed_index=2),
    "bf16_causal_gqa_h32_kv8_n16384_d128": FwdShape(1, 32, 8, 16384, 16384, 128, "bf16", True, seed_index=3),
    "bf16_keymask_b2_h8_n4096_d64_qstd4": FwdShape(2, 8, 8, 4096, 4096, 64, "bf16", False, q_std=4.0,
                                                   prefix_mask=True, seed_index=5),
}
# The key-mask workload with scale 1: scaled scores in the hundreds (std 32), where
# exp overflows fp32 unless the running maximum is subtracted; a parity case of its
# own beside the literal workload, not a benchmark line.
FWD_SUPPLEMENTARY: dict[str, FwdShape] = {
    "bf16_keymask_b2_h8_n4096_d64_qstd4_scale1": FwdShape(2, 8, 8, 4096, 4096, 64, "bf16", False, q_std=4.0,
                                                          scale=1.0, prefix_mask=True, seed_index=5),
}
# FP8 E4M3 forward (one scale per 128-row block): the long-context causal GQA shape
FP8_WORKLOADS: dict[str, FwdShape] = {
    "fp8_causal_gqa_h32_kv8_n16384_d128": FwdShape(1, 32, 8, 16384, 16384, 128, "fp8", True, seed_index=10),
}
DECODE_WORKLOADS: dict[str, DecodeShape] = {
    "bf16_paged_decode_64seq_h32_kv8_d128_p16": DecodeShape(64, 32, 8, 128, 16, 512, 8192, seed_index=4),
}

# Reduced copies with the same structure (dtype, masking, GQA ratio, value
# distribution) at sizes the oracle finishes in seconds; sizes are chosen to
# span several 128-row tiles and end in a ragged tail.
SMALL_FWD: dict[str, FwdShape] = {
    "fp32_h1_n256_d64": FWD_WORKLOADS["fp32_h1_n256_d64"],
    "bf16_causal_b2_h4_n645_d128": FwdShape(2, 4, 4, 645, 645, 128, "bf16", True, seed_index=2),
    "bf16_causal_gqa_h8_kv2_n1100_d128": FwdShape(1, 8, 2, 1100, 1100, 128, "bf16", True, seed_index=3),
    "bf16_keymask_b2_h2_n777_d64_qstd4": FwdShape(2, 2, 2, 777, 777, 64, "bf16", False, q_std=4.0,
                                                  prefix_mask=True, seed_index=5),
}
SMALL_DECODE: dict[str, DecodeShape] = {
    "bf16_paged_decode_8seq_h32_kv8_d128_p16": DecodeShape(8, 32, 8, 128, 16, 1, 700, seed_index=4),
}


FP8_BLOCK = 128   # rows per FP8 scale block (a query tile, a key block)


def quantize_e4m3_blocks(t: torch.Tensor, block: int = FP8_BLOCK):
    """Encode t [B, heads, n, d] (fp32) as FP8 E4M3 with one scale per block of `block` rows:
    s = max|X| / 448 over the block's rows and all d columns (1 for an all-zero block), and
    X_fp8 = round-to-nearest(X / s).  Returns (uint8 bit patterns [B, heads, n, d], fp32
    descales [B, heads, ceil(n / block)])."""
    B, Hh, n, d = t.shape
    nb = -(-n // block)
    pad = torch.zeros(B, Hh, nb * block, d, dtype=torch.float32)
    pad[:, :, :n] = t
    amax = pad.view(B, Hh, nb, block * d).abs().amax(dim=3)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    scaled = pad / s.repeat_interleave(block, dim=2)[..., None]
    bits = scaled[:, :, :n].to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return bits, s.to(torch.float32).contiguous()


def make_fwd_inputs(shape: FwdShape, seed: int | None = None) -> dict:
    """Draw Q, K, V (and the key mask) for one forward workload on the CPU."""
    if seed is None:
        seed = SEED_BASE + shape.seed_index
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(shape.B, shape.H, shape.n_q, shape.d, generator=g) * shape.q_std
    k = torch.randn(shape.B, shape.H_kv, shape.n_kv, shape.d, generator=g)
    v = torch.randn(shape.B, shape.H_kv, shape.n_kv, shape.d, generator=g)
    descale = {}
    if shape.dtype == "bf16":
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    elif shape.dtype == "fp8":
        # FP8 E4M3 with one scale per block of FP8_BLOCK rows (per query tile and per key
        # block of each head): the block's largest magnitude maps to 448, the format's
        # largest finite value; stored as uint8 bit patterns plus fp32 descales
        enc = {}
        for n, t in (("q", q), ("k", k), ("v", v)):
            enc[n], descale[n] = quantize_e4m3_blocks(t)
        q, k, v = enc["q"], enc["k"], enc["v"]
    elif shape.dtype != "f32":
        raise ValueError(f"unknown dtype {shape.dtype}")
    key_mask = None
    kept = None
    if shape.prefix_mask:
        kept = torch.randint(1, shape.n_kv + 1, (shape.B,), generator=g)
        key_mask = (torch.arange(shape.n_kv)[None, :] < kept[:, None]).to(torch.uint8).contiguous()
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), key_mask=key_mask,
                kept=kept, scale=shape.softmax_scale, causal=shape.causal, seed=seed, descale=descale)


def make_rising_score_inputs(n: int, d: int, dtype: str, c_max: float, seed_index: int, B: int = 1,
                             H: int = 2) -> dict:
    """Q and K along one shared unit direction u (Q = 10 u, each key c_j u, plus N(0, 0.3^2)
    noise on both), with the keys' coordinate c_j rising linearly from -c_max to c_max along
    the sequence: each key block's scores sit above the previous block's, so every block moves
    the rows' running maximum.  V ~ N(0, 1); non-causal, no mask, H_kv = H, scale 1/sqrt(d)."""
    seed = SEED_BASE + seed_index
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(d, generator=g)
    u = u / u.norm()
    q = 10.0 * u + 0.3 * torch.randn(B, H, n, d, generator=g)
    c = torch.linspace(-c_max, c_max, n)
    k = c[:, None] * u + 0.3 * torch.randn(B, H, n, d, generator=g)
    v = torch.randn(B, H, n, d, generator=g)
    descale = {}
    if dtype == "bf16":
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    elif dtype == "fp8":
        enc = {}
        for name, t in (("q", q), ("k", k), ("v", v)):
            enc[name], descale[name] = quantize_e4m3_blocks(t)
        q, k, v = enc["q"], enc["k"], enc["v"]
    else:
        raise ValueError(f"unknown dtype {dtype}")
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), key_mask=None, kept=None,
                scale=1.0 / math.sqrt(d), causal=False, seed=seed, descale=descale)


# Backward: a forward workload plus the output gradient dO [B, H, n_q, d] ~ N(0, 1),
# drawn in fp32 from its own generator (seed + DO_SEED_OFFSET) and rounded to bf16.
DO_SEED_OFFSET = 1000
BWD_WORKLOADS: dict[str, FwdShape] = {
    "bf16_bwd_causal_gqa_h32_kv8_n16384_d128": FwdShape(1, 32, 8, 16384, 16384, 128, "bf16", True, seed_index=11),
}
# Reduced copies: several 64-row tiles with a ragged tail, both head dims, GQA,
# a key mask with sharp weights (Q ~ N(0, 4^2)), and n_q != n_kv both ways (with
# n_q > n_kv under a causal mask the first rows keep no key).
SMALL_BWD: dict[str, FwdShape] = {
    "bf16_bwd_causal_gqa_h8_kv2_n300_d128": FwdShape(1, 8, 2, 300, 300, 128, "bf16", True, seed_index=11),
    "bf16_bwd_b2_h4_n200_d64": FwdShape(2, 4, 4, 200, 200, 64, "bf16", False, seed_index=12),
    "bf16_bwd_keymask_b2_h2_n333_d64_qstd4": FwdShape(2, 2, 2, 333, 333, 64, "bf16", False, q_std=4.0,
                                                      prefix_mask=True, seed_index=13),
    "bf16_bwd_causal_b1_h4_kv1_nq100_nkv250_d128": FwdShape(1, 4, 1, 100, 250, 128, "bf16", True, seed_index=14),
    "bf16_bwd_causal_b1_h2_nq250_nkv100_d64": FwdShape(1, 2, 2, 250, 100, 64, "bf16", True, seed_index=15),
}


def make_bwd_inputs(shape: FwdShape, seed: int | None = None) -> dict:
    """The forward inputs of ``shape`` plus ``do``, the gradient of the output."""
    x = make_fwd_inputs(shape, seed)
    g = torch.Generator().manual_seed(x["seed"] + DO_SEED_OFFSET)
    do = torch.randn(shape.B, shape.H, shape.n_q, shape.d, generator=g).to(torch.bfloat16).contiguous()
    x["do"] = do
    return x


def _paged_pool(g, lens, H_kv, d, ps, spare_pages, max_pages, k_tok=None, v_tok=None):
    """K and V for every token of every sequence, scattered into a page pool.

    Draws K, then V (token order; unless given, bf16 [total tokens, H_kv, d]), then one
    permutation of the pool, handed out in (sequence, logical page) order.  Spare pages and
    the slots past each sequence's end hold NaN; unused block-table entries point at a
    spare page."""
    S = lens.numel()
    total = int(lens.sum())
    if k_tok is None:
        k_tok = torch.randn(total, H_kv, d, generator=g).to(torch.bfloat16)
    if v_tok is None:
        v_tok = torch.randn(total, H_kv, d, generator=g).to(torch.bfloat16)
    pages_per_seq = (lens + ps - 1) // ps
    n_pages = int(pages_per_seq.sum()) + spare_pages
    perm = torch.randperm(n_pages, generator=g).to(torch.int32)
    spare = perm[n_pages - 1]
    block_table = torch.full((S, max_pages), int(spare), dtype=torch.int32)
    k_pages = torch.full((n_pages, ps, H_kv, d), float("nan"), dtype=torch.bfloat16)
    v_pages = torch.full_like(k_pages, float("nan"))
    # hand the permutation out in (sequence, logical page) order
    starts = torch.cumsum(pages_per_seq, 0) - pages_per_seq
    for s in range(S):
        npg = int(pages_per_seq[s])
        block_table[s, :npg] = perm[int(starts[s]):int(starts[s]) + npg]
    # scatter every token to its (physical page, slot)
    seq_of_tok = torch.repeat_interleave(torch.arange(S), lens)
    tok_start = torch.cumsum(lens, 0) - lens
    t_in_seq = torch.arange(total) - tok_start[seq_of_tok]
    phys = block_table[seq_of_tok, t_in_seq // ps].long()
    slot = t_in_seq % ps
    k_pages[phys, slot] = k_tok
    v_pages[phys, slot] = v_tok
    return dict(k_pages=k_pages, v_pages=v_pages, block_table=block_table, k_tok=k_tok, v_tok=v_tok,
                num_pages=n_pages)


def make_decode_inputs(shape: DecodeShape, seed: int | None = None) -> dict:
    """Draw a paged KV cache, block table, lengths and one query token per sequence."""
    if seed is None:
        seed = SEED_BASE + shape.seed_index
    g = torch.Generator().manual_seed(seed)
    S, ps = shape.num_seqs, shape.page_size
    lens = torch.randint(shape.len_lo, shape.len_hi + 1, (S,), generator=g)
    q = torch.randn(S, shape.H, shape.d, generator=g).to(torch.bfloat16)
    pool = _paged_pool(g, lens, shape.H_kv, shape.d, ps, shape.spare_pages, shape.max_pages_per_seq)
    return dict(q=q.contiguous(), seq_lens=lens.to(torch.int32), scale=shape.softmax_scale, page_size=ps,
                max_pages_per_seq=shape.max_pages_per_seq, max_seq_len=shape.len_hi, seed=seed, **pool)


def make_rising_decode_inputs(shape: DecodeShape, slope: float) -> dict:
    """A decode batch whose scores rise along each sequence: Q = 10 u and the key of position
    t is slope * (t - len / 2) u, both plus N(0, 0.3^2) noise, along one random unit vector u,
    so later pages keep raising every head's running maximum.  V ~ N(0, 1).  Lengths, the
    page pool and the block table as in make_decode_inputs."""
    seed = SEED_BASE + shape.seed_index
    g = torch.Generator().manual_seed(seed)
    S, ps = shape.num_seqs, shape.page_size
    lens = torch.randint(shape.len_lo, shape.len_hi + 1, (S,), generator=g)
    u = torch.randn(shape.d, generator=g)
    u = u / u.norm()
    q = (10.0 * u + 0.3 * torch.randn(S, shape.H, shape.d, generator=g)).to(torch.bfloat16)
    pos = torch.cat([torch.arange(int(n), dtype=torch.float32) - float(n) / 2 for n in lens])
    total = int(lens.sum())
    k_tok = ((slope * pos)[:, None, None] * u + 0.3 * torch.randn(total, shape.H_kv, shape.d, generator=g))
    v_tok = torch.randn(total, shape.H_kv, shape.d, generator=g)
    pool = _paged_pool(g, lens, shape.H_kv, shape.d, ps, shape.spare_pages, shape.max_pages_per_seq,
                       k_tok=k_tok.to(torch.bfloat16), v_tok=v_tok.to(torch.bfloat16))
    return dict(q=q.contiguous(), seq_lens=lens.to(torch.int32), scale=shape.softmax_scale, page_size=ps,
                max_pages_per_seq=shape.max_pages_per_seq, max_seq_len=shape.len_hi, seed=seed, **pool)


@dataclass(frozen=True)
class PagedPrefillShape:
    """A block of n_q new query tokens per sequence (its last positions) against the
    sequence's whole paged KV cache (lengths U{len_lo..len_hi}, len_lo >= n_q)."""
    num_seqs: int
    H: int
    H_kv: int
    d: int
    n_q: int
    len_lo: int
    len_hi: int
    page_size: int = 16
    spare_pages: int = 64
    causal: bool = True
    scale: float | None = None
    seed_index: int = 0

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def max_pages_per_seq(self) -> int:
        return -(-self.len_hi // self.page_size)


def make_paged_prefill_inputs(shape: PagedPrefillShape, seed: int | None = None) -> dict:
    """Draw lengths, the n_q query tokens of every sequence, then the paged KV cache."""
    if seed is None:
        seed = SEED_BASE + shape.seed_index
    if shape.len_lo < shape.n_q:
        raise ValueError("every sequence must hold its n_q query tokens")
    g = torch.Generator().manual_seed(seed)
    S, ps = shape.num_seqs, shape.page_size
    lens = torch.randint(shape.len_lo, shape.len_hi + 1, (S,), generator=g)
    q = torch.randn(S, shape.H, shape.n_q, shape.d, generator=g).to(torch.bfloat16)
    pool = _paged_pool(g, lens, shape.H_kv, shape.d, ps, shape.spare_pages, shape.max_pages_per_seq)
    return dict(q=q.contiguous(), seq_lens=lens.to(torch.int32), scale=shape.softmax_scale, page_size=ps,
                causal=shape.causal, max_pages_per_seq=shape.max_pages_per_seq, max_seq_len=shape.len_hi,
                seed=seed, **pool)


# Chunked prefill over a paged cache: the newest 2048 tokens of each of 8 long
# sequences (contexts of 4096..16384 tokens) attend causally to the whole cache.
PAGED_PREFILL_WORKLOADS: dict[str, PagedPrefillShape] = {
    "bf16_paged_prefill_8seq_chunk2048_h32_kv8_d128_p16": PagedPrefillShape(8, 32, 8, 128, 2048, 4096, 16384,
                                                                              seed_index=6),
}


def paged_prefill_flops(x: dict, H: int, d: int) -> float:
    """Algorithmic FLOPs of a paged prefill: 4*d per (query, kept key) pair."""
    n_q = x["q"].shape[2]
    total = 0
    for n in x["seq_lens"].tolist():
        if x["causal"]:
            # query i keeps min(n, i + n - n_q + 1) keys (0 if negative)
            kept = [min(n, max(0, i + n - n_q + 1)) for i in range(n_q)]
            total += sum(kept)
        else:
            total += n * n_q
    return 4.0 * d * H * total


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous block partition of ``n_units`` independent units over ``world`` ranks."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, rem = divmod(n_units, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def with_batch(shape: FwdShape, B: int) -> FwdShape:
    return replace(shape, B=B)
