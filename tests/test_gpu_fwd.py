"""Parity of the forward kernels (fp32 SIMT and bf16 tcgen05) with the float64 oracle."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN
from online_softmax_12_b200 import inputs
from parity import compare

pytestmark = pytest.mark.gpu


def _attn():
    from online_softmax_12_b200 import attn

    return attn


def _run(x, dev, with_lse=True, out_f32=False):
    attn = _attn()
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    km = x["key_mask"].to(dev) if x.get("key_mask") is not None else None
    o, lse = attn.attn_fwd(q, k, v, x["scale"], x["causal"], km, with_lse=with_lse, out_f32=out_f32)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    return o.float().cpu().numpy(), (lse.cpu().numpy() if lse is not None else None)


@pytest.mark.parametrize("name", sorted(inputs.SMALL_FWD))
def test_small_workloads_match_oracle(name, cuda_device):
    sh = inputs.SMALL_FWD[name]
    x = inputs.make_fwd_inputs(sh)
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], x["scale"], x["causal"], x["key_mask"])
    if sh.dtype == "bf16":
        # the arithmetic, on the fp32 output, against the literal bound
        o32, lse32 = _run(x, cuda_device, out_f32=True)
        print(name, "fp32 out", compare(o32, lse32, o_ref, lse_ref, "bf16"))
        o, lse = _run(x, cuda_device)
        assert np.array_equal(lse, lse32)
        # the bf16 output is the fp32 output rounded to nearest
        assert np.array_equal(o, torch.from_numpy(o32).to(torch.bfloat16).float().numpy())
        print(name, "bf16 out", compare(o, lse, o_ref, lse_ref, "bf16", bf16_output=True))
    else:
        o, lse = _run(x, cuda_device)
        print(name, compare(o, lse, o_ref, lse_ref, sh.dtype))


def _worked_example(dtype, d):
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    s = ex["scores"]
    if dtype == torch.float32:
        # q = e0, k_j = s_j e0: q.k_j = s_j exactly in fp32
        q = torch.zeros(1, 1, 1, d)
        q[0, 0, 0, 0] = 1.0
        k = torch.zeros(1, 1, 3, d)
        k[0, 0, :, 0] = torch.tensor(s)
    else:
        # 1001 and 999 are not bf16 numbers, 1000 and +-1 are: q = e0 + e1, k = 1000 e0 + {0, 1, -1} e1
        q = torch.zeros(1, 1, 1, d)
        q[0, 0, 0, :2] = 1.0
        k = torch.zeros(1, 1, 3, d)
        k[0, 0, :, 0] = 1000.0
        k[0, 0, :, 1] = torch.tensor([x - 1000.0 for x in s])
    v = torch.zeros(1, 1, 3, d)
    v[0, 0, :, :2] = torch.tensor(ex["values"])
    return ex, q.to(dtype), k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("dtype, d", [(torch.float32, 64), (torch.bfloat16, 64), (torch.bfloat16, 128)])
def test_worked_example_on_gpu(dtype, d, cuda_device):
    """The three-key example of "Attenzione: softmax online, riscalamento e memoria",
    section 3, through the real kernels: scores (1000, 1001, 999) overflow exp in
    fp32 unless the maximum is subtracted."""
    ex, q, k, v = _worked_example(dtype, d)
    assert torch.equal(torch.einsum("d,jd->j", q[0, 0, 0].double(), k[0, 0].double()),
                       torch.tensor(ex["scores"], dtype=torch.float64))
    o, lse = _run(dict(q=q, k=k, v=v, scale=1.0, causal=False), cuda_device)
    tol = 2e-5 if dtype == torch.float32 else 1e-2
    assert np.max(np.abs(o[0, 0, 0, :2] - np.array(ex["final_o"]))) <= tol
    assert np.all(o[0, 0, 0, 2:] == 0)
    want_lse = ex["steps"][-1]["m"] + math.log(ex["steps"][-1]["l"])
    assert abs(lse[0, 0, 0] - want_lse) <= (1e-5 if dtype == torch.float32 else 1e-3) * abs(want_lse)
    # the wrong rescale's value is far outside the tolerance
    assert abs(o[0, 0, 0, 0] - ex["wrong_rescale_o1"]) > 0.4


@pytest.mark.parametrize("case", [
    dict(B=1, H=2, H_kv=2, n_q=1, n_kv=1, d=128, causal=True),
    dict(B=1, H=2, H_kv=1, n_q=3, n_kv=3, d=64, causal=False),
    dict(B=2, H=2, H_kv=2, n_q=127, n_kv=127, d=128, causal=True),
    dict(B=1, H=4, H_kv=2, n_q=129, n_kv=129, d=64, causal=True),
    dict(B=1, H=2, H_kv=2, n_q=100, n_kv=300, d=128, causal=True),   # n_q < n_kv, bottom-right
    dict(B=1, H=2, H_kv=2, n_q=300, n_kv=100, d=128, causal=True),   # n_q > n_kv: first rows see nothing
    dict(B=1, H=8, H_kv=1, n_q=257, n_kv=257, d=128, causal=True),   # 8 query heads per kv head
    dict(B=2, H=2, H_kv=2, n_q=200, n_kv=333, d=64, causal=False),
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_and_degenerate_shapes(case, dtype, cuda_device):
    g = torch.Generator().manual_seed(case["n_q"] * 7 + case["n_kv"])
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn(case["B"], case["H"], case["n_q"], case["d"], generator=g).to(tdt)
    k = torch.randn(case["B"], case["H_kv"], case["n_kv"], case["d"], generator=g).to(tdt)
    v = torch.randn(case["B"], case["H_kv"], case["n_kv"], case["d"], generator=g).to(tdt)
    scale = 1 / math.sqrt(case["d"])
    o, lse = _run(dict(q=q, k=k, v=v, scale=scale, causal=case["causal"]), cuda_device, out_f32=dtype == "bf16")
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, case["causal"])
    compare(o, lse, o_ref, lse_ref, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_key_mask_patterns(dtype, cuda_device):
    """Prefix masks, a fully masked batch row, and a scattered mask."""
    g = torch.Generator().manual_seed(99)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    B, H, n, d = 4, 2, 300, 64
    q = (torch.randn(B, H, n, d, generator=g) * 4).to(tdt)
    k = torch.randn(B, H, n, d, generator=g).to(tdt)
    v = torch.randn(B, H, n, d, generator=g).to(tdt)
    km = torch.zeros(B, n, dtype=torch.uint8)
    km[0, :1] = 1                                          # a single kept key
    km[1, :] = 0                                           # nothing kept
    km[2, :257] = 1                                        # prefix ending inside the third block
    km[3] = (torch.rand(n, generator=g) < 0.3).to(torch.uint8)   # scattered
    o, lse = _run(dict(q=q, k=k, v=v, scale=0.125, causal=False, key_mask=km), cuda_device,
                  out_f32=dtype == "bf16")
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 0.125, False, km)
    compare(o, lse, o_ref, lse_ref, dtype)
    # one kept key: the output is that value row exactly
    assert np.array_equal(o[0, :, :, :], np.broadcast_to(v[0, :, 0:1, :].float().numpy(), o[0].shape))
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))


@pytest.mark.parametrize("n", [304, 301])
def test_many_masked_batch_rows_and_causal(n, cuda_device):
    """Twenty batch rows (more rows than warps summarising the masks, each with its own
    item of work in the persistent grid), fully masked rows among them, causal
    alignment and GQA; n = 304 takes the 16-byte mask loads, n = 301 the byte loads."""
    g = torch.Generator().manual_seed(n)
    B, H, H_kv, d = 20, 4, 2, 128
    q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H_kv, n, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H_kv, n, d, generator=g).to(torch.bfloat16)
    km = (torch.rand(B, n, generator=g) < 0.6).to(torch.uint8)
    km[3] = 0
    km[11] = 0
    km[19, :] = 0
    km[19, n - 1] = 1                                      # only the last key
    o, lse = _run(dict(q=q, k=k, v=v, scale=d ** -0.5, causal=True, key_mask=km), cuda_device, out_f32=True)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, d ** -0.5, True, km)
    compare(o, lse, o_ref, lse_ref, "bf16")
    assert np.all(o[3] == 0) and np.all(np.isneginf(lse[11]))


def test_empty_key_set(cuda_device):
    attn = _attn()
    q = torch.randn(1, 2, 5, 64, device=cuda_device).to(torch.bfloat16)
    k = torch.empty(1, 2, 0, 64, device=cuda_device, dtype=torch.bfloat16)
    o, lse = attn.attn_fwd(q, k, k.clone(), 0.125, False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_causal_first_row_and_dominant_key_are_exact(cuda_device):
    """Row 0 of a causal problem keeps one key, so P = 1 exactly and O = v_0 to the
    last bit; likewise a key that dominates by more than 127 in base 2 makes every
    other weight exactly 0."""
    g = torch.Generator().manual_seed(5)
    B, H, n, d = 1, 4, 384, 128
    q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    o, _ = _run(dict(q=q, k=k, v=v, scale=d ** -0.5, causal=True), cuda_device)
    assert np.array_equal(o[0, :, 0, :], v[0, :, 0, :].float().numpy())
    hot = torch.tensor([5, 130, 250, 383])
    k2 = k.clone()
    k2[0, :, hot, :] = (q[0, :, hot, :].float() * 24).to(torch.bfloat16)
    o2, _ = _run(dict(q=q, k=k2, v=v, scale=d ** -0.5, causal=False), cuda_device)
    for t in hot.tolist():
        assert np.array_equal(o2[0, :, t, :], v[0, :, t, :].float().numpy())


def test_output_is_a_convex_combination(cuda_device):
    sh = inputs.SMALL_FWD["bf16_causal_b2_h4_n645_d128"]
    x = inputs.make_fwd_inputs(sh)
    o, _ = _run(x, cuda_device)
    v = x["v"].float().numpy()
    for i in (0, 1, 200, 644):
        vi = v[:, :, : i + 1, :]
        assert np.all(o[:, :, i, :] >= vi.min(axis=2) - 1e-2)
        assert np.all(o[:, :, i, :] <= vi.max(axis=2) + 1e-2)


def test_run_to_run_deterministic(cuda_device):
    sh = inputs.SMALL_FWD["bf16_causal_gqa_h8_kv2_n1100_d128"]
    x = inputs.make_fwd_inputs(sh)
    a = _run(x, cuda_device)
    b = _run(x, cuda_device)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def _sample_rows(sh, n_samples, seed):
    rng = np.random.default_rng(seed)
    total = sh.B * sh.H * sh.n_q
    fixed = [0, 1, sh.n_q - 1, total - 1, total - sh.n_q, (sh.B * sh.H // 2) * sh.n_q + sh.n_q // 2]
    return np.unique(np.concatenate([np.array(fixed), rng.integers(0, total, n_samples)])).astype(np.int64)


def _check_rows(name, sh, x, rows, dev):
    """The kernel's bf16 output (1e-2 plus half an ulp) and fp32 output (the literal 1e-2)
    against the oracle on `rows` (flat ids; None = every row)."""
    o_ref, lse_ref = oracle.attn_rows(x["q"], x["k"], x["v"], x["scale"], x["causal"], x["key_mask"], rows)
    sel = slice(None) if rows is None else rows
    o, lse = _run(x, dev)
    assert np.all(np.isfinite(o))
    print(name, "bf16 out", compare(o.reshape(-1, sh.d)[sel], lse.reshape(-1)[sel], o_ref, lse_ref, "bf16",
                                    bf16_output=True))
    o32, lse32 = _run(x, dev, out_f32=True)
    print(name, "fp32 out", compare(o32.reshape(-1, sh.d)[sel], lse32.reshape(-1)[sel], o_ref, lse_ref, "bf16"))
    assert np.array_equal(lse, lse32)


@pytest.mark.parametrize("name", ["bf16_causal_b4_h16_n2048_d128", "bf16_keymask_b2_h8_n4096_d64_qstd4"])
def test_full_size_workloads_every_element(name, cuda_device):
    """The causal B = 4 workload and the key-mask workload at full size, in the launch
    configuration the benchmark times: every element of O and every LSE against the
    oracle (a few seconds of float64 work each)."""
    sh = inputs.FWD_WORKLOADS[name]
    _check_rows(name, sh, inputs.make_fwd_inputs(sh), None, cuda_device)


def test_scores_in_the_hundreds_every_element(cuda_device):
    """The key-mask workload with scale 1: scaled scores reach the hundreds, so exp
    overflows fp32 unless the running maximum is subtracted (the overflow argument of
    "Attenzione: softmax online, riscalamento e memoria", sections 1 and 3); every
    element against the oracle."""
    name = "bf16_keymask_b2_h8_n4096_d64_qstd4_scale1"
    sh = inputs.FWD_SUPPLEMENTARY[name]
    x = inputs.make_fwd_inputs(sh)
    s_max = float(torch.einsum("bhid,bhjd->bhij", x["q"][:, :1, :256].float(), x["k"][:, :1].float()).abs().max())
    assert s_max > 88.0, s_max       # exp(88.8) is fp32's largest finite value
    _check_rows(name, sh, x, None, cuda_device)


def test_kv_group_slices_on_streams_match_the_whole_call(cuda_device):
    """The end-to-end measurement's call pattern: with B = 1 each kv head's group of query heads is
    a contiguous slice of Q, K, V, O and the LSE, and each slice's call runs on a side stream after
    an event.  Every slice's output must equal the whole call's, bit for bit (each query head's
    rows are computed the same way whichever call holds them)."""
    attn = _attn()
    sh = inputs.SMALL_FWD["bf16_causal_gqa_h8_kv2_n1100_d128"]
    x = inputs.make_fwd_inputs(sh)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    o_all, lse_all = attn.attn_fwd(q, k, v, x["scale"], True)
    o = torch.zeros_like(o_all)
    lse = torch.zeros_like(lse_all)
    hg, streams = sh.H // sh.H_kv, [torch.cuda.Stream(cuda_device) for _ in range(sh.H_kv)]
    start = torch.cuda.Event()
    start.record()
    for g, st in enumerate(streams):
        st.wait_event(start)
        attn.attn_fwd(q[:, g * hg:(g + 1) * hg], k[:, g:g + 1], v[:, g:g + 1], x["scale"], True, None,
                      o=o[:, g * hg:(g + 1) * hg], lse=lse[:, g * hg:(g + 1) * hg], stream=st)
    for st in streams:
        torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    assert torch.equal(o, o_all) and torch.equal(lse, lse_all)


def _moved_fraction(q, k, scale, threshold_base2):
    """Fraction of (row, full key block after the first) whose block maximum of the scaled
    scores passes the running maximum of the blocks before it by more than the threshold."""
    s = scale * np.einsum("bhid,bhjd->bhij", np.asarray(q, np.float64), np.asarray(k, np.float64))
    n = s.shape[-1]
    run = s[..., :128].max(-1)
    moved = []
    for j0 in range(128, n - 127, 128):
        bm = s[..., j0:j0 + 128].max(-1)
        moved.append((bm - run) / math.log(2.0) > threshold_base2)
        run = np.maximum(run, bm)
    return float(np.mean(moved))


def test_reference_moves_every_block(cuda_device):
    """Scores that rise along the keys: each 128-key block lifts every row's maximum by more
    than the kernel's rescale threshold (8 in base 2), so every block after the first rescales
    O.  Every element against the oracle, fp32 and bf16 output."""
    x = inputs.make_rising_score_inputs(777, 128, "bf16", 24.0, seed_index=41)
    frac = _moved_fraction(x["q"].float().numpy(), x["k"].float().numpy(), x["scale"], 8.0)
    assert frac > 0.9, frac
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], x["scale"], False)
    o32, lse32 = _run(x, cuda_device, out_f32=True)
    print("fp32 out", compare(o32, lse32, o_ref, lse_ref, "bf16"))
    o, lse = _run(x, cuda_device)
    print("bf16 out", compare(o, lse, o_ref, lse_ref, "bf16", bf16_output=True))


def test_long_context_two_whole_planes_and_sampled_rows(cuda_device):
    """The long-context causal GQA workload (n = 16384) at full size: every row of the
    first and the last query head of kv head 3 (heads 12 and 15), plus sampled rows of
    the other heads."""
    name = "bf16_causal_gqa_h32_kv8_n16384_d128"
    sh = inputs.FWD_WORKLOADS[name]
    x = inputs.make_fwd_inputs(sh)
    G = sh.H // sh.H_kv
    planes = [3 * G, 3 * G + G - 1]
    rows = np.concatenate([np.arange(h * sh.n_q, (h + 1) * sh.n_q) for h in planes] +
                          [_sample_rows(sh, 300, 17)])
    _check_rows(name, sh, x, np.unique(rows), cuda_device)


def test_fp32_workload_every_element(cuda_device):
    """The fp32 workload at full size: all 256 rows against the oracle at the fp32 bars."""
    name = "fp32_h1_n256_d64"
    sh = inputs.FWD_WORKLOADS[name]
    x = inputs.make_fwd_inputs(sh)
    o_ref, lse_ref = oracle.attn_rows(x["q"], x["k"], x["v"], x["scale"], x["causal"], x["key_mask"])
    o, lse = _run(x, cuda_device)
    print(name, compare(o.reshape(-1, sh.d), lse.reshape(-1), o_ref, lse_ref, sh.dtype))
