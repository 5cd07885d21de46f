"""Parity of the backward pass (attn_bwd) with the float64 oracle's gradients.

The kernel gets the oracle's forward output rounded to bf16 and its LSE in fp32
(no input comes from the CUDA forward), and its dQ, dK, dV are compared element
by element with ``oracle.backward.attn_bwd``.

Tolerance (derived; the pages fix none for the backward).  Q, K, V and dO are
exact bf16 inputs and every product accumulates in fp32.  Three roundings enter:
each weight P_ij is rounded to bf16 before P^T dO (relative 2^-9), each dS_ij is
rounded to bf16 before dS^T Q and dS K (relative 2^-9), and the O the kernel is
given is bf16 (relative 2^-9 per element, which moves dO_i . O_i by at most
2^-9 |dO_i| . |O_i|).  With every factor replaced by its magnitude, the oracle's
``error_scales`` sum these terms per element (e.g. for dV_j: sum_i P_ij |dO_i|),
so the kernel is within 2^-9 times them; the bar is 2^-7 times them (a factor 4
for the fp32 accumulation and the exponential), plus a bf16 ulp of the element
for the output rounding, plus 1e-6 of the tensor's largest element.  The
relative Frobenius error must also stay below 8e-3: the roundings are random,
so a systematic fault that the loose bound would admit shows up there.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as obwd
from online_softmax_12_b200 import inputs

pytestmark = pytest.mark.gpu

R_BOUND = 2.0 ** -7
FROB = 8e-3


def _attn():
    from online_softmax_12_b200 import attn

    return attn


def _ulp_bf16(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def _oracle_fwd_inputs(x):
    o, lse = oracle.attn_fwd(x["q"], x["k"], x["v"], x["scale"], x["causal"], x.get("key_mask"))
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).to(torch.float32)


def _gpu_bwd(x, o_bf, lse32, dev):
    attn = _attn()
    km = x["key_mask"].to(dev) if x.get("key_mask") is not None else None
    dq, dk, dv = attn.attn_bwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), o_bf.to(dev), x["do"].to(dev),
                               lse32.to(dev), x["scale"], x["causal"], km)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    return dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()


def _check(name, got, ref, scale):
    bound = R_BOUND * scale + _ulp_bf16(ref) + 1e-6 * max(float(np.abs(ref).max()), 1e-30)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), name
    bad = err > bound
    assert not bad.any(), (name, int(bad.sum()), float((err - bound).max()))
    nref = float(np.linalg.norm(ref))
    if nref > 0:
        rel = float(np.linalg.norm(got - ref)) / nref
        assert rel <= FROB, (name, rel)
        return float(err.max()), rel
    return float(err.max()), 0.0


@pytest.mark.parametrize("name", sorted(inputs.SMALL_BWD))
def test_bwd_parity_small(name, cuda_device):
    sh = inputs.SMALL_BWD[name]
    x = inputs.make_bwd_inputs(sh)
    o_bf, lse32 = _oracle_fwd_inputs(x)
    dq, dk, dv = _gpu_bwd(x, o_bf, lse32, cuda_device)
    rq, rk, rv, sc = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], x["causal"], x.get("key_mask"),
                                   with_scale=True)
    out = {}
    for n, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        out[n] = _check(n, got, ref, sc[n])
    print(name, out)


def test_bwd_non_causal_variant_and_causal_differ(cuda_device):
    # the same inputs with the mask switched: both match their own oracle
    sh = inputs.SMALL_BWD["bf16_bwd_causal_gqa_h8_kv2_n300_d128"]
    for causal in (False, True):
        x = dict(inputs.make_bwd_inputs(sh))
        x["causal"] = causal
        o_bf, lse32 = _oracle_fwd_inputs(x)
        dq, dk, dv = _gpu_bwd(x, o_bf, lse32, cuda_device)
        rq, rk, rv, sc = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], causal, None, with_scale=True)
        for n, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            _check(f"{n} causal={causal}", got, ref, sc[n])


def test_bwd_single_kept_key_closed_form(cuda_device):
    # each batch row keeps one key: P = 1 there, so dQ = dK = 0 (the kernel's P is
    # within an fp32 rounding of 1, so they are within the bound of 0), dV of the kept
    # key is the sum of the group's dO rows, and every other key's dK and dV are
    # exactly 0 (weight exactly 0)
    sh = inputs.FwdShape(2, 4, 2, 130, 130, 128, "bf16", False, seed_index=16)
    x = dict(inputs.make_bwd_inputs(sh))
    mask = torch.zeros(2, 130, dtype=torch.uint8)
    mask[0, 7] = 1
    mask[1, 129] = 1
    x["key_mask"] = mask
    o_bf, lse32 = _oracle_fwd_inputs(x)
    dq, dk, dv = _gpu_bwd(x, o_bf, lse32, cuda_device)
    rq, rk, rv, sc = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], False, mask, with_scale=True)
    assert np.all(rq == 0) and np.all(rk == 0)
    _check("dq", dq, rq, sc["dq"])
    _check("dk", dk, rk, sc["dk"])
    do = x["do"].double().numpy()
    for b, j in ((0, 7), (1, 129)):
        for g in range(2):
            want = do[b, 2 * g:2 * g + 2].sum(axis=(0, 1))
            assert np.all(np.abs(dv[b, g, j] - want) <= 2.0 ** -7 * np.abs(do[b, 2 * g:2 * g + 2]).sum(axis=(0, 1))
                          + _ulp_bf16(want))
        others = [i for i in range(130) if i != j]
        assert np.all(dv[b, :, others] == 0) and np.all(dk[b, :, others] == 0)


def test_bwd_fully_masked_rows_add_nothing(cuda_device):
    # batch row 1 keeps no key: LSE = -inf there; its dQ rows and its dK, dV are 0,
    # and batch row 0 is unaffected
    sh = inputs.FwdShape(2, 2, 2, 96, 96, 64, "bf16", False, seed_index=17)
    x = dict(inputs.make_bwd_inputs(sh))
    mask = torch.ones(2, 96, dtype=torch.uint8)
    mask[1] = 0
    x["key_mask"] = mask
    o_bf, lse32 = _oracle_fwd_inputs(x)
    assert bool(torch.isneginf(lse32[1]).all())
    dq, dk, dv = _gpu_bwd(x, o_bf, lse32, cuda_device)
    assert np.all(dq[1] == 0) and np.all(dk[1] == 0) and np.all(dv[1] == 0)
    rq, rk, rv, sc = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], False, mask, with_scale=True)
    for n, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _check(n, got, ref, sc[n])


def test_bwd_one_row_and_one_key(cuda_device):
    # n_q = n_kv = 1: P = 1, dQ = dK = 0, dV = dO
    sh = inputs.FwdShape(1, 2, 1, 1, 1, 128, "bf16", True, seed_index=18)
    x = inputs.make_bwd_inputs(sh)
    o_bf, lse32 = _oracle_fwd_inputs(x)
    dq, dk, dv = _gpu_bwd(x, o_bf, lse32, cuda_device)
    rq, rk, rv, sc = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], True, None, with_scale=True)
    _check("dq", dq, rq, sc["dq"])
    _check("dk", dk, rk, sc["dk"])
    want = x["do"].double().numpy()[0].sum(axis=0)
    assert np.all(np.abs(dv[0] - want) <= _ulp_bf16(want))


def test_bwd_is_deterministic(cuda_device):
    sh = inputs.SMALL_BWD["bf16_bwd_causal_gqa_h8_kv2_n300_d128"]
    x = inputs.make_bwd_inputs(sh)
    o_bf, lse32 = _oracle_fwd_inputs(x)
    a = _gpu_bwd(x, o_bf, lse32, cuda_device)
    b = _gpu_bwd(x, o_bf, lse32, cuda_device)
    for u, w in zip(a, b):
        assert np.array_equal(u, w)


def test_bwd_after_gpu_forward(cuda_device):
    # the user path: forward on the GPU, then backward from its own O and LSE; the
    # result agrees with the oracle at the forward's own accuracy (a bf16 O within
    # 1e-2 moves dO . O by at most 1e-2 |dO|_1 per row)
    attn = _attn()
    sh = inputs.SMALL_BWD["bf16_bwd_causal_gqa_h8_kv2_n300_d128"]
    x = inputs.make_bwd_inputs(sh)
    dev = cuda_device
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd(q, k, v, x["scale"], True)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, do, lse, x["scale"], True)
    torch.cuda.synchronize()
    rq, rk, rv = obwd.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], True)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        got = got.float().cpu().numpy()
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert rel <= 2e-2, rel


def _sample(n, count, seed):
    """Block boundaries (first and last of every 64 near the ends and the middle), plus random picks."""
    fixed = [0, 1, 63, 64, 127, 128, n // 2 - 1, n // 2, n - 129, n - 128, n - 65, n - 64, n - 2, n - 1]
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.array(fixed), rng.choice(n, size=count, replace=False)]))


def test_bwd_full_size_sampled(cuda_device):
    """The benchmark's workload in the benchmark's launch: dK and dV of 512+ sampled keys
    and dQ of 512+ sampled rows of two kv heads' groups (the first and the last kv head),
    against the oracle's full-length computation of those groups (their O and LSE are what
    the kernel gets for those heads), at the same derived bar as the reduced workloads."""
    attn = _attn()
    name = "bf16_bwd_causal_gqa_h32_kv8_n16384_d128"
    sh = inputs.BWD_WORKLOADS[name]
    x = inputs.make_bwd_inputs(sh)
    dev = cuda_device
    group = sh.H // sh.H_kv
    b = 0
    groups = (0, sh.H_kv - 1)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd(q, k, v, x["scale"], True)
    fwd = {}
    for g in groups:
        o_g, lse_g = obwd.group_forward(x["q"], x["k"], x["v"], x["scale"], True, None, b, g, group)
        fwd[g] = (o_g, lse_g)
        o[b, g * group:(g + 1) * group] = torch.from_numpy(o_g).to(torch.bfloat16).to(dev)
        lse[b, g * group:(g + 1) * group] = torch.from_numpy(lse_g).to(torch.float32).to(dev)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, do, lse, x["scale"], True)
    torch.cuda.synchronize()
    assert attn.check_status() == attn.OK, attn.last_error()
    keys = _sample(sh.n_kv, 512, 41)
    rows = _sample(sh.n_q, 512, 42)
    assert keys.size >= 512 and rows.size >= 512
    for g in groups:
        o_g, lse_g = fwd[g]
        o_b = torch.from_numpy(o_g).to(torch.bfloat16).double().numpy()
        rk, rv, rq, sc = obwd.group_bwd_sampled(x["q"], x["k"], x["v"], x["do"], o_b, lse_g, x["scale"], True,
                                                None, b, g, group, keys, rows, with_scale=True)
        gk = dk[b, g].float().cpu().numpy()[keys]
        gv = dv[b, g].float().cpu().numpy()[keys]
        gq = dq[b, g * group:(g + 1) * group].float().cpu().numpy()[:, rows]
        for nm, got, ref in (("dk", gk, rk), ("dv", gv, rv), ("dq", gq, rq)):
            print(g, nm, _check(f"{nm} group {g}", got, ref, sc[nm]))
    # an invariant over the whole tensor: each kv head's dV rows sum to its query
    # heads' dO rows (every row's weights sum to 1), within the rounding bound summed
    # over the keys: 2^-7 sum_i |dO_i| plus a bf16 ulp of each dV element
    dv_d = dv.double()
    dv_sum = dv_d.sum(dim=2)
    do_g = do.double().view(sh.B, sh.H_kv, group, sh.n_q, sh.d)
    do_sum = do_g.sum(dim=(2, 3))
    ulp_sum = torch.from_numpy(_ulp_bf16(dv_d.cpu().numpy())).to(dev).sum(dim=2)
    tol = 2.0 ** -7 * do_g.abs().sum(dim=(2, 3)) + ulp_sum
    assert bool(((dv_sum - do_sum).abs() <= tol).all()), float(((dv_sum - do_sum).abs() - tol).max())
    del q, k, v, do, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    assert math.isfinite(float(np.abs(rk).max()))
