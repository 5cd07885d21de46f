"""Parity helpers: compare the CUDA path with the float64 oracle.

Tolerances (written here once, used by every GPU test):
* fp32 inputs: max |O_gpu - O_ref| <= 2e-5 and |LSE_gpu - LSE_ref| <= 1e-5 * max(|LSE_ref|, 1).
* bf16 inputs with fp32 accumulation: max |O_gpu - O_ref| <= 1e-2 over every element, and
  |LSE_gpu - LSE_ref| <= 1e-3 * max(|LSE_ref|, 1) (the relative LSE bound, made absolute
  near LSE = 0 where a relative error is meaningless).  The 1e-2 bound applies to the
  kernel's arithmetic, checked on its fp32 output.  A bf16 output adds its own final
  rounding, up to half a bf16 ulp of O (0.0156 where |O| >= 4, above the bound by
  itself), so bf16 outputs are checked against 1e-2 + half an ulp of O_ref.
Rows with no kept key must give O = 0 and LSE = -inf on both sides.
"""
import numpy as np

TOL = {
    "f32": dict(o=2e-5, lse=1e-5),
    "bf16": dict(o=1e-2, lse=1e-3),
}


def half_ulp_bf16(x):
    """Half the spacing of bfloat16 numbers (8 significant bits) around |x|."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8.0), 0.0)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype, bf16_output=False):
    """o_*: [..., d]; lse_*: [...].  Returns a dict of error figures; raises AssertionError on failure.
    bf16_output=True: O was rounded to bf16 at the end, allow half a bf16 ulp on top of the bound."""
    tol = TOL[dtype]
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), "non-finite output"
    diff = np.abs(o_gpu - o_ref)
    err_o = float(np.max(diff)) if o_ref.size else 0.0
    out = dict(max_abs_o=err_o, max_abs_o_ref=float(np.max(np.abs(o_ref))) if o_ref.size else 0.0)
    if bf16_output:
        excess = float(np.max(diff - (tol["o"] + half_ulp_bf16(o_ref)))) if o_ref.size else -1.0
        out["max_excess_over_bound"] = excess
        assert excess <= 0.0, f"max |dO| - (1e-2 + half ulp) = {excess:.3e} > 0 (max |dO| {err_o:.3e})"
    else:
        assert err_o <= tol["o"], f"max |dO| = {err_o:.3e} > {tol['o']}"
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        empty = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), empty), "empty-row pattern differs"
        if np.any(empty):
            assert np.all(o_gpu[empty] == 0.0)
        fin = ~empty
        if np.any(fin):
            d = np.abs(lse_gpu[fin] - lse_ref[fin])
            bound = tol["lse"] * np.maximum(np.abs(lse_ref[fin]), 1.0)
            worst = float(np.max(d / bound))
            out["max_lse_err_over_bound"] = worst
            big = np.abs(lse_ref[fin]) >= 1.0
            if np.any(big):
                out["max_rel_lse"] = float(np.max(d[big] / np.abs(lse_ref[fin][big])))
            assert worst <= 1.0, f"LSE error {worst:.3f} x bound"
    return out
