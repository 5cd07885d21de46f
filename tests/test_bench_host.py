"""Host-side pieces of bench.py that need no GPU: the oracle samples behind the
CPU baselines of the extra bench lines."""
import bench
from online_softmax_12_b200 import inputs


def test_backward_oracle_sample_sizes_and_counts_work():
    sh = inputs.SMALL_BWD["bf16_bwd_causal_gqa_h8_kv2_n300_d128"]
    x = inputs.make_bwd_inputs(sh)
    tf, secs, m = bench.oracle_bwd_sample(x, sh, 0.0)
    assert m == 128 and secs > 0 and tf > 0
    group = sh.H // sh.H_kv
    # the rate counts 10 * d FLOP per attended pair of the causal leading block
    assert abs(tf * secs * 1e12 - 10.0 * sh.d * group * 128 * 129 / 2) < 1e-6 * tf * secs * 1e12
    # a large budget stops at the workload's own size
    tf, secs, m = bench.oracle_bwd_sample(x, sh, 1e9)
    assert m == min(sh.n_q, sh.n_kv)


def test_blas_thread_count_is_positive():
    assert bench.blas_threads() >= 1


def test_paged_prefill_oracle_sample_counts_work():
    sh = inputs.PagedPrefillShape(3, 4, 2, 128, 100, 100, 400, seed_index=9)
    x = inputs.make_paged_prefill_inputs(sh)
    tf, secs, nseq = bench.oracle_paged_prefill_sample(x, sh, 0.0)
    assert nseq == 1 and secs > 0 and tf > 0
    # one query head per kv head of sequence 0 (G = 2: heads 0 and 2)
    q0 = x["q"][0:1, ::2]
    want = inputs.paged_prefill_flops({"q": q0, "seq_lens": x["seq_lens"][0:1], "causal": True}, sh.H_kv, sh.d)
    assert abs(tf * secs * 1e12 - want) < 1e-6 * want
    tf, secs, nseq = bench.oracle_paged_prefill_sample(x, sh, 1e9)
    assert nseq == sh.num_seqs


def test_fp8_oracle_sample_runs():
    sh = inputs.FwdShape(1, 4, 2, 200, 200, 128, "fp8", True, seed_index=10)
    x = inputs.make_fwd_inputs(sh)
    tf, secs, nrows = bench.oracle_fp8_sample(x, sh, 0.0)
    assert nrows == 16 and secs > 0 and tf > 0


def test_prefill_oracle_sample_counts_kept_keys():
    import numpy as np

    sh = inputs.SMALL_FWD["bf16_keymask_b2_h2_n777_d64_qstd4"]
    x = inputs.make_fwd_inputs(sh)
    tf, secs, n, _ = bench.oracle_sample(x, sh, 0.0, seed=3, kept=x["kept"], key_mask=x["key_mask"])
    rows = np.random.default_rng(3).integers(0, sh.B * sh.H * sh.n_q, n)
    want = 4.0 * sh.d * float(x["kept"].numpy()[rows // (sh.H * sh.n_q)].sum())
    assert abs(tf * secs * 1e12 - want) < 1e-6 * want


def test_extras_cover_every_further_path():
    assert set(bench.EXTRAS) == {"c1_fp32", "c2_causal_b4", "c5_keymask", "paged_prefill", "fp8", "bwd"}
