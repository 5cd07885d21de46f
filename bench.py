"""Benchmark: causal GQA bf16 prefill (TFLOP/s) and paged split-KV decode (KV GB/s) on B200.

One step = one pass of the whole hot path over one batch of synthetic inputs:
  1. attn_fwd on the long-context causal GQA prefill workload
     (bf16, B=1, H=32, H_kv=8, n_q=n_kv=16384, d=128, scale 1/sqrt(128)), then
  2. attn_decode_paged (split-KV kernel + merge kernel) on the paged decode workload
     (64 sequences of U{512..8192} tokens, H=32, H_kv=8, d=128, 16-token pages).
Both run on one CUDA stream through the C ABI.  `value` is the prefill
throughput in algorithmic TFLOP/s (4*d FLOPs per attended query-key pair; the
causal count); `decode` carries the decode bandwidth in useful GB/s (K, V, Q
and O bytes).  Inputs are resident in HBM before timing and larger than L2, so
no L2 flush is done.  `e2e` repeats both through the same C ABI with the
inputs copied from pinned host memory and the outputs read back inside the
timed region; the prefill's copies are split by kv-head group and overlap the
attention calls on the other groups (three streams), the decode's are not.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
copy of the step on its own seeded inputs (weak scaling, no data-path
collective); times are the max over ranks.

`--impl reference` times the float64 CPU oracle (the plain definition) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "bf16_causal_gqa_h32_kv8_n16384_d128"
DECODE = "bf16_paged_decode_64seq_h32_kv8_d128_p16"
BWD = "bf16_bwd_causal_gqa_h32_kv8_n16384_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------- work accounting
def prefill_flops(sh, kept_per_batch=None) -> float:
    """4*d FLOPs per (query, kept key) pair, summed over all rows."""
    total_pairs = 0
    off = sh.n_kv - sh.n_q
    for b in range(sh.B):
        n_keys = sh.n_kv if kept_per_batch is None else int(kept_per_batch[b])
        if sh.causal:
            # row i keeps keys j <= min(i + off, n_keys - 1)
            pairs = 0
            for i in range(sh.n_q):
                pairs += max(0, min(i + off, n_keys - 1) + 1)
        else:
            pairs = sh.n_q * n_keys
        total_pairs += pairs * sh.H
    return 4.0 * sh.d * total_pairs


def decode_bytes(x, d) -> int:
    """Useful bytes: every token's K and V row for each kv head, plus Q and O."""
    S, H, _ = x["q"].shape
    H_kv = x["k_pages"].shape[2]
    kv = int(x["seq_lens"].sum()) * H_kv * d * 2 * 2
    return kv + 2 * S * H * d * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel_file):
    """DRAM bytes per launch from the committed ncu summary, only if the kernel
    source is unchanged since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, "online_softmax_12_b200", "csrc", kernel_file)
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    ent = rec.get(kernel_file)
    if not ent or ent.get("source_sha256_16") != digest:
        return None
    return ent.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- ranks
def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent problem instance (weak scaling)."""
    return base_seed + 1000 * rank


def reduce_max(values, device=None):
    """Element-wise max over ranks of a list of floats (identity on one rank)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate(world, steps, flops_per_step, bytes_per_step, prefill_ms_max, decode_ms_max):
    """Whole-job throughput: units processed by all ranks over the slowest rank's time."""
    tflops = world * steps * flops_per_step / (prefill_ms_max / 1e3) / 1e12
    gbs = world * steps * bytes_per_step / (decode_ms_max / 1e3) / 1e9
    return tflops, gbs


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.sw_power_cap",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.hw_power_brake_slowdown"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "hw_power_brake"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle baseline
def oracle_sample(x_pre, sh, budget_s, seed=0, kept=None, key_mask=None):
    """Time the float64 oracle on a random sample of prefill rows sized to about budget_s seconds.
    kept / key_mask: a prefix key mask's kept lengths per batch row (for the work count) and the
    mask itself.  Returns (TFLOP/s, seconds, rows, threads)."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(seed)
    total_rows = sh.B * sh.H * sh.n_q
    off = sh.n_kv - sh.n_q

    def flops_of(rows):
        i = rows % sh.n_q
        n_keys = np.full_like(i, sh.n_kv) if kept is None else np.asarray(kept)[rows // (sh.H * sh.n_q)]
        keys = np.minimum(i + off + 1, n_keys) if sh.causal else n_keys
        return float(4.0 * sh.d * keys.sum())

    threads = oracle.default_threads()
    n = 64
    while True:
        rows = rng.integers(0, total_rows, n)
        t0 = time.perf_counter()
        oracle.attn_rows(x_pre["q"], x_pre["k"], x_pre["v"], sh.softmax_scale, sh.causal, key_mask, rows, threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n >= 1 << 17:
            return flops_of(rows) / dt / 1e12, dt, int(n), threads
        n = int(min(n * max(2.0, 1.2 * budget_s / max(dt, 1e-3)), 1 << 17))


def blas_threads() -> int:
    """Threads the float64 numpy oracle's matrix products run on."""
    try:
        from threadpoolctl import threadpool_info

        n = [int(i.get("num_threads", 0)) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:  # noqa: BLE001 - the count is informational
        pass
    return os.cpu_count() or 1


def oracle_bwd_sample(x, sh, budget_s):
    """Time the float64 backward oracle on the leading m x m block of one kv head's query heads
    (queries and keys 0..m-1: every attended pair of the block, causal or not), doubling m until
    about budget_s seconds.  Returns (TFLOP/s at 10*d per attended pair, seconds, m)."""
    from oracle import backward as obwd

    group = sh.H // sh.H_kv
    m = min(128, sh.n_q, sh.n_kv)
    while True:
        t0 = time.perf_counter()
        obwd.attn_bwd(x["q"][:1, :group, :m], x["k"][:1, :1, :m], x["v"][:1, :1, :m], x["do"][:1, :group, :m],
                      sh.softmax_scale, sh.causal)
        dt = time.perf_counter() - t0
        pairs = group * (m * (m + 1) / 2 if sh.causal else m * m)
        if dt >= budget_s or m >= min(sh.n_q, sh.n_kv):
            return 10.0 * sh.d * pairs / dt / 1e12, dt, m
        m = min(2 * m, sh.n_q, sh.n_kv)


def oracle_paged_prefill_sample(x, sh, budget_s):
    """Time the float64 paged-prefill oracle on whole sequences, one query head per kv head
    (heads 0, G, 2G, ... keep their own kv heads under the GQA mapping), until about budget_s
    seconds.  Returns (TFLOP/s at 4*d per attended pair, seconds, sequences)."""
    import oracle
    from online_softmax_12_b200 import inputs

    group = sh.H // sh.H_kv
    threads = oracle.default_threads()
    t_total, flops, seqs = 0.0, 0.0, 0
    for s in range(sh.num_seqs):
        q = x["q"][s:s + 1, ::group].contiguous()
        bt, sl = x["block_table"][s:s + 1], x["seq_lens"][s:s + 1]
        t0 = time.perf_counter()
        oracle.prefill_paged(q, x["k_pages"], x["v_pages"], bt, sl, sh.softmax_scale, True, threads)
        t_total += time.perf_counter() - t0
        flops += inputs.paged_prefill_flops({"q": q, "seq_lens": sl, "causal": True}, sh.H_kv, sh.d)
        seqs += 1
        if t_total >= budget_s:
            break
    return flops / t_total / 1e12, t_total, seqs


def oracle_fp8_sample(x, sh, budget_s, seed=0):
    """Time the float64 oracle on decoded FP8 inputs for random query rows, sized to about
    budget_s seconds.  Returns (TFLOP/s at 4*d per attended pair, seconds, rows)."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(seed)
    total_rows = sh.B * sh.H * sh.n_q
    off = sh.n_kv - sh.n_q
    d8 = x["descale"]
    threads = oracle.default_threads()
    n = 16
    while True:
        rows = rng.integers(0, total_rows, n)
        t0 = time.perf_counter()
        oracle.attn_fwd_fp8(x["q"], x["k"], x["v"], d8["q"], d8["k"], d8["v"], sh.softmax_scale, sh.causal, None,
                            rows, threads)
        dt = time.perf_counter() - t0
        i = rows % sh.n_q
        keys = np.minimum(i + off, sh.n_kv - 1) + 1 if sh.causal else np.full_like(i, sh.n_kv)
        if dt >= budget_s or n >= 1 << 15:
            return float(4.0 * sh.d * keys.sum()) / dt / 1e12, dt, int(n)
        n = int(min(n * max(2.0, 1.2 * budget_s / max(dt, 1e-3)), 1 << 15))


def oracle_decode_sample(x_dec, budget_s):
    """Time the oracle's paged decode on whole sequences until about budget_s seconds; GB/s of useful bytes."""
    import oracle

    t_total, bytes_total, seqs = 0.0, 0, 0
    S = x_dec["q"].shape[0]
    d = x_dec["q"].shape[2]
    H_kv = x_dec["k_pages"].shape[2]
    threads = oracle.default_threads()
    for s in range(S):
        sl = x_dec["seq_lens"][s:s + 1]
        t0 = time.perf_counter()
        oracle.decode_paged(x_dec["q"][s:s + 1], x_dec["k_pages"], x_dec["v_pages"], x_dec["block_table"][s:s + 1],
                            sl, x_dec["scale"], threads)
        t_total += time.perf_counter() - t0
        bytes_total += int(sl[0]) * H_kv * d * 4 + 2 * x_dec["q"].shape[1] * d * 2
        seqs += 1
        if t_total >= budget_s:
            break
    return bytes_total / t_total / 1e9, t_total, seqs, threads


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--small", action="store_true",
                    help="test aid: the reduced workloads (same structure) instead of the full-size ones")
    ap.add_argument("--ncu-case", choices=["prefill", "decode", "bwd", "fp8"], default=None,
                    help="profiling aid: launch only one kernel family on a reduced case (inputs still larger "
                         "than L2, a few hundred MB on the device), --warmup then --steps times, and exit")
    ap.add_argument("--case", choices=[k.replace("_", "-") for k in EXTRAS], default=None,
                    help="measure one further path on its own workload instead of the main step (one JSON line)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the further paths (C1, C2, C5, paged prefill, FP8, backward) after the main step")
    args = ap.parse_args()
    if args.ncu_case:
        return ncu_case(args)
    if args.case:
        return case_line(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: WORLD_SIZE={world} but --gpus={args.gpus}; using WORLD_SIZE")

    from online_softmax_12_b200 import inputs

    pre_name, dec_name = PREFILL, DECODE
    if args.small:
        pre_name, dec_name = "bf16_causal_gqa_h8_kv2_n1100_d128", "bf16_paged_decode_8seq_h32_kv8_d128_p16"
    pre_sh = {**inputs.FWD_WORKLOADS, **inputs.SMALL_FWD}[pre_name]
    dec_sh = {**inputs.DECODE_WORKLOADS, **inputs.SMALL_DECODE}[dec_name]
    config = {"workload": f"prefill:{pre_name} + decode:{dec_name}", "prefill": {
        "B": pre_sh.B, "H": pre_sh.H, "H_kv": pre_sh.H_kv, "n_q": pre_sh.n_q, "n_kv": pre_sh.n_kv, "d": pre_sh.d,
        "causal": True}, "decode": {"num_seqs": dec_sh.num_seqs, "H": dec_sh.H, "H_kv": dec_sh.H_kv, "d": dec_sh.d,
                                    "page_size": dec_sh.page_size, "len": [dec_sh.len_lo, dec_sh.len_hi]},
        "l2": "inputs larger than L2 (prefill 335 MB, decode ~1.15 GB); no flush", "parallelism": f"replicas{world}"}
    metric = "prefill attn TFLOP/s & paged-decode KV GB/s, % of B200 roofline"

    if args.impl == "reference":
        return run_reference(args, rank, world, pre_sh, dec_sh, config, metric)

    import torch
    import torch.distributed as dist

    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    from online_softmax_12_b200 import attn

    # each rank: its own independent problem instance (weak scaling)
    x_pre = inputs.make_fwd_inputs(pre_sh, seed=rank_seed(inputs.SEED_BASE + pre_sh.seed_index, rank))
    x_dec = inputs.make_decode_inputs(dec_sh, seed=rank_seed(inputs.SEED_BASE + dec_sh.seed_index, rank))
    flops = prefill_flops(pre_sh)
    dbytes = decode_bytes(x_dec, dec_sh.d)

    q, k, v = (x_pre[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty(pre_sh.B, pre_sh.H, pre_sh.n_q, dtype=torch.float32, device=dev)
    dq = x_dec["q"].to(dev)
    kp, vp = x_dec["k_pages"].to(dev), x_dec["v_pages"].to(dev)
    bt, sl = x_dec["block_table"].to(dev), x_dec["seq_lens"].to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty(dq.shape[0], dq.shape[1], dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_bytes(dq.shape[0], dec_sh.H, dec_sh.H_kv, dec_sh.d, dec_sh.len_hi),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        attn.attn_fwd(q, k, v, pre_sh.softmax_scale, True, None, o=o, lse=lse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        attn.attn_decode_paged(dq, kp, vp, bt, sl, dec_sh.len_hi, dec_sh.softmax_scale, workspace=ws, o=do,
                               lse=dlse, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    if attn.check_status() != attn.OK:
        raise SystemExit(f"device status after warm-up: {attn.last_error()}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    pre_sum, dec_sum = sum(pre_ms), sum(dec_ms)

    # e2e: same calls with host buffers, copies inside the timed region
    hq, hk, hv = (x_pre[n].pin_memory() for n in ("q", "k", "v"))
    ho, hlse = torch.empty_like(hq).pin_memory(), torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    hdq, hkp, hvp = x_dec["q"].pin_memory(), x_dec["k_pages"].pin_memory(), x_dec["v_pages"].pin_memory()
    hbt, hsl = x_dec["block_table"].pin_memory(), x_dec["seq_lens"].pin_memory()
    hdo, hdlse = torch.empty_like(hdq).pin_memory(), torch.empty(dlse.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hkp, hvp, hbt, hsl))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdo, hdlse))

    # The prefill is split by kv-head group (B = 1: each group's Q, K, V, O and LSE are contiguous
    # slices), and each group's input copy, attention call and output copy run on three streams, so
    # the host-to-device copies, the kernels and the device-to-host copies overlap.  Every byte is
    # still copied inside the timed region of every step.
    n_chunks = pre_sh.H_kv if pre_sh.B == 1 else 1
    hg, kg = pre_sh.H // n_chunks, pre_sh.H_kv // n_chunks

    def chunk(t, c, heads):
        return t[:, c * heads:(c + 1) * heads]

    copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_step(ev):
        ev[0].record(stream)
        copy_in.wait_event(ev[0])
        copy_out.wait_event(ev[0])
        for c in range(n_chunks):
            with torch.cuda.stream(copy_in):
                for dst, src, heads in ((q, hq, hg), (k, hk, kg), (v, hv, kg)):
                    chunk(dst, c, heads).copy_(chunk(src, c, heads), non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(copy_in)
            stream.wait_event(landed)
            attn.attn_fwd(chunk(q, c, hg), chunk(k, c, kg), chunk(v, c, kg), pre_sh.softmax_scale, True, None,
                          o=chunk(o, c, hg), lse=chunk(lse, c, hg), stream=stream)
            computed = torch.cuda.Event()
            computed.record(stream)
            copy_out.wait_event(computed)
            with torch.cuda.stream(copy_out):
                chunk(ho, c, hg).copy_(chunk(o, c, hg), non_blocking=True)
                chunk(hlse, c, hg).copy_(chunk(lse, c, hg), non_blocking=True)
        drained = torch.cuda.Event()
        drained.record(copy_out)
        stream.wait_event(drained)
        ev[1].record(stream)
        dq.copy_(hdq, non_blocking=True); kp.copy_(hkp, non_blocking=True); vp.copy_(hvp, non_blocking=True)
        bt.copy_(hbt, non_blocking=True); sl.copy_(hsl, non_blocking=True)
        attn.attn_decode_paged(dq, kp, vp, bt, sl, dec_sh.len_hi, dec_sh.softmax_scale, workspace=ws, o=do,
                               lse=dlse, stream=stream)
        hdo.copy_(do, non_blocking=True); hdlse.copy_(dlse, non_blocking=True)
        ev[2].record(stream)

    e2e_steps = max(3, min(args.steps, 5))
    e2e_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(e2e_steps + 1)]
    e2e_step(e2e_evs[-1])  # warm the copy engines
    barrier()
    for i in range(e2e_steps):
        e2e_step(e2e_evs[i])
    barrier()
    e2e_pre = sum(e[0].elapsed_time(e[1]) for e in e2e_evs[:e2e_steps])
    e2e_dec = sum(e[1].elapsed_time(e[2]) for e in e2e_evs[:e2e_steps])

    # max over ranks
    total_ms, pre_sum, dec_sum, e2e_pre, e2e_dec = reduce_max([total_ms, pre_sum, dec_sum, e2e_pre, e2e_dec], dev)
    if attn.check_status() != attn.OK:
        raise SystemExit(f"device status after timing: {attn.last_error()}")

    # the decode's other path on the same inputs: one kernel, clusters merging on chip
    one = None
    if not args.no_extras:
        def run_one():
            attn.attn_decode_paged(dq, kp, vp, bt, sl, dec_sh.len_hi, dec_sh.softmax_scale,
                                   split_tokens=attn.DECODE_ONE_LAUNCH, workspace=ws, o=do, lse=dlse, stream=stream)
        one_ms = Ctx(args, dev, rank, world).time(run_one)
        if attn.check_status() != attn.OK:
            raise SystemExit(f"device status after the single-launch decode: {attn.last_error()}")
        one = {"value": dbytes / (one_ms / 1e3) / 1e9, "unit": "GB/s", "ms_per_launch": one_ms,
               "split_tokens": "ATTN_DECODE_ONE_LAUNCH (clusters of 2 CTAs, on-chip merge)"}

    # the further paths, each on its own workload with its own CUDA-event times
    extras = {}
    if not args.no_extras and not args.small:
        del hq, hk, hv, ho, hkp, hvp
        ctx = Ctx(args, dev, rank, world)
        for key, fn in EXTRAS.items():
            extras[key] = fn(ctx)
            torch.cuda.empty_cache()

    if rank == 0:
        peaks, peak_src = load_peaks()
        K = args.steps
        value, dec_gbs = aggregate(world, K, flops, dbytes, pre_sum, dec_sum)
        per_launch_tflops = flops / (pre_sum / K / 1e3) / 1e12
        peak_t = float(peaks["bf16_tflops"])
        traffic = load_traffic("fwd_bf16_sm100.cu")
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            tf, secs, nrows, thr = oracle_sample(x_pre, pre_sh, args.cpu_budget)
            gbs, dsecs, nseq, _ = oracle_decode_sample(x_dec, max(2.0, args.cpu_budget / 3))
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                   "sample": f"{nrows} random query rows of the prefill workload ({secs:.1f} s, float64 C oracle, "
                             f"OpenMP); decode: {nseq} whole sequences ({dsecs:.1f} s) -> {gbs:.3f} GB/s",
                   "decode_value": gbs, "decode_unit": "GB/s"}
        line = {
            "metric": metric, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; see inputs.py)",
            "config": config,
            "decode": {"value": dec_gbs, "unit": "GB/s", "ms_per_launch_pair": dec_sum / K,
                       "useful_bytes_per_step": dbytes,
                       "roofline": {"bound": "hbm", "achieved": dbytes / (dec_sum / K / 1e3) / 1e9,
                                    "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                    "frac": dbytes / (dec_sum / K / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
                                    "frac_of_datasheet_8000": dbytes / (dec_sum / K / 1e3) / 1e9 / 8000.0,
                                    "peak_source": peak_src, "traffic": load_traffic("decode_mma.cu")},
                       "one_launch": one},
            "roofline": {"bound": "tensor", "achieved": per_launch_tflops, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": per_launch_tflops / peak_t, "traffic": traffic,
                         "kernel": "fwd_bf16_kernel<128> (tcgen05)", "peak_source": f"{peak_src} burst",
                         "frac_of_sustained": per_launch_tflops / float(peaks.get("bf16_tflops_sustained", peak_t)),
                         "frac_of_datasheet_2250": per_launch_tflops / 2250.0,
                         "flops_per_launch": flops, "ms_per_launch": pre_sum / K},
            "e2e": {"value": world * e2e_steps * flops / (e2e_pre / 1e3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "decode_value": world * e2e_steps * dbytes / (e2e_dec / 1e3) / 1e9, "decode_unit": "GB/s",
                    "steps": e2e_steps},
            "gpu_launches": 3 * K,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def ncu_case(args):
    """Reduced cases for ncu captures: the prefill workload at n = 8192 (Q 67 MB, K and V 17 MB each,
    O 67 MB), its backward and its FP8 E4M3 version at the same length, and the decode workload
    with 16 sequences (about 290 MB of K and V)."""
    import dataclasses

    import torch

    from online_softmax_12_b200 import attn, inputs

    dev = torch.device("cuda:0")
    if args.ncu_case == "prefill":
        sh = dataclasses.replace(inputs.FWD_WORKLOADS[PREFILL], n_q=8192, n_kv=8192)
        x = inputs.make_fwd_inputs(sh)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
        lse = torch.empty(sh.B, sh.H, sh.n_q, dtype=torch.float32, device=dev)
        run = lambda: attn.attn_fwd(q, k, v, sh.softmax_scale, True, None, o=o, lse=lse)  # noqa: E731
        work = f"prefill n=8192: {prefill_flops(sh) / 1e12:.4f} TFLOP per launch"
    elif args.ncu_case == "bwd":
        sh = dataclasses.replace(inputs.BWD_WORKLOADS[BWD], n_q=8192, n_kv=8192)
        x = inputs.make_bwd_inputs(sh)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
        o, lse = attn.attn_fwd(q, k, v, sh.softmax_scale, True)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.bwd_workspace_bytes(sh.B, sh.H, sh.n_q), dtype=torch.uint8, device=dev)
        run = lambda: attn.attn_bwd(q, k, v, o, do, lse, sh.softmax_scale, True, None, dq, dk, dv, ws)  # noqa: E731
        work = f"backward n=8192: {2.5 * prefill_flops(sh) / 1e12:.4f} algorithmic TFLOP per call"
    elif args.ncu_case == "fp8":
        sh = dataclasses.replace(inputs.FP8_WORKLOADS["fp8_causal_gqa_h32_kv8_n16384_d128"], n_q=8192, n_kv=8192)
        x = inputs.make_fwd_inputs(sh)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        dsc = {n: t.to(dev) for n, t in x["descale"].items()}
        o = torch.empty(sh.B, sh.H, sh.n_q, sh.d, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(sh.B, sh.H, sh.n_q, dtype=torch.float32, device=dev)
        run = lambda: attn.attn_fwd_fp8(q, k, v, dsc["q"], dsc["k"], dsc["v"], sh.softmax_scale, True,  # noqa: E731
                                        o=o, lse=lse)
        work = f"fp8 prefill n=8192: {prefill_flops(sh) / 1e12:.4f} TFLOP per launch"
    else:
        sh = dataclasses.replace(inputs.DECODE_WORKLOADS[DECODE], num_seqs=16)
        x = inputs.make_decode_inputs(sh)
        g = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        ws = torch.empty(attn.decode_workspace_bytes(sh.num_seqs, sh.H, sh.H_kv, sh.d, sh.len_hi), dtype=torch.uint8,
                         device=dev)
        o = torch.empty_like(g["q"])
        run = lambda: attn.attn_decode_paged(g["q"], g["k_pages"], g["v_pages"], g["block_table"],  # noqa: E731
                                             g["seq_lens"], sh.len_hi, sh.softmax_scale, workspace=ws, o=o)
        work = f"decode 16 seqs: {decode_bytes(x, sh.d)} useful bytes per launch pair"
    for _ in range(args.warmup + args.steps):
        run()
    torch.cuda.synchronize()
    if attn.check_status() != attn.OK:
        raise SystemExit(attn.last_error())
    print(json.dumps({"ncu_case": args.ncu_case, "launches": args.warmup + args.steps, "work": work}))


# ----------------------------------------------------------------------------- further paths
FP32_FMA_LANES_PER_SM = 128      # fp32 FMA lanes per SM (4 sub-partitions x 32)
SM_COUNT = 148
SM_MAX_MHZ = 1965.0              # clocks.max.sm of this machine's B200s


class Ctx:
    """What every further measurement needs: device, stream, step counts, peaks, CPU-baseline budget."""

    def __init__(self, args, dev, rank=0, world=1):
        self.dev, self.rank, self.world = dev, rank, world
        self.steps, self.warmup = max(3, min(args.steps, 10)), args.warmup
        self.cpu = not args.no_cpu_baseline and world == 1
        self.cpu_budget = max(0.5, args.cpu_budget / 4)
        self.peaks, self.peak_src = load_peaks()
        import torch

        self.stream = torch.cuda.current_stream()
        self._flush_buf = None

    def flush(self):
        """Write 256 MB (twice the L2) on the stream, so the next launch starts with a cold L2."""
        import torch

        if self._flush_buf is None:
            self._flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=self.dev)
        self._flush_buf.zero_()

    def time(self, run, flush=False):
        """Mean ms per call of run() over self.steps calls after self.warmup, CUDA events on the
        launching stream around each call (a flush, when asked, runs before the start event);
        the max over ranks."""
        import torch

        for _ in range(self.warmup):
            if flush:
                self.flush()
            run()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(self.steps)]
        for e0, e1 in ev:
            if flush:
                self.flush()
            e0.record(self.stream)
            run()
            e1.record(self.stream)
        torch.cuda.synchronize()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / self.steps
        return reduce_max([ms], self.dev)[0]

    def check(self, what):
        from online_softmax_12_b200 import attn

        if attn.check_status() != attn.OK:
            raise SystemExit(f"device status after {what}: {attn.last_error()}")

    def tensor_roofline(self, flops, ms, peak=None, src=None, **extra):
        peak = float(self.peaks["bf16_tflops"]) if peak is None else peak
        tf = flops / (ms / 1e3) / 1e12
        out = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
               "peak_source": src or f"{self.peak_src} burst", "flops_per_launch": flops, "ms_per_launch": ms}
        out.update(extra)
        return out


def measure_c1_fp32(ctx):
    """The fp32 workload (B = H = 1, n = 256, d = 64): microseconds per launch of the SIMT kernel,
    warm (its 0.3 MB of inputs live in L2 between launches; the launch latency is the bound)."""
    import oracle
    from online_softmax_12_b200 import attn, inputs

    name = "fp32_h1_n256_d64"
    sh = inputs.FWD_WORKLOADS[name]
    x = inputs.make_fwd_inputs(sh, seed=rank_seed(inputs.SEED_BASE + sh.seed_index, ctx.rank))
    q, k, v = (x[n].to(ctx.dev) for n in ("q", "k", "v"))
    o = torch_empty_like(q)
    lse = torch_empty((sh.B, sh.H, sh.n_q), ctx.dev)
    run = lambda: attn.attn_fwd(q, k, v, sh.softmax_scale, False, None, o=o, lse=lse, stream=ctx.stream)  # noqa: E731
    ms = ctx.time(run)
    ctx.check(name)
    flops = prefill_flops(sh)
    peak = SM_COUNT * FP32_FMA_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12
    tf = flops / (ms / 1e3) / 1e12
    out = {"value": ms * 1e3, "unit": "us", "higher_is_better": False, "tflops": tf, "workload": name,
           "steps": ctx.steps, "l2": "warm (inputs 0.2 MB)",
           "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz (nominal)",
                        "flops_per_launch": flops, "ms_per_launch": ms},
           "gpu_launches": ctx.steps}
    if ctx.cpu:
        t0, n = time.perf_counter(), 0
        while time.perf_counter() - t0 < ctx.cpu_budget:
            oracle.attn_rows(x["q"], x["k"], x["v"], sh.softmax_scale, False)
            n += 1
        secs = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": secs / n * 1e6, "unit": "us", "cores": oracle.default_threads(),
                               "kind": "oracle", "sample": f"the whole workload {n} times ({secs:.1f} s)"}
    return out


def measure_prefill_flushed_warm(ctx, name, kept=False):
    """A bf16 forward workload whose inputs fit in (or near) the L2: TFLOP/s with the L2 flushed
    before every launch (the headline of the entry) and warm (back-to-back launches)."""
    from online_softmax_12_b200 import attn, inputs

    sh = inputs.FWD_WORKLOADS[name]
    x = inputs.make_fwd_inputs(sh, seed=rank_seed(inputs.SEED_BASE + sh.seed_index, ctx.rank))
    q, k, v = (x[n].to(ctx.dev) for n in ("q", "k", "v"))
    km = x["key_mask"].to(ctx.dev) if x["key_mask"] is not None else None
    o = torch_empty_like(q)
    lse = torch_empty((sh.B, sh.H, sh.n_q), ctx.dev)
    run = lambda: attn.attn_fwd(q, k, v, sh.softmax_scale, sh.causal, km, o=o, lse=lse,  # noqa: E731
                                stream=ctx.stream)
    ms_cold = ctx.time(run, flush=True)
    ms_warm = ctx.time(run)
    ctx.check(name)
    flops = prefill_flops(sh, x["kept"].tolist() if kept else None)
    tf = flops / (ms_cold / 1e3) / 1e12
    out = {"value": tf, "unit": "TFLOP/s", "warm_value": flops / (ms_warm / 1e3) / 1e12, "workload": name,
           "flop_count": "4*d per kept (query, key) pair" + (" (kept keys only)" if kept else " (causal count)"),
           "l2": "flushed (256 MB write) before each launch; warm_value: back-to-back launches",
           "steps": ctx.steps,
           "roofline": ctx.tensor_roofline(flops, ms_cold, warm_frac=flops / (ms_warm / 1e3) / 1e12 /
                                           float(ctx.peaks["bf16_tflops"])),
           "gpu_launches": 2 * ctx.steps}
    if ctx.cpu:
        ctf, secs, nrows, thr = oracle_sample(x, sh, ctx.cpu_budget, kept=x["kept"] if kept else None,
                                              key_mask=x["key_mask"])
        out["cpu_baseline"] = {"value": ctf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                               "sample": f"{nrows} random query rows ({secs:.1f} s, float64 C oracle)"}
    return out


def torch_empty_like(t):
    import torch

    return torch.empty_like(t)


def torch_empty(shape, dev, dtype=None):
    import torch

    return torch.empty(*shape, dtype=torch.float32 if dtype is None else dtype, device=dev)


def measure_paged_prefill(ctx):
    """Chunked prefill over a paged KV cache (attn_prefill_paged): 8 sequences of
    4096..16384 tokens, the newest 2048 of each as causal queries, 16-token pages.
    Algorithmic TFLOP/s (4*d per attended pair) against the measured dense bf16 peak."""
    import torch

    from online_softmax_12_b200 import attn, inputs

    name = "bf16_paged_prefill_8seq_chunk2048_h32_kv8_d128_p16"
    sh = inputs.PAGED_PREFILL_WORKLOADS[name]
    x = inputs.make_paged_prefill_inputs(sh, seed=rank_seed(inputs.SEED_BASE + sh.seed_index, ctx.rank))
    g = {n: (t.to(ctx.dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
    flops = inputs.paged_prefill_flops(x, sh.H, sh.d)
    o = torch.empty_like(g["q"])
    lse = torch_empty((sh.num_seqs, sh.H, sh.n_q), ctx.dev)
    run = lambda: attn.attn_prefill_paged(g["q"], g["k_pages"], g["v_pages"], g["block_table"],  # noqa: E731
                                          g["seq_lens"], sh.softmax_scale, True, o=o, lse=lse, stream=ctx.stream)
    ms = ctx.time(run)
    ctx.check(name)
    out = {"value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "workload": name, "steps": ctx.steps,
           "config": {"num_seqs": sh.num_seqs, "chunk": sh.n_q, "len": [sh.len_lo, sh.len_hi], "H": sh.H,
                      "H_kv": sh.H_kv, "d": sh.d, "page_size": sh.page_size, "causal": True},
           "l2": "K/V pool and Q larger than L2; no flush",
           "roofline": ctx.tensor_roofline(flops, ms), "gpu_launches": ctx.steps}
    if ctx.cpu:
        import oracle

        ctf, csecs, nseq = oracle_paged_prefill_sample(x, sh, ctx.cpu_budget)
        out["cpu_baseline"] = {"value": ctf, "unit": "TFLOP/s", "cores": oracle.default_threads(), "kind": "oracle",
                               "sample": f"{nseq} whole sequence(s), one query head per kv head ({csecs:.1f} s, "
                                         "float64 C oracle)"}
    return out


def measure_fp8(ctx):
    """The long-context causal GQA prefill shape on block-scaled FP8 E4M3 inputs (attn_fwd_fp8,
    one descale per 128-row block, bf16 output).  Algorithmic TFLOP/s against the dense FP8 peak, taken as the measured bf16
    peak times 2 (the nominal FP8 : bf16 ratio)."""
    import torch

    from online_softmax_12_b200 import attn, inputs

    name = "fp8_causal_gqa_h32_kv8_n16384_d128"
    sh = inputs.FP8_WORKLOADS[name]
    x = inputs.make_fwd_inputs(sh, seed=rank_seed(inputs.SEED_BASE + sh.seed_index, ctx.rank))
    q, k, v = (x[n].to(ctx.dev) for n in ("q", "k", "v"))
    dsc = {n: t.to(ctx.dev) for n, t in x["descale"].items()}
    flops = prefill_flops(sh)
    o = torch.empty(sh.B, sh.H, sh.n_q, sh.d, dtype=torch.bfloat16, device=ctx.dev)
    lse = torch_empty((sh.B, sh.H, sh.n_q), ctx.dev)
    run = lambda: attn.attn_fwd_fp8(q, k, v, dsc["q"], dsc["k"], dsc["v"], sh.softmax_scale, True,  # noqa: E731
                                    o=o, lse=lse, stream=ctx.stream)
    ms = ctx.time(run)
    ctx.check(name)
    peak = 2.0 * float(ctx.peaks["bf16_tflops"])
    out = {"value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "workload": name, "dtype": "fp8-e4m3",
           "steps": ctx.steps, "l2": "inputs larger than L2; no flush",
           "roofline": ctx.tensor_roofline(flops, ms, peak, f"{ctx.peak_src} bf16 burst x 2 (nominal fp8 ratio)"),
           "gpu_launches": ctx.steps}
    if ctx.cpu:
        import oracle

        ctf, csecs, nrows = oracle_fp8_sample(x, sh, ctx.cpu_budget)
        out["cpu_baseline"] = {"value": ctf, "unit": "TFLOP/s", "cores": oracle.default_threads(), "kind": "oracle",
                               "sample": f"{nrows} random query rows on the decoded E4M3 inputs ({csecs:.1f} s, "
                                         "float64 C oracle)"}
    return out


def measure_bwd(ctx):
    """Backward pass (attn_bwd) of the long-context causal GQA prefill shape, from the
    forward's own O and LSE.  Algorithmic TFLOP/s: 10 * d per attended pair and head
    (the five products S, dP, dV, dK, dQ; 2.5 times the forward's 4 * d), whatever the
    kernels recompute; CUDA events around the whole call."""
    import torch

    from online_softmax_12_b200 import attn, inputs

    sh = inputs.BWD_WORKLOADS[BWD]
    x = inputs.make_bwd_inputs(sh, seed=rank_seed(inputs.SEED_BASE + sh.seed_index, ctx.rank))
    q, k, v, do = (x[n].to(ctx.dev) for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd(q, k, v, sh.softmax_scale, True, stream=ctx.stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn.bwd_workspace_bytes(sh.B, sh.H, sh.n_q), dtype=torch.uint8, device=ctx.dev)
    flops = 2.5 * prefill_flops(sh)
    run = lambda: attn.attn_bwd(q, k, v, o, do, lse, sh.softmax_scale, True, None, dq, dk, dv, ws,  # noqa: E731
                                stream=ctx.stream)
    ms = ctx.time(run)
    ctx.check(BWD)
    out = {"value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "workload": BWD, "steps": ctx.steps,
           "l2": "inputs larger than L2; no flush",
           "roofline": ctx.tensor_roofline(flops, ms, flops_executed_per_launch=1.4 * flops),
           "gpu_launches": 3 * ctx.steps}
    if ctx.cpu:
        ctf, csecs, m = oracle_bwd_sample(x, sh, ctx.cpu_budget)
        out["cpu_baseline"] = {"value": ctf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": f"float64 gradients of the leading {m}x{m} causal block of one kv head's "
                                         f"{sh.H // sh.H_kv} query heads ({csecs:.1f} s, numpy)"}
    return out


EXTRAS = {"c1_fp32": measure_c1_fp32,
          "c2_causal_b4": lambda ctx: measure_prefill_flushed_warm(ctx, "bf16_causal_b4_h16_n2048_d128"),
          "c5_keymask": lambda ctx: measure_prefill_flushed_warm(ctx, "bf16_keymask_b2_h8_n4096_d64_qstd4", True),
          "paged_prefill": measure_paged_prefill, "fp8": measure_fp8, "bwd": measure_bwd}


def case_line(args):
    """--case X: one further path alone, as its own JSON line."""
    import torch

    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    key = args.case.replace("-", "_")
    out = EXTRAS[key](Ctx(args, dev))
    out.update({"metric": key, "n_gpus": 1, "warmup": args.warmup})
    print(json.dumps(out))


def run_reference(args, rank, world, pre_sh, dec_sh, config, metric):
    """The float64 oracle on the host cores, one bounded sample of the workload per step."""
    if rank != 0:
        return
    from online_softmax_12_b200 import inputs

    x_pre = inputs.make_fwd_inputs(pre_sh)
    x_dec = inputs.make_decode_inputs(dec_sh)
    # about 90 s of oracle work in all, at least 1 s per step (0.1 s with --small)
    per_step = max(0.1 if args.small else 1.0, 90.0 / (args.steps + args.warmup))
    if args.small:
        per_step = min(per_step, 0.5)
    for i in range(args.warmup):
        oracle_sample(x_pre, pre_sh, min(per_step, 1.0), seed=100 + i)
    vals, secs_all = [], 0.0
    for i in range(args.steps):
        tf, secs, nrows, thr = oracle_sample(x_pre, pre_sh, per_step, seed=i)
        vals.append(tf)
        secs_all += secs
    gbs, dsecs, nseq, _ = oracle_decode_sample(x_dec, max(0.1 if args.small else 2.0, per_step))
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs_all / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 inputs widened to float64)", "config": config,
        "decode": {"value": gbs, "unit": "GB/s"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": f"each step: random query rows of the prefill workload, ~{per_step:.1f} s of "
                                   f"float64 oracle work; decode: {nseq} whole sequences"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
