#!/usr/bin/env python
"""Benchmark of the packed-sequence encoder stack on B200.

Metric: packed tokens/s per layer forward (jagged causal attention + top-2
MoE) on the 60-user / 6823-token packing, and its fraction of the tensor
core roofline.  One step = the whole hot path once over one batch: the
attention work list, 8 layers (LayerNorm1 + QKV GEMM, jagged attention,
output projection + residual, LayerNorm2 + gate + top-2, route counting
sort, expert GEMM1 + ReLU, expert GEMM2 + combine + residual) and the
prediction head.  value = tokens x layers / step time, summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload stack8|layer]

N > 1 runs under torch.distributed.run: the job's batch is N copies of the
packing (N x 60 users), split into contiguous user ranges balanced by cost
(ptl_partition_users), one per rank; each rank runs the stack on its range
and the head probabilities are all-gathered over NCCL at the end of every
step (weak scaling: per-rank work stays one packing's worth).  The step
time is the max over ranks.  --impl reference times the CPU oracle (numpy
fp64) on this host on a bounded sample of the same workload.

value is measured on device-resident inputs, one step at a time (CUDA graph
replays, L2 flushed between steps).  e2e goes through the public serving API
(the bucketed graph runner) with pinned host buffers: every step flushes L2,
copies its batch in and its head probabilities out, and two runners on two
streams alternate so that a step's copies overlap the previous step's graph,
as a serving loop double-buffers its batches; the one-runner, one-step-at-a-
time figure is in detail.runner.
"""
from __future__ import annotations

import argparse
import datetime
import faulthandler
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed tokens/s per layer fwd (attn+top-2 MoE), 6823 tok/60 users; % TC peak"
GEMM_FLOPS_PER_TOKEN = 2 * 512 * 1536 + 2 * 512 * 512 + 2 * 512 * 8 + 2 * 2 * (2 * 512 * 1024)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
RUNNER_STRIDE = 128  # token granule of the graph runner's buckets in the end-to-end leg
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of each
# kernel kind, from one ncu --set full capture of this workload's layer 0
# (ncu flushes caches between replays, so these are cold-cache figures).  A
# kernel changed since its capture is dropped from this table until it is
# captured again.
NCU_DRAM_BYTES = {
    # the QKV launch also brings the layer's expert weights (16.8 MB) into L2
    "gemm_qkv": 25.023232e6 + 0.001280e6,
    "gemm_out": 14.528256e6,
    "gemm_expert1": 31.805440e6 + 5.067776e6,
    "attention": 21.016832e6,
    "gate": 14.056960e6,
    "combine": 28.080896e6 + 0.004352e6,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["stack8", "layer"], default="stack8")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def make_workload(name, world=1):
    """The job's batch: the 60-user / 6823-token packing (stack: 8 layers +
    head, weights from seed 2; layer: one layer, gate std 0.1, seed 1), as
    `world` copies laid end to end with their own activations and one set of
    weights when world > 1."""
    from packed_sequence_transformer_b200 import synthetic as S
    lengths = S.config1_lengths()
    if name == "stack8":
        c = S.make_case("stack8_6823tok_60u", lengths=lengths, seed=2, dtype="bf16",
                        num_layers=8, with_head=True)
    else:
        c = S.make_case("layer_6823tok_60u", lengths=lengths, seed=1, dtype="bf16",
                        gate_std=0.1)
    return S.replicate_batch(c, world, seed=1000)


def rank_part(case, world, rank):
    """This rank's share of the job's batch: contiguous users balanced by cost
    (ptl_partition_users).  Returns (t0, t1, rebased int32 offsets)."""
    from packed_sequence_transformer_b200 import ptl
    begin = ptl.partition_users(case.cu_seqlens, world)
    t0, t1, _, _, cu = ptl.part_of_batch(case.cu_seqlens, begin, rank)
    return t0, t1, cu


def gather_parts(local, count, world, cap):
    """All-gather of every rank's first `count` entries of `local` (1-D,
    padded to `cap` entries on every rank): returns (gathered [world * cap],
    counts [world]) on local's device.  Collectives only; no host sync."""
    import torch
    import torch.distributed as dist
    buf = torch.empty(world * cap, dtype=local.dtype, device=local.device)
    cnt = torch.empty(world, dtype=count.dtype, device=count.device)
    dist.all_gather_into_tensor(buf, local[:cap].contiguous())
    dist.all_gather_into_tensor(cnt, count.reshape(1))
    return buf, cnt


def concat_parts(buf, cnt, cap):
    """The gathered parts' entries in rank order (host numpy): the whole
    batch's result, since each part is a contiguous range of users."""
    buf = buf.cpu().numpy()
    return np.concatenate([buf[r * cap:r * cap + int(c)] for r, c in enumerate(cnt.cpu().tolist())])


def pct(xs, q):
    return float(np.percentile(np.asarray(xs, np.float64), q))


def max_over_ranks(x, world, device="cpu"):
    """The largest of each rank's `x` (every rank gets it); `x` itself at world 1.
    The collective runs on `device` (cuda for NCCL, cpu for gloo)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_rank, layers, world, ms_max):
    """Whole-job throughput: the token-layers all ranks processed (each rank
    runs its own batch) over the slowest rank's step time."""
    return tokens_per_rank * layers * world / (ms_max / 1e3)


def attention_flops(lengths):
    L = np.asarray(lengths, np.int64)
    return 2048 * int((L * (L + 1) // 2).sum())


# HSTU-style mask of the masked-attention leg: per user, a tenth of the
# tokens contextual, a tenth of the rest candidates in groups of four
MASKED_LEG = {"ctx_frac": 0.1, "tgt_frac": 0.1, "group": 4, "window": 0, "causal": True}


def masked_counts(lengths):
    L = np.asarray(lengths, np.int64)
    ctx = (L * MASKED_LEG["ctx_frac"]).astype(np.int32)
    tgt = ((L - ctx) * MASKED_LEG["tgt_frac"]).astype(np.int32)
    return ctx, tgt


def visible_pairs(lengths, ctx, tgt):
    """(query, key) pairs the masked leg's mask leaves visible, counted per
    user: the algorithmic work of the masked attention is 2048 FLOPs per
    visible pair (QK^T and PV over 8 heads of 64)."""
    total = 0
    for L, C, N in zip(lengths, ctx, tgt):
        L, C, N = int(L), int(C), int(N)
        if L == 0:
            continue
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        v = (j <= i) if MASKED_LEG["causal"] else np.ones((L, L), bool)
        v |= (i < C) & (j < C)
        Hs, G = L - N, MASKED_LEG["group"]
        v &= (j < Hs) | ((i >= Hs) & ((i - Hs) // G == (j - Hs) // G))
        if MASKED_LEG["window"] > 0:
            v &= np.abs(i - j) < MASKED_LEG["window"]
        total += int(v.sum())
    return total


def time_attention_legs(case, dev, stream, flush, reps=20, masked=True):
    """Device time (CUDA events, L2 flushed between launches) of the causal
    attention and (masked=True) of the masked variant on the workload's
    packing."""
    import torch

    from packed_sequence_transformer_b200 import ptl
    T, U = case.total_tokens, case.num_users
    g = torch.Generator(device="cpu").manual_seed(5)
    qkv = torch.randn(T, 1536, generator=g).to(dev, torch.bfloat16)
    cu = torch.as_tensor(case.cu_seqlens).to(dev, torch.int32)
    ctx_h, tgt_h = masked_counts(case.lengths)
    ctx, tgt = torch.as_tensor(ctx_h).to(dev), torch.as_tensor(tgt_h).to(dev)
    out = torch.empty(T, 512, dtype=torch.bfloat16, device=dev)
    ws = ptl.alloc_workspace(T, U, "bf16", dev)
    calls = {
        "causal": lambda: ptl.attention(qkv, out, cu, ws, stream=stream),
        "masked": lambda: ptl.attention_masked(qkv, out, cu, ws, causal=MASKED_LEG["causal"],
                                               num_contexts=ctx, num_targets=tgt,
                                               target_group_size=MASKED_LEG["group"],
                                               window=MASKED_LEG["window"], stream=stream),
    }
    if not masked:
        calls.pop("masked")
    res = {}
    for name, fn in calls.items():
        kt = ptl.KernelTrace(capacity=8)
        times = []
        with torch.cuda.stream(stream):
            for i in range(reps + 3):
                with kt:
                    fn()
                torch.cuda.synchronize()
                if i >= 3:
                    times.extend(t for k, t in kt.launches() if k == "attention")
                flush.fill_(float(i))
        torch.cuda.synchronize()
        st = ptl.last_device_error(ws, stream)
        if st != 0:
            raise RuntimeError(f"device error {ptl.STATUS.get(st)} in the {name} attention leg")
        res[name] = 1e3 * statistics.median(times)
    pairs = visible_pairs(case.lengths, ctx_h, tgt_h) if masked else None
    return res, pairs


def time_rep_leg(T, dev, stream, flush, reps=10, vocab=50_000, max_bag=4, seed=9):
    """The RepEncoder front end on T tokens: 28 device tables of `vocab` rows
    (1.4 GB in bf16, beyond L2), bags of 1..max_bag ids (a tenth empty);
    device time of the embedding-bag + LayerNorm kernel and of the Linear."""
    import torch

    from packed_sequence_transformer_b200 import ptl
    rng = np.random.default_rng(seed)
    g = torch.Generator(device=dev).manual_seed(seed)
    tables = [torch.randn(vocab, 512, device=dev, generator=g).to(torch.bfloat16) for _ in range(28)]
    sizes = rng.integers(1, max_bag + 1, size=T * 28)
    sizes[rng.random(T * 28) < 0.1] = 0
    off_h = np.zeros(T * 28 + 1, np.int64)
    np.cumsum(sizes, out=off_h[1:])
    ids = torch.as_tensor(rng.integers(0, vocab, size=int(off_h[-1])), dtype=torch.int64).to(dev)
    off = torch.as_tensor(off_h).to(dev)
    ln_g = torch.ones(14336, device=dev)
    ln_b = torch.zeros(14336, device=dev)
    w = (0.02 * torch.randn(512, 14336, device=dev, generator=g)).to(torch.bfloat16)
    b = torch.zeros(512, device=dev)
    st = ptl.rep_weights_struct(tables, ln_g, ln_b, w, b)
    out = torch.empty(T, 512, dtype=torch.bfloat16, device=dev)
    ws = ptl.rep_encoder_workspace(T, "bf16", dev)
    kt = ptl.KernelTrace(capacity=8)
    t_bag, t_gemm = [], []
    with torch.cuda.stream(stream):
        for i in range(reps + 3):
            with kt:
                ptl.rep_encoder(ids, off, T, st, out, ws, stream=stream)
            torch.cuda.synchronize()
            if i >= 3:
                ks = kt.launches()
                t_bag += [t for k, t in ks if k == "layernorm"]
                t_gemm += [t for k, t in ks if k == "gemm_qkv"]
            flush.fill_(float(i))
    torch.cuda.synchronize()
    if ptl.last_device_error(ws, stream) != 0:
        raise RuntimeError("device error in the RepEncoder leg")
    n_ids = int(off_h[-1])
    bag_bytes = n_ids * (1024 + 8) + T * 28 * 8 + T * 14336 * 2  # rows + ids + offsets, normalised rows out
    flops = 2 * T * 14336 * 512
    bag_us, gemm_us = 1e3 * statistics.mean(t_bag), 1e3 * statistics.mean(t_gemm)
    return {"tokens": T, "ids": n_ids, "vocab_per_slot": vocab, "embag_ln_us": bag_us,
            "embag_ln_gbs": bag_bytes / bag_us / 1e3, "linear_us": gemm_us,
            "linear_tflops": flops / gemm_us / 1e6}


def time_fp8_leg(T, dev, stream, flush, peaks, reps=10, seed=12):
    """The FP8 (e4m3) linear layers on T tokens: per-row quantisation of the
    activations, then the tcgen05 kind::f8f6f4 GEMM at the QKV shape
    (512 -> 1536), the expert GEMM1 shape (512 -> 1024) and the RepEncoder
    projection's shape (14336 -> 512, where the contraction is long enough
    for the MMA rate to show), against an e4m3 dense peak taken as the
    measured bf16 peak times the nominal e4m3 / bf16 ratio (4.5 / 2.25
    PFLOP/s)."""
    import torch

    from packed_sequence_transformer_b200 import ptl
    g = torch.Generator(device=dev).manual_seed(seed)
    x = torch.randn(T, 512, device=dev, generator=g).to(torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    fp8_peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    res = {"tokens": T, "fp8_peak_tflops": fp8_peak,
           "fp8_peak_source": "measured bf16_tflops burst x 2 (nominal e4m3 / bf16 dense ratio 4.5 / 2.25)"}
    with torch.cuda.stream(stream):
        xq, sx = ptl.quantize_rows_e4m3(x, stream=stream)
        for name, k_in, n_out in (("qkv_512x1536", 512, 1536), ("expert1_512x1024", 512, 1024),
                                  ("rep_14336x512", 14336, 512)):
            if k_in == 512:
                aq, sa = xq, sx
            else:
                xa = torch.randn(T, k_in, device=dev, generator=g).to(torch.bfloat16)
                aq, sa = ptl.quantize_rows_e4m3(xa, stream=stream)
                del xa
            w = (0.02 * torch.randn(n_out, k_in, device=dev, generator=g)).to(torch.bfloat16)
            wq, sw = ptl.quantize_rows_e4m3(w, stream=stream)
            out = torch.empty(T, n_out, dtype=torch.bfloat16, device=dev)
            ms = []
            for i in range(reps + 3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                ptl.linear_fp8(aq, sa, wq, sw, None, out, ws, stream=stream)
                b.record(stream)
                if i >= 3:
                    ms.append((a, b))
                flush.fill_(float(i))
            torch.cuda.synchronize()
            us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ms)
            tf = 2 * T * k_in * n_out / us / 1e6
            res[name] = {"us": us, "tflops": tf, "frac_of_fp8_peak": tf / fp8_peak}
        qs = []
        for i in range(reps + 3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ptl.quantize_rows_e4m3(x, xq, sx, stream=stream)
            b.record(stream)
            if i >= 3:
                qs.append((a, b))
            flush.fill_(float(i))
        torch.cuda.synchronize()
        q_us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in qs)
    if ptl.last_device_error(ws, stream) != 0:
        raise RuntimeError("device error in the FP8 leg")
    qbytes = T * 512 * (2 + 1) + 4 * T
    res["quantize_rows_us"] = q_us
    res["quantize_rows_gbs"] = qbytes / q_us / 1e3
    return res


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_id)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mhz, maxm, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                maxm = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxm, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------------- oracle
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def blas_name():
    try:
        from threadpoolctl import threadpool_info
        libs = [f"{i.get('internal_api')} {i.get('version')}" for i in threadpool_info()
                if i.get("user_api") == "blas"]
        return ", ".join(libs) if libs else "unknown"
    except Exception:
        return "unknown"


def time_oracle_layers(case, budget_s=12.0, max_reps=8, min_reps=1, layer_offset=0, threads=None):
    """Time the oracle's full-batch layer forward (layers of the case in turn),
    with the BLAS pool limited to `threads` (None: as configured); returns
    (seconds per layer: median, p10, p90; reps)."""
    from oracle import ptl_oracle as O
    ctx = None
    if threads is not None:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=threads, user_api="blas")
    try:
        times = []
        h = case.x
        t_all = time.perf_counter()
        i = 0
        while i < max_reps and (i < min_reps or time.perf_counter() - t_all < budget_s):
            w = case.layers[(layer_offset + i) % len(case.layers)]
            t0 = time.perf_counter()
            O.layer_forward(h, case.cu_seqlens, w)
            times.append(time.perf_counter() - t0)
            i += 1
    finally:
        if ctx is not None:
            ctx.unregister()
    return (statistics.median(times), pct(times, 10), pct(times, 90)), len(times)


def cpu_baseline(case, budget_all=8.0, budget_one=10.0):
    """The oracle on this host's cores: full-batch layers with every BLAS
    thread, then with one; tokens/s from the median layer time."""
    T = case.total_tokens
    (med, p10, p90), reps = time_oracle_layers(case, budget_s=budget_all, max_reps=6, min_reps=2)
    (med1, p10_1, p90_1), reps1 = time_oracle_layers(case, budget_s=budget_one, max_reps=4, min_reps=1,
                                                     threads=1)
    return {"value": T / med, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"numpy fp64 oracle, {reps} full-batch layers of this workload ({T} tokens each) "
                      f"on all BLAS threads and {reps1} on one; median layer time",
            "blas": blas_name(), "layer_s_median": med, "layer_s_p10": p10, "layer_s_p90": p90,
            "one_thread": {"value": T / med1, "layer_s_median": med1, "layer_s_p10": p10_1,
                           "layer_s_p90": p90_1, "reps": reps1}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    case = make_workload(args.workload)
    T = case.total_tokens
    # warm-up and timed steps: one oracle layer over the full batch each
    for i in range(args.warmup):
        time_oracle_layers(case, max_reps=1, layer_offset=i)
    secs = []
    for i in range(args.steps):
        (s, _, _), _ = time_oracle_layers(case, max_reps=1, layer_offset=i)
        secs.append(s)
    sec = statistics.median(secs)
    value = T / sec
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": case.name + (" (one layer per step)" if args.workload == "stack8" else ""),
                   "tokens": T, "users": case.num_users, "layers_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"numpy fp64 oracle, one full-batch layer ({T} tokens) per step; median step",
                         "blas": blas_name()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- ours
# Algorithmic work per launch of each kernel kind on T tokens: FLOPs for the
# tensor-core kernels, bytes for the bandwidth-bound ones (bf16 build, fp32
# residual x1: gate + route reads x1 and writes the LayerNorm2 row to both of
# its expert rows plus ids / weights / positions; the combine reads two
# per-route rows, x1 and the weights, writes the output and the next layer's
# LayerNorm1 row; LayerNorm reads and writes one row).
def kernel_work(T, attn_fl, separate_expert2):
    return {
        "gemm_qkv": ("tensor", 2 * T * 512 * 1536),
        "attention": ("tensor", attn_fl),
        "gemm_out": ("tensor", 2 * T * 512 * 512),
        # both expert GEMMs run in one launch (traced as gemm_expert1) unless
        # gemm_expert2 shows up as a launch of its own
        "gemm_expert1": ("tensor", 2 * (2 * T) * 512 * 1024 * (1 if separate_expert2 else 2)),
        "gemm_expert2": ("tensor", 2 * (2 * T) * 1024 * 512),
        "combine": ("hbm", T * (2 * 1024 + 2048 + 1024 + 1024 + 16)),
        "gate": ("hbm", T * (2048 + 2 * 1024 + 24)),
        "layernorm": ("hbm", T * 2048),
        "route": ("hbm", T * 24),
    }


def trace_kernels(step, stream, flush, n_launch_cap, reps):
    """Per-kernel device times: the step captured with a CUDA event before
    every launch (event nodes inside the graph), replayed `reps` times with
    the L2 flushed in between; launch i takes events[i] -> events[i + 1].
    An event node stops the next launch from starting early (programmatic
    dependent launch), so each time includes its launch gap and prologue.
    Returns {kind: {launches_per_step, avg_us, share}} and the sum of the
    per-step times (ms)."""
    import torch

    from packed_sequence_transformer_b200 import ptl
    kt = ptl.KernelTrace(capacity=n_launch_cap)
    tgraph = torch.cuda.CUDAGraph()
    with kt:
        with torch.cuda.graph(tgraph, stream=stream):
            step()
    torch.cuda.synchronize()
    recorded = []
    with torch.cuda.stream(stream):
        for i in range(reps):
            tgraph.replay()
            torch.cuda.synchronize()
            recorded.extend(kt.launches())
            flush.fill_(float(i))
    torch.cuda.synchronize()
    tgraph.reset()
    per_kind = {}
    for kind, t_ms in recorded:
        d = per_kind.setdefault(kind, [0.0, 0])
        d[0] += t_ms
        d[1] += 1
    kinds = {k: {"launches_per_step": v[1] / reps, "avg_us": 1e3 * v[0] / v[1], "share": 0.0}
             for k, v in per_kind.items()}
    tot = sum(v[0] for v in per_kind.values())
    for k, v in per_kind.items():
        kinds[k]["share"] = v[0] / tot if tot else 0.0
    return kinds, tot / reps


def apportion(kinds, step_ms):
    """Each kind's per-launch time with the event-node times scaled so that a
    step's launches add up to the measured step time (the event nodes' launch
    gaps, which programmatic launch hides in the real step, spread in
    proportion)."""
    tot_us = sum(v["avg_us"] * v["launches_per_step"] for v in kinds.values())
    f = 1e3 * step_ms / tot_us if tot_us else 0.0
    for v in kinds.values():
        v["apportioned_us"] = v["avg_us"] * f
    return kinds


def fractions(kinds, T, attn_fl, peaks):
    """Achieved throughput and fraction of the measured peak per kernel kind
    (event-node time; apportioned time in parentheses of the key names)."""
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    work = kernel_work(T, attn_fl, "gemm_expert2" in kinds)
    out = {}
    for k, v in kinds.items():
        if k not in work:
            continue
        bound, w = work[k]
        scale, peak = (1e12, bf16) if bound == "tensor" else (1e9, hbm)
        a = w / (v["avg_us"] / 1e6) / scale
        out[k] = {"bound": bound, "achieved": a, "frac": a / peak}
        if v.get("apportioned_us"):
            out[k]["frac_apportioned"] = w / (v["apportioned_us"] / 1e6) / scale / peak
    return out


def time_graph_steps(graph, stream, flush, steps, warmup):
    """Median, p10 and p90 (ms) of `steps` replays of `graph`, CUDA events on
    `stream` around each, the L2 flushed (256 MiB write) in between."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
            flush.fill_(1.0)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
            flush.fill_(float(i))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    return statistics.median(ms), pct(ms, 10), pct(ms, 90)


def time_workload_leg(case, dev, stream, flush, peaks, steps=10, attention_alone=False):
    """A larger packing through the same entry points: the stack (or layer)
    captured in a graph and replayed with the L2 flushed in between; packed
    tokens/s per layer, the per-kernel fractions of the measured peaks and,
    optionally, the attention alone on its packing."""
    import torch

    from packed_sequence_transformer_b200 import ptl
    T, U = case.total_tokens, case.num_users
    n_layers = len(case.layers)
    layers = [ptl.to_device_layer(w, "bf16", dev) for w in case.layers]
    x = torch.as_tensor(case.x).to(dev, torch.bfloat16).contiguous()
    cu = torch.as_tensor(case.cu_seqlens).to(dev, torch.int32)
    out = torch.empty_like(x)
    ws = ptl.alloc_workspace(T, U, "bf16", dev)

    def step():
        if n_layers > 1:
            ptl.stack_forward(x, out, cu, layers, ws)
        else:
            ptl.layer_forward(x, out, cu, layers[0], ws)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    st = ptl.last_device_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error {ptl.STATUS.get(st)} in the {case.name} leg")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()
    med, p10, p90 = time_graph_steps(graph, stream, flush, steps, 3)
    graph.reset()
    kinds, _ = trace_kernels(step, stream, flush, 8 * n_layers + 16, min(steps, 5))
    apportion(kinds, med)
    attn_fl = attention_flops(case.lengths)
    step_flops = n_layers * (GEMM_FLOPS_PER_TOKEN * T + attn_fl)
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    leg = {"workload": case.name, "tokens": T, "users": U, "layers": n_layers,
           "ms_per_step": med, "ms_p10": p10, "ms_p90": p90,
           "tokens_per_s_per_layer": T * n_layers / (med / 1e3),
           "us_per_layer": 1e3 * med / n_layers,
           "step_frac_of_peak": step_flops / (med / 1e3) / 1e12 / bf16,
           "kernels": kinds, "fractions": fractions(kinds, T, attn_fl, peaks)}
    if attention_alone:
        a_us, _ = time_attention_legs(case, dev, stream, flush, reps=10, masked=False)
        leg["attention_alone_us"] = a_us["causal"]
        leg["attention_alone_tflops"] = attn_fl / a_us["causal"] / 1e6
        leg["attention_alone_frac"] = leg["attention_alone_tflops"] / bf16
    del ws
    torch.cuda.empty_cache()
    return leg


def run_ours(args):
    import torch
    import torch.distributed as dist
    from packed_sequence_transformer_b200 import ptl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    ptl.lib()  # no library, no benchmark

    def barrier():
        if world > 1:
            dist.barrier()

    # the job's batch, and this rank's contiguous share of its users
    job = make_workload(args.workload, world)
    t0, t1, cu_part = rank_part(job, world, rank)
    T, U = t1 - t0, len(cu_part) - 1
    if T == 0:
        raise RuntimeError(f"rank {rank} received no tokens")
    n_layers = len(job.layers)
    layers = [ptl.to_device_layer(w, "bf16", dev) for w in job.layers]
    head = ptl.to_device_head(job.head, dev) if job.head is not None else None
    x_part = job.x[t0:t1]
    mask_part = job.pred_mask[t0:t1] if head is not None else None
    x = torch.as_tensor(x_part).to(dev, torch.bfloat16).contiguous()
    cu = torch.as_tensor(cu_part).to(dev, torch.int32)
    mask = torch.as_tensor(mask_part).to(dev, torch.uint8) if head is not None else None
    out = torch.empty_like(x)
    probs = torch.empty(T, dtype=torch.float32, device=dev) if head is not None else None
    n_pred = torch.zeros(1, dtype=torch.int32, device=dev) if head is not None else None
    ws = ptl.alloc_workspace(T, U, "bf16", dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MiB > L2
    # N > 1: the head probabilities (or output rows) of every rank are
    # all-gathered at the end of each step, padded to the largest part
    cap = int(max_over_ranks(T, world, dev))
    if world > 1:
        res_local = (torch.zeros(cap, dtype=torch.float32, device=dev) if head is not None
                     else torch.zeros(cap * 512, dtype=torch.bfloat16, device=dev))
        res_count = n_pred if head is not None else torch.tensor([T * 512], dtype=torch.int32, device=dev)
        res_cap = cap if head is not None else cap * 512

    stream = torch.cuda.Stream(device=dev)

    def step():
        if head is not None:
            ptl.stack_forward(x, out, cu, layers, ws, head=head, pred_mask=mask, probs=probs,
                              n_pred=n_pred)
        else:
            ptl.layer_forward(x, out, cu, layers[0], ws)

    def gather():
        if world > 1:
            if head is not None:
                res_local[:T].copy_(probs)
            else:
                res_local[:T * 512].copy_(out.reshape(-1))
            return gather_parts(res_local, res_count, world, res_cap)
        return None

    # eager warm-up (configures kernels), error check, then graph capture
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    st = ptl.last_device_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error {ptl.STATUS.get(st)}")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()
    # the prologue (work list, the head's output slots, layer 0's LayerNorm1)
    # in one launch, 6 kernels per layer (QKV, attention, out-projection,
    # gate + route, both expert GEMMs in one launch, combine; each layer's
    # combine writes the next layer's LayerNorm1, the last one computes the
    # head)
    launches_per_step = 1 + 6 * n_layers

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            graph.replay()
            gather()
            flush.fill_(1.0)
    torch.cuda.synchronize()

    # ---- timed region: K graph replays (+ the all-gather at N > 1), L2
    # flushed between them
    gpu_index = torch.cuda.current_device()
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = str(gpu_index)
    clocks = ClockSampler(uuid)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            evs[i][0].record(stream)
            graph.replay()
            gathered = gather()
            evs[i][1].record(stream)
            flush.fill_(float(i))
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    med_ms = statistics.median(step_ms)
    ms_max = max_over_ranks(med_ms, world, dev)
    p10_max = max_over_ranks(pct(step_ms, 10), world, dev)
    p90_max = max_over_ranks(pct(step_ms, 90), world, dev)
    value = job.total_tokens * n_layers / (ms_max / 1e3)
    if world > 1 and head is not None:
        # the gathered probabilities are the whole batch's, in token order
        n_all = int(sum(gathered[1].cpu().tolist()))
        assert n_all == int(job.pred_mask.sum())

    # ---- per-kernel device times (event nodes in a second captured graph)
    kinds, trace_ms = trace_kernels(step, stream, flush, 2 * launches_per_step + 16, min(args.steps, 10))
    apportion(kinds, med_ms)

    peaks, peak_src = load_peaks()
    lengths = np.diff(cu_part)
    attn_fl = attention_flops(lengths)
    alg = kernel_work(T, attn_fl, "gemm_expert2" in kinds)
    dom = max((k for k in kinds if k in alg), key=lambda k: kinds[k]["avg_us"] * kinds[k]["launches_per_step"])
    bound, work = alg[dom]
    t_s = kinds[dom]["avg_us"] / 1e6
    if bound == "tensor":
        achieved = work / t_s / 1e12
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        unit = "TFLOP/s"
    else:
        achieved = work / t_s / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        unit = "GB/s"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": NCU_DRAM_BYTES.get(dom), "kernel": dom,
                "peak_source": f"{peak_src} ({'bf16_tflops burst' if bound == 'tensor' else 'hbm_gbs'})",
                "algorithmic_per_launch": work,
                "time": "event nodes around each launch (includes the launch gap that programmatic "
                        "launch hides in the step); frac_apportioned scales them to the step time",
                "frac_apportioned": work / (kinds[dom]["apportioned_us"] / 1e6) / (1e12 if bound == "tensor" else 1e9) / peak}
    step_flops = n_layers * (GEMM_FLOPS_PER_TOKEN * T + attn_fl)
    whole_step_tflops = step_flops / (ms_max / 1e3) / 1e12

    # ---- end to end through the public API: the bucketed graph runner with
    # host (pinned) buffers; each step copies the batch in, replays the
    # bucket's graph and copies the result (head probabilities + count, or
    # the hidden rows) out
    x_h = torch.as_tensor(x_part).to(torch.bfloat16).pin_memory()
    cu_h = torch.as_tensor(cu_part).to(torch.int32).pin_memory()
    mask_h = torch.as_tensor(mask_part).to(torch.uint8).pin_memory() if head is not None else None
    res_h = (torch.empty(T, dtype=torch.float32).pin_memory() if head is not None
             else torch.empty(T, 512, dtype=torch.bfloat16).pin_memory())
    n_h = torch.zeros(1, dtype=torch.int32).pin_memory()
    h2d = x_h.numel() * 2 + cu_h.numel() * 4 + (mask_h.numel() if mask_h is not None else 0)
    d2h = res_h.numel() * res_h.element_size() + (4 if head is not None else 0)
    # 128-token buckets: a serving process holds one small graph per bucket,
    # and the finer stride keeps the padding work to under 128 tokens
    runner = ptl.StackRunner(T, U, layers, "bf16", head=head, stride=RUNNER_STRIDE)
    bucket = ptl.runner_bucket(T, U, RUNNER_STRIDE)[0]
    runner.capture(T)

    def run_runner(src_x, src_cu, src_mask, dst, dst_n):
        if head is not None:
            runner.forward(src_x, src_cu, pred_mask=src_mask, probs=dst, n_pred=dst_n, stream=stream)
        else:
            runner.forward(src_x, src_cu, out=dst, stream=stream)

    def timed(fn, n_warm, n_timed, host_sync):
        ms = []
        with torch.cuda.stream(stream):
            for i in range(n_warm + n_timed):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                if host_sync:
                    b.synchronize()
                if i >= n_warm:
                    ms.append((a, b))
                flush.fill_(float(i))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ms)

    e2e_serial_ms = timed(lambda: run_runner(x_h, cu_h, mask_h, res_h, n_h), args.warmup, args.steps, True)
    st = runner.last_device_error(stream)
    if st != 0:
        raise RuntimeError(f"device error {ptl.STATUS.get(st)} in the runner")

    # A serving loop double-buffers its batches: a second runner on a second
    # stream, so that step i's copies overlap step i - 1's graph.  Every step
    # still flushes L2 (its own 256 MiB buffer, on its own stream), copies its
    # inputs in from pinned host memory and its result out, inside the timed
    # region; the time is the whole run's over the steps.
    runner2 = ptl.StackRunner(T, U, layers, "bf16", head=head, stride=RUNNER_STRIDE)
    runner2.capture(T)
    stream2 = torch.cuda.Stream(device=dev)
    flush2 = torch.empty_like(flush)
    res_h2, n_h2 = torch.empty_like(res_h).pin_memory(), torch.zeros(1, dtype=torch.int32).pin_memory()
    lanes = [(runner, stream, flush, res_h, n_h), (runner2, stream2, flush2, res_h2, n_h2)]

    def pipelined_step(i):
        r, s_, fl, dst, dst_n = lanes[i % 2]
        with torch.cuda.stream(s_):
            fl.fill_(float(i))
            if head is not None:
                r.forward(x_h, cu_h, pred_mask=mask_h, probs=dst, n_pred=dst_n, stream=s_)
            else:
                r.forward(x_h, cu_h, out=dst, stream=s_)

    for i in range(args.warmup):
        pipelined_step(i)
    torch.cuda.synchronize()
    t_start, t_end, t_other = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    t_start.record(stream)
    stream2.wait_event(t_start)
    for i in range(args.steps):
        pipelined_step(i)
    t_other.record(stream2)
    stream.wait_event(t_other)
    t_end.record(stream)
    t_end.synchronize()
    e2e_ms = t_start.elapsed_time(t_end) / args.steps
    for r, s_, _, _, _ in lanes:
        st = r.last_device_error(s_)
        if st != 0:
            raise RuntimeError(f"device error {ptl.STATUS.get(st)} in the runner")
    if head is not None and not (torch.equal(res_h2[:int(n_h2.item())], res_h[:int(n_h.item())]) and
                                 int(n_h2.item()) == int(n_h.item())):
        raise RuntimeError("the two pipelined runners disagree")
    runner2.close()
    del flush2
    e2e_value = job.total_tokens * n_layers / (max_over_ranks(e2e_ms, world, dev) / 1e3)
    # the same runner on device-resident buffers (device copies + graph), and
    # the stack issued kernel by kernel from the host without a graph
    res_d = probs if head is not None else torch.empty_like(out)
    runner_ms = timed(lambda: run_runner(x, cu, mask, res_d, n_pred), 2, args.steps, False)
    eager_ms = timed(step, 2, args.steps, False)
    runner.close()

    detail = {"step_tflops": whole_step_tflops,
              "step_frac_of_peak": whole_step_tflops / float(peaks.get("bf16_tflops", 1590.0)),
              "us_per_layer": ms_max * 1e3 / n_layers,
              "ms_p10": p10_max, "ms_p90": p90_max,
              "runner": {"stride": RUNNER_STRIDE, "bucket_tokens": bucket,
                         "device_buffers_ms_per_step": runner_ms,
                         "host_buffers_ms_per_step": e2e_ms,
                         "host_buffers_serial_ms_per_step": e2e_serial_ms,
                         "host_buffers_mode": "two runners on two streams, step i's copies overlapping "
                                              "step i-1's graph; serial: one runner, one step at a time"},
              "eager_ms_per_step": eager_ms,
              "kernels": kinds, "kernel_fractions": fractions(kinds, T, attn_fl, peaks),
              "traced_step_ms": trace_ms,
              "attention_flops_per_layer": attn_fl, "gemm_flops_per_layer": GEMM_FLOPS_PER_TOKEN * T}
    cpu = None
    if rank == 0 and world == 1:
        bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        attn_us, masked_pairs = time_attention_legs(job, dev, stream, flush)
        masked_leg = {
            "mask": dict(MASKED_LEG), "visible_pairs": masked_pairs,
            "causal_us": attn_us["causal"], "masked_us": attn_us["masked"],
            "causal_tflops": attn_fl / attn_us["causal"] / 1e6,
            "masked_tflops": 2048 * masked_pairs / attn_us["masked"] / 1e6,
        }
        masked_leg["masked_frac"] = masked_leg["masked_tflops"] / bf16_peak
        rep_leg = time_rep_leg(T, dev, stream, flush)
        rep_leg["embag_ln_frac"] = rep_leg["embag_ln_gbs"] / hbm_peak
        rep_leg["linear_frac"] = rep_leg["linear_tflops"] / bf16_peak
        detail["attention_legs"] = masked_leg
        detail["rep_encoder"] = rep_leg
        detail["fp8_linear"] = time_fp8_leg(T, dev, stream, flush, peaks)
        if os.environ.get("PTL_BENCH_LARGE", "1") != "0":
            from packed_sequence_transformer_b200 import synthetic as S
            detail["config3_stack8_44000tok"] = time_workload_leg(S.config3(), dev, stream, flush, peaks)
            detail["config4_16x4096_skewed"] = time_workload_leg(S.config4(), dev, stream, flush, peaks,
                                                                 attention_alone=True)
        cpu = cpu_baseline(job)

    graph.reset()
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; lognormal user lengths, random-init weights)",
            "config": {"workload": job.name, "tokens": job.total_tokens, "users": job.num_users,
                       "layers": n_layers, "head": head is not None,
                       "parallelism": (f"users split by cost over {world} GPUs, head outputs all-gathered (NCCL)"
                                       if world > 1 else "1 GPU"),
                       "l2": "flushed between timed steps (256 MiB write)",
                       "timing": "CUDA graph replay, CUDA events per step, median of the steps (max over ranks); "
                                 "per-kernel times from event nodes in a second captured graph"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "detail": detail,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    # watchdog: a run that has not finished after this many seconds prints
    # every thread's Python stack to stderr and exits (the default run takes
    # well under a minute of GPU time)
    faulthandler.dump_traceback_later(float(os.environ.get("PTL_BENCH_WATCHDOG_S", "600")), exit=True)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
