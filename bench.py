#!/usr/bin/env python
"""Throughput of the shared-QK LSH attention forward pass on B200.

One step = the whole hot path over one batch of synthetic input already in
HBM: lsh_hash -> lsh_sort_permute -> lsh_chunk_attend -> lsh_combine_rounds
(four C-ABI calls).  Metric: tokens/s = B*H*L / step time, all rounds
included, at the 64K workload (B 8, H 8, L 65536, D 128, bf16, 1024 buckets,
chunk 64, 8 rounds).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU.  The (b, h) slices are
independent, so there is no collective on the data path; the step time is the
max over ranks.  --split replicas (default): every rank processes its own full
workload -> weak scaling.  --split slices: the ranks split the B*H slices of one
batch -> strong scaling (the 1M workload's 8 heads over up to 8 GPUs).

--impl reference times the float64 CPU oracle (the only other implementation
of the method here) on rank 0, one bounded sample of the same workload per
step.  Rank 0 prints one JSON line.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LSH-attn fwd tokens/s (B·H·L) at L=64K, 8 rounds, 1×B200; % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ("hash", "sort", "attend", "combine")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def algorithmic(w):
    """Algorithmic bytes / flops per stage (per launch = one step over the whole workload).

    Per token-round: bucket write+read 8 B, perm write+read 8 B, gather of the
    QK and V rows 2*D*s, per-round output write+read 2*(D*s + 4).  Per token:
    the hash reads the row (D*s) and the merge writes the output (D*s).
    """
    s = 2 if w.dtype == "bf16" else 4
    T = w.tokens
    TR = T * w.n_rounds
    row = w.D * s
    return {
        "hash": {"bytes": T * row + TR * 4, "flops": 2.0 * T * w.D * (w.n_buckets // 2) * w.n_rounds},
        "sort": {"bytes": TR * (4 + 4), "flops": 0.0},
        "attend": {"bytes": TR * (4 + 2 * row + row + 4), "flops": 8.0 * TR * w.chunk * w.D},
        "combine": {"bytes": TR * (row + 4) + T * row, "flops": 0.0},
        "total_bytes": TR * (2 * row + 2 * (row + 4) + 8 + 8) + T * 2 * row,
        "attn_flops": 8.0 * TR * w.chunk * w.D,
    }


def backward_flops(w):
    """Algorithmic FLOPs of one backward over the workload: per admissible-window pair
    (query, key) of a round, five length-D dot products or rank-1 updates (the logit, dout . v,
    and the dq, dk, dv contributions), 2 D flops each.  A query of chunk 0 sees c keys, every
    other query 2 c, so a (b, h, round) segment has L 2c - c^2 pairs."""
    pairs = w.B * w.H * w.n_rounds * (w.L * 2 * w.chunk - w.chunk * w.chunk)
    return 10.0 * w.D * pairs


def backward_on_tensor_cores(w, args):
    """The library's tensor-core backward serves bf16, D 128, chunk 64, L % 128 == 0 with every mask
    (the union correction up to 8 rounds); everything else runs on the CUDA cores."""
    return (w.dtype == "bf16" and w.D == 128 and w.chunk == 64 and w.L % 128 == 0
            and not (args.union and w.n_rounds > 8))


def measured_sm_max_mhz(default=1965.0):
    """Maximum SM clock recorded with the measured peaks (the nominal 1965 MHz otherwise)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return default
    with open(path) as f:
        return float(json.load(f).get("sm_max_mhz", default))


def alu_peak_tflops(sms, sm_mhz):
    """FP32 FMA peak of the CUDA cores: 128 FP32 lanes per SM, 2 flops per FMA."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def kernel_bound(stage):
    return "tensor" if stage == "hash" else "hbm"


def source_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(stage, workload):
    """DRAM bytes per launch of `stage` on `workload` from the committed ncu
    summary (profiles/traffic.json), or None.

    The summary stores a digest of the kernel sources it was taken on; a
    changed kernel invalidates it.
    """
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(stage)
    if not rec or workload not in rec.get("per_launch_bytes", {}):
        return None
    try:
        if source_digest(rec["sources"]) != rec["digest"]:
            return None
    except OSError:
        return None
    return rec["per_launch_bytes"][workload]


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def mask_options(args):
    """Keyword arguments of the attention masks the command line selects."""
    return {"causal": args.causal, "bucket_mask": args.bucket_mask or args.union, "union": args.union}


def mask_config(args):
    """The "mask" entry of the JSON config (absent for the plain window)."""
    names = [n for n, on in (("causal", args.causal), ("bucket", args.bucket_mask or args.union),
                             ("union", args.union)) if on]
    return {"mask": "+".join(names)} if names else {}


def oracle_sample(w, slices=1, seed=0, masks=None, threads=None, max_tokens=None):
    """Runs the float64 oracle on `slices` (b, h) slices of the workload, all rounds.

    `threads` caps the BLAS thread pools (None: as many as the library starts).
    `max_tokens` (a multiple of the chunk) bounds the sample on very long
    sequences: the oracle then runs on the first `max_tokens` positions of each
    slice with the workload's own D, buckets, chunk and rounds.
    Returns (seconds, tokens, threads).
    """
    import contextlib

    import numpy as np
    import threadpoolctl

    from lsh_attention_hash_b200 import synth
    from oracle import oracle_lsh_attention

    R = synth.projections(w, seed)
    tokens, secs = 0, 0.0
    limit = threadpoolctl.threadpool_limits(threads) if threads else contextlib.nullcontext()
    with limit:
        for n in range(slices):
            b, h = divmod(n % (w.B * w.H), w.H)
            qk_s, v_s = synth.slice_inputs(w, b, h, seed)
            if max_tokens is not None and max_tokens < w.L:
                qk_s, v_s = qk_s[:max_tokens], v_s[:max_tokens]
            qk = qk_s[None, None]
            v = v_s[None, None]
            t0 = time.perf_counter()
            oracle_lsh_attention(qk, v, R, w.n_buckets, w.chunk, **(masks or {}))
            secs += time.perf_counter() - t0
            tokens += qk_s.shape[0]
        info = threadpoolctl.threadpool_info()
        used = max([i.get("num_threads", 1) for i in info] + [1])
    return secs, tokens, used


def cpu_sample_plan(w, seconds=10.0):
    """(slices, max_tokens) of a bounded oracle sample of about `seconds` of float64 CPU work: the
    oracle runs at about 1.5e10 operations/s here, and a token costs its hash (D * n_buckets per
    round) and its attention (8 * chunk * D per round).  Long sequences are cut to a prefix of a
    slice (a multiple of the chunk); short ones repeat slices (at most 256)."""
    per_token = w.n_rounds * (w.D * w.n_buckets + 8 * w.chunk * w.D) + 2000
    tokens = max(w.chunk, int(1.5e10 * seconds / per_token))
    if tokens >= w.L:
        return min(256, max(1, tokens // w.L)), None
    return 1, max(w.chunk, (tokens // w.chunk) * w.chunk)


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    slices, cap = cpu_sample_plan(w, seconds=4.0)
    for _ in range(args.warmup):
        oracle_sample(w, 1, masks=mask_options(args), max_tokens=cap)
    secs, tokens, threads = 0.0, 0, 1
    for _ in range(args.steps):
        s, t, threads = oracle_sample(w, slices, masks=mask_options(args), max_tokens=cap)
        secs += s
        tokens += t
    value = tokens / secs
    what = f"the first {cap} tokens of a (b,h) slice" if cap else f"{slices} (b,h) slice(s) ({slices * w.L} tokens)"
    sample = f"per step {what} of the workload, all {w.n_rounds} rounds, float64 NumPy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "strong" if args.split == "slices" else "weak",
        "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(workload_config(w, args.split, world), **mask_config(args)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def workload_config(w, split="replicas", world=1):
    parallelism = ("replicas (independent (b,h) slices per GPU)" if split == "replicas" else
                   f"slices ({w.B * w.H} (b,h) slices of one batch split over {world} GPU(s))")
    return {
        "workload": f"{w.name}: B={w.B} H={w.H} L={w.L} D={w.D} {w.dtype} n_buckets={w.n_buckets} "
                    f"chunk={w.chunk} n_rounds={w.n_rounds}",
        "global_batch": w.B, "seq_len": w.L, "heads": w.H, "head_dim": w.D,
        "parallelism": parallelism,
        "l2": "inputs larger than L2 (QK+V = %.1f GiB per GPU), no flush" % (2 * w.tokens * w.D * (2 if w.dtype == 'bf16' else 4) / 2**30),
    }


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, w, rank, world, local_rank):
    import dataclasses

    import torch
    import torch.distributed as dist

    import lsh_attention_hash_b200 as lsh
    from lsh_attention_hash_b200 import binding, multi, synth

    masks = mask_options(args)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w_job = w  # the whole job's workload (tokens counted for the metric)
    if args.split == "slices":
        # this rank's contiguous share of the batch's (b, h) slices, run as one B = 1 batch
        mine = multi.shard_slices(w.B, w.H, rank, world)
        if not mine:
            raise SystemExit(f"--split slices: {world} ranks for {w.B * w.H} slices")
        qk_h, v_h, R_h = synth.make_shard_inputs(w, mine, seed=0, pin=True)
        w = dataclasses.replace(w, B=1, H=len(mine))
    else:
        qk_h, v_h, R_h = synth.make_inputs(w, seed=multi.rank_seed(0, rank), pin=True)
    qk = qk_h.to(dev)
    v = v_h.to(dev)
    R = R_h.to(dev)
    bufs = binding.alloc_buffers(w.B, w.H, w.L, w.D, w.n_rounds, w.n_buckets, w.torch_dtype, dev)
    stream = torch.cuda.current_stream(dev)
    # stage boundaries of every timed step (read after the timed region: no host sync inside it)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(args.steps)]

    def step(ev):
        if ev:
            ev[0].record(stream)
        lsh.lsh_hash(qk, R, w.n_buckets, buckets=bufs["buckets"], with_near_tie=False, stream=stream)
        if ev:
            ev[1].record(stream)
        lsh.lsh_sort_permute(bufs["buckets"], w.n_buckets, perm=bufs["perm"], workspace=bufs["workspace"],
                             stream=stream)
        if ev:
            ev[2].record(stream)
        lsh.lsh_chunk_attend(qk, v, bufs["perm"], w.chunk, out_rounds=bufs["out_rounds"],
                             lse=bufs["lse_rounds"], buckets=bufs["buckets"], stream=stream, **masks)
        if ev:
            ev[3].record(stream)
        lsh.lsh_combine_rounds(bufs["out_rounds"], bufs["lse_rounds"], out=bufs["out"], want_lse=False,
                               stream=stream)
        if ev:
            ev[4].record(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status(stream) == 0

    stage_ms = {s: 0.0 for s in STAGES}
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    for ev in evs:
        for i, s in enumerate(STAGES):
            stage_ms[s] += ev[i].elapsed_time(ev[i + 1])
    assert lsh.lsh_get_device_status(stream) == 0

    # end to end through the public API with host buffers (lsh_attention_host): every step
    # copies its inputs from pinned memory and the merged output back, in runs of (b, h)
    # slices whose copies overlap the other runs' kernels
    out_h = torch.empty((w.B, w.H, w.L, w.D), dtype=w.torch_dtype, pin_memory=True)
    host_state = {}
    e2e_steps = max(1, min(args.steps, 3))
    lsh.lsh_attention_host(qk_h, v_h, R_h, w.n_buckets, w.chunk, out_h, groups=args.e2e_groups, stream=stream,
                           state=host_state, **masks)  # buffers and streams, outside the timed region
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for _ in range(e2e_steps):
        lsh.lsh_attention_host(qk_h, v_h, R_h, w.n_buckets, w.chunk, out_h, groups=args.e2e_groups,
                               stream=stream, state=host_state, **masks)
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)
    del host_state

    # backward of the step (optional): gradients of sum(dout * out) from the forward's merged
    # output and LSE, inputs resident; timed on its own after the forward line's region
    bwd_ms, bwd_steps = 0.0, 0
    if args.backward:
        lse_m = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
        lsh.lsh_attention(qk, v, R, w.n_buckets, w.chunk, stream=stream, bufs=dict(bufs, lse=lse_m), **masks)
        gen = torch.Generator(device=dev).manual_seed(multi.rank_seed(1, rank))
        dout = torch.randn((w.B, w.H, w.L, w.D), generator=gen, device=dev).to(w.torch_dtype)
        dqk = torch.empty((w.B, w.H, w.L, w.D), dtype=torch.float32, device=dev)
        dvv = torch.empty_like(dqk)

        def backward():
            lsh.lsh_chunk_attend_backward(qk, v, bufs["perm"], w.chunk, bufs["out"], lse_m, dout,
                                          buckets=bufs["buckets"], dqk=dqk, dv=dvv, stream=stream, **masks)

        backward()
        torch.cuda.synchronize()
        bwd_steps = max(1, min(args.steps, 3))
        b_start = torch.cuda.Event(enable_timing=True)
        b_end = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        b_start.record(stream)
        for _ in range(bwd_steps):
            backward()
        b_end.record(stream)
        torch.cuda.synchronize()
        barrier()
        assert lsh.lsh_get_device_status(stream) == 0
        bwd_ms = b_start.elapsed_time(b_end)
        del dout, dqk, dvv

    elapsed_ms, e2e_ms, bwd_ms = multi.max_over_ranks([elapsed_ms, e2e_ms, bwd_ms], device=dev)

    if rank != 0:
        return
    ms_step = elapsed_ms / args.steps
    job_tokens = w_job.tokens if args.split == "slices" else world * w.tokens
    value = job_tokens / (ms_step / 1e3)
    e2e_value = job_tokens / (e2e_ms / e2e_steps / 1e3)
    h2d = qk_h.numel() * qk_h.element_size() + v_h.numel() * v_h.element_size() + R_h.numel() * R_h.element_size()
    d2h = out_h.numel() * out_h.element_size()

    peaks, peak_src = load_peaks()
    alg = algorithmic(w)
    per_stage = {s: stage_ms[s] / args.steps for s in STAGES}
    dominant = max(per_stage, key=per_stage.get)
    bound = kernel_bound(dominant)
    t_launch = per_stage[dominant] / 1e3
    if bound == "hbm":
        achieved = alg[dominant]["bytes"] / t_launch / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    else:
        achieved = alg[dominant]["flops"] / t_launch / 1e12
        peak = peaks["bf16_tflops_sustained"]
        unit = "TFLOP/s"
    t_roof = max(alg["total_bytes"] / (peaks["hbm_gbs"] * 1e9), alg["attn_flops"] / (peaks["bf16_tflops"] * 1e12))
    # method-inclusive bound: the hash GEMM's FLOPs added to the attention FLOPs
    t_roof_hash = max(alg["total_bytes"] / (peaks["hbm_gbs"] * 1e9),
                      (alg["attn_flops"] + alg["hash"]["flops"]) / (peaks["bf16_tflops"] * 1e12))
    if w.L <= 65536 and w.n_buckets <= 1024:
        sort_launches = 1                                  # one CTA per segment
    else:
        sort_launches = 3 + (1 if w.n_buckets > 16384 else 0)  # count, scan, scatter (+ counter clear)
    launches_per_step = 3 + sort_launches                  # hash, sort, attend, combine
    sample_slices, sample_cap = cpu_sample_plan(w, 10.0)  # about 10 s of float64 CPU work
    c_secs, c_tokens, c_threads = oracle_sample(w, sample_slices, masks=masks, max_tokens=sample_cap)
    one_slices, one_cap = cpu_sample_plan(w, 6.0)
    o_secs, o_tokens, _ = oracle_sample(w, one_slices, masks=masks, threads=1, max_tokens=one_cap)

    def sample_text(slices, cap, tokens):
        if cap:
            return f"the first {cap} tokens of a (b,h) slice"
        return f"{slices} (b,h) slice(s) of the workload ({tokens} tokens)"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.split == "slices" else "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": dict(workload_config(w_job, args.split, world), **mask_config(args)),
        "roofline": {"bound": bound, "kernel": dominant, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": recorded_traffic(dominant, args.workload),
                     "peak_source": peak_src + (", sustained tensor peak" if bound == "tensor" else "")},
        "step_roofline": {"t_roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_step,
                          "t_roofline_hash_inclusive_ms": t_roof_hash * 1e3,
                          "frac_hash_inclusive": t_roof_hash * 1e3 / ms_step,
                          "alg_bytes": alg["total_bytes"], "attn_flops": alg["attn_flops"],
                          "hash_flops": alg["hash"]["flops"],
                          "note": "max(alg. bytes / HBM peak, chunk-attention FLOPs / bf16 peak) over measured step time"},
        "stage_ms": per_stage,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "api": f"lsh_attention_host: {args.e2e_groups} runs of (b, h) slices, copies overlapping kernels"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": {"value": c_tokens / c_secs, "unit": UNIT, "cores": c_threads, "kind": "oracle",
                         "affinity_cores": len(os.sched_getaffinity(0)),
                         "sample": f"{sample_text(sample_slices, sample_cap, c_tokens)}, all {w.n_rounds} rounds, "
                                   f"float64 NumPy oracle, {c_secs:.1f} s",
                         "one_core": {"value": o_tokens / o_secs, "unit": UNIT, "cores": 1,
                                      "sample": f"{sample_text(one_slices, one_cap, o_tokens)}, all {w.n_rounds} "
                                                f"rounds, BLAS pools capped at one thread, {o_secs:.1f} s"}},
    }
    if args.backward:
        b_ach = backward_flops(w) / (bwd_ms / bwd_steps / 1e3) / 1e12
        if backward_on_tensor_cores(w, args):
            b_peak, b_bound, b_unit = peaks["bf16_tflops"], "tensor", "TFLOP/s"
            b_src = peak_src + ", bf16 tensor peak (the five products run as UMMAs)"
            b_launches = (w.n_rounds + 1) * bwd_steps  # per-token terms, then one launch per round
            b_note = ("lsh_chunk_attend_backward alone (tensor cores: one per-token pass, then one launch per "
                      "round), inputs resident")
        else:
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            sm_mhz = measured_sm_max_mhz()
            b_peak, b_bound, b_unit = alu_peak_tflops(sms, sm_mhz), "alu", "TFLOP/s"
            b_src = f"FP32 FMA on the CUDA cores: {sms} SMs x 128 lanes x 2 x {sm_mhz:.0f} MHz"
            b_launches = w.n_rounds * bwd_steps
            b_note = "lsh_chunk_attend_backward alone (CUDA-core kernels, one launch per round), inputs resident"
        line["backward"] = {
            "ms": bwd_ms / bwd_steps, "value": world * w.tokens / (bwd_ms / bwd_steps / 1e3), "unit": UNIT,
            "steps": bwd_steps, "gpu_launches": b_launches,
            "roofline": {"bound": b_bound, "achieved": b_ach, "peak": b_peak, "unit": b_unit,
                         "frac": b_ach / b_peak,
                         "traffic": (recorded_traffic("backward", args.workload)
                                     if backward_on_tensor_cores(w, args) and not mask_config(args) else None),
                         "traffic_note": "DRAM bytes of one round launch (ncu, profiles/traffic.json)",
                         "peak_source": b_src},
            "note": b_note}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="64k")
    ap.add_argument("--split", choices=["replicas", "slices"], default="replicas",
                    help="N > 1: replicas (each rank its own batch) or slices (the ranks split one batch)")
    ap.add_argument("--causal", action="store_true",
                    help="causal window: keys after the query's position are masked")
    ap.add_argument("--bucket-mask", action="store_true",
                    help="keys outside the query's bucket are masked")
    ap.add_argument("--e2e-groups", type=int, default=16,
                    help="runs of (b, h) slices in the host-buffer pipeline of the e2e measurement")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward call (gradients w.r.t. the shared rows and the values)")
    ap.add_argument("--union", action="store_true",
                    help="multi-round union correction (implies --bucket-mask; CUDA-core attention path)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from lsh_attention_hash_b200 import synth

    w = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
