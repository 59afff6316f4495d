#!/usr/bin/env python
"""Benchmark of the fused verify-and-distill step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...     (one process per GPU, NCCL)

One step = one pass of the whole hot path over one batch: the length head (a1), then the fused
row pass (a2-a5: verification, acceptance, sampling, loss and gradient) over B = 128 sequences,
k = 16 drafts, V = 151936 (the ragged high-concurrency workload; b_k varies per sequence).  Inputs
are seeded synthetic bf16 logits resident in HBM; each step reads 1.2 GB of logits, far more
than the 126 MB L2, so no flush is needed between steps.  The timed region is bracketed by a
barrier and a device synchronize on both sides and measured with CUDA events on the launching
stream; with N GPUs every rank runs its own batch (weak scaling) and the step time is the max
over ranks.  Rank 0 prints one JSON line.

`--impl reference` times the CPU oracle (fp64, all host cores) on a bounded sample of the same
workload instead and prints the same line with "impl": "reference".

Besides the metric, the line carries the row pass's roofline, the end-to-end rate with host
buffers, the CPU oracle baseline, clocks sampled during the timed region, and the other legs of
the path timed on the same inputs: the length head and its online update, the full-k label mode,
the speedup report and one rank of the 8-way vocab-sharded pass.  `--workload` and
`--profile-head` are for profiling runs only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_decoding_verify_distill_b200 import api  # noqa: E402
from speculative_decoding_verify_distill_b200 import parallel  # noqa: E402
from speculative_decoding_verify_distill_b200 import synthetic as syn  # noqa: E402
from speculative_decoding_verify_distill_b200 import vocab_parallel  # noqa: E402

WORKLOAD = "ragged_qwen_b128"
METRIC = "verified draft tokens/s and fused-pass HBM GB/s (% of B200 peak) at B=128,k=16"
UNIT = "verified draft tokens/s"
CSRC = os.path.join(ROOT, "speculative_decoding_verify_distill_b200", "csrc")
# the sources the row-pass kernel is compiled from (its recorded DRAM traffic is tied to them)
KERNEL_SRCS = [os.path.join(CSRC, f) for f in ("verify_distill.cu", "svd_device.cuh", "svd_internal.h",
                                                "svd_head_unit.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "row_pass_kernel_ragged_qwen_b128.md")


def algorithmic_bytes(bk: np.ndarray, k: int, kt: int, V: int) -> int:
    """Bytes the row pass must move, each once: a verified row reads D and T and writes the
    gradient (6V), an unverified row is zero-filled (2V), a bonus row reads T (2V)."""
    bk = np.asarray(bk, np.int64)
    per_seq = bk * 6 * V + (k - bk) * 2 * V + (bk < kt) * 2 * V
    out = int(per_seq.sum())
    # per-sequence outputs: accept_len, n_emitted, emitted[k+1], bk, loss rows
    out += len(bk) * 4 * (3 + k + 1 + k)
    return out


def head_bytes(B: int, H: int, M: int) -> int:
    return 2 * B * H + 2 * M * H + 2 * M + 4 * M + 8 * B


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "hbm_gbs" in d:
            return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for path in KERNEL_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the row pass from the committed ncu summary, if it was taken
    on the current kernel source and on this workload; else None."""
    if workload != WORKLOAD or not os.path.exists(TRAFFIC_FILE):
        return None
    txt = open(TRAFFIC_FILE).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not h or not t or h.group(1) != kernel_hash():
        return None
    return float(t.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def build_inputs(w: syn.Workload, seed_offset: int, dev):
    wr = w.with_(seed=w.seed + seed_offset)
    D, T = syn.make_logits(wr, pin=True)
    h, W1, b1, w2, b2 = syn.make_head(wr)
    host = dict(D=D, T=T, h=h.pin_memory(), W1=W1, b1=b1, w2=w2, b2=b2)
    devd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    return wr, host, devd


def cpu_oracle_sample(w: syn.Workload, host, n_seqs: int, threads: int, target_s: float = 10.0,
                      draft=None, bk_gpu=None):
    """Times the oracle (a1..a5, fp64) on the first n_seqs sequences, repeated until about
    target_s seconds of CPU work have been timed; returns (tokens/s, info).

    The same oracle calls also count, on that sample, the boundary cases the parity readings
    exclude from exact comparison: stochastic accept tests with |u - p/q| < 1e-6, draws whose
    sample point lies within 1e-6 R of a running-sum boundary, and clip decisions within the
    fp32 band of the clip bound (entries with |d_v - c| < 2e-5 q_v (1 + |s_v|)).  With bk_gpu
    (the GPU's b_k) the counts use the lengths the GPU verified."""
    import oracle
    oracle.build()
    oracle.set_threads(threads)
    seqs = list(range(n_seqs))
    D, T = host["D"][seqs], host["T"][seqs]
    h = host["h"][seqs]
    dr = None if draft is None else draft[seqs].numpy()
    total, verified, reps = 0.0, 0, 0
    ref = None
    while total < target_s and reps < 64:
        t0 = time.perf_counter()
        _, bk, _ = oracle.length_head(h, host["W1"], host["b1"].double().numpy(), host["w2"], host["b2"], w.k)
        ref = oracle.verify(D, T, dr, bk, w.mode, w.tau, w.philox_seed, 0, seq_ids=seqs)
        oracle.distill(D, T, bk, w.lam, w.clip_c, w.tau, 1.0, want_grad=True)
        total += time.perf_counter() - t0
        verified += int(bk.sum())
        reps += 1
    bk_c = np.asarray(bk if bk_gpu is None else bk_gpu[seqs], np.int32)
    if bk_gpu is not None:
        ref = oracle.verify(D, T, dr, bk_c, w.mode, w.tau, w.philox_seed, 0, seq_ids=seqs)
    cases = {"sample": "first %d sequences, %d verified rows" % (n_seqs, int(bk_c.sum()))}
    if w.mode == 1:
        ver = np.arange(w.k)[None, :] < bk_c[:, None]
        margin = np.abs(ref["row_u"] - np.minimum(1.0, ref["row_ratio"]))
        cases["u_near_ratio"] = int((ver & (margin < 1e-6)).sum())
        draws = ref["n_emitted"] > ref["accept_len"]
        cases["sample_near_boundary"] = int((draws & (ref["fix_margin"] < 1e-6)).sum())
    else:
        cases["u_near_ratio"] = 0          # greedy: no uniform is drawn
        cases["sample_near_boundary"] = 0
    cb = oracle.clip_band(D, T, bk_c, w.clip_c, w.tau, 2e-5, want_mask=False)
    cases["clip_band_entries"] = int(cb["n_band"].sum())
    cases["clip_entries"] = int(bk_c.sum()) * w.V
    return verified / total, dict(seconds=total, verified=verified, seqs=n_seqs, reps=reps,
                                  cases=cases)


def run_reference(args, info):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if info.rank != 0:
        return
    w = syn.WORKLOADS[WORKLOAD]
    wr = w.with_()
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    # bounded sample per step: `threads` sequences (one per host core), cycling over the batch,
    # capped so the whole run stays within a few minutes
    per_step = max(1, min(threads, w.B))
    needed = (args.warmup + args.steps) * per_step
    seqs = [s % w.B for s in range(needed)]
    uniq = sorted(set(seqs))
    D, T = syn.make_logits(wr, seqs=uniq)
    h, W1, b1, w2, b2 = syn.make_head(wr)
    pos = {s: j for j, s in enumerate(uniq)}
    oracle.set_threads(threads)
    times, verified = [], 0
    for step in range(args.warmup + args.steps):
        ss = seqs[step * per_step:(step + 1) * per_step]
        idx = [pos[s] for s in ss]
        t0 = time.perf_counter()
        _, bk, _ = oracle.length_head(h[ss], W1, b1.double().numpy(), w2, b2, w.k)
        oracle.verify(D[idx], T[idx], None, bk, w.mode, w.tau, w.philox_seed, 0, seq_ids=ss)
        oracle.distill(D[idx], T[idx], bk, w.lam, w.clip_c, w.tau, 1.0, want_grad=True)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
            verified += int(bk.sum())
    total = sum(times)
    value = verified / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "k": w.k, "V": w.V, "H": w.H, "M": w.M,
                   "sample_per_step": "%d sequences" % per_step},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "%d sequences per step (of %d), fp64 oracle a1-a5 with gradient"
                                   % (per_step, w.B)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_vocab_shard(w, d, bk, bk_host, draft, P, stream, n=20):
    """One rank's calls of the P-way vocab-sharded pass over this workload's rows (rank 0's
    slice).  The other ranks' records come from one emulated step on this GPU; the two
    all-gathers between the calls (NVLink, exchange_bytes_per_rank per rank) are not timed."""
    slices = vocab_parallel.vocab_slices(w.V, P)
    shards = [api.VocabShard(d["D"][..., v0:v0 + nv].contiguous(), d["T"][..., v0:v0 + nv].contiguous(),
                             bk, V=w.V, v0=v0, P=P, rank=r, draft_tok=draft, mode=w.mode,
                             temperature=w.tau, seed=w.philox_seed, lam=w.lam, clip_c=w.clip_c)
              for r, (v0, nv) in enumerate(slices)]
    vocab_parallel.run_emulated(shards, stream)
    s0 = shards[0]
    for _ in range(3):
        s0.stats(stream)
        s0.resolve(stream)
        s0.finish(stream)
    torch.cuda.synchronize()
    if s0.device_error() != 0:
        raise SystemExit("device error in the vocab-sharded pass")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    hold_device(150.0 * n)   # the calls then run back to back on the device
    for j in range(n):
        ev[j][0].record(stream)
        s0.stats(stream)
        ev[j][1].record(stream)
        s0.resolve(stream)
        ev[j][2].record(stream)
        s0.finish(stream)
        ev[j][3].record(stream)
    torch.cuda.synchronize()
    part = [statistics.mean(ev[j][q].elapsed_time(ev[j][q + 1]) for j in range(n)) for q in range(3)]
    # the rank step as it runs: the calls back to back, no events between them (an event
    # between two launches keeps the second from starting in the first one's tail)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_device(150.0 * n)
    r0.record(stream)
    for j in range(n):
        s0.stats(stream)
        s0.resolve(stream)
        s0.finish(stream)
    r1.record(stream)
    torch.cuda.synchronize()
    rank_ms = r0.elapsed_time(r1) / n
    Vl = slices[0][1]
    alg = algorithmic_bytes(bk_host, w.k, w.kt, Vl)
    n1 = api.svd_vs_exchange_bytes(w.B, w.kt, 1)
    n2 = api.svd_vs_exchange_bytes(w.B, w.kt, 2)
    del shards, s0
    return {"P": P, "slice": Vl, "rank_step_ms": rank_ms, "stats_ms": part[0],
            "resolve_ms": part[1], "finish_ms": part[2],
            "rank_algorithmic_bytes": alg, "rank_hbm_gbs": alg / (rank_ms / 1000.0) / 1e9,
            "exchange_bytes_per_rank": n1 + n2, "launches_per_rank_step": 4,
            "note": "all-gathers not timed (one GPU)"}


def hold_device(us: float):
    """Keep the current stream busy for about `us` microseconds (a spin kernel), so that the
    launches queued behind it run back to back on the device: timing a run of short kernels
    this way measures the device, not the host's launch rate."""
    torch.cuda._sleep(int(us * 2000))   # ~2 cycles per ns at the B200's 1.965 GHz clock


def profile_head(w, dev, warmup, steps):
    """The length head and one online update of it at the workload's (B, H, M), no logits."""
    h, W1, b1, w2, b2 = (t.to(dev) if torch.is_tensor(t) else t for t in syn.make_head(w))
    ws = api.Workspace(w.B, w.k, w.k, w.M, device=dev)
    trainer = api.LengthHeadTrainer(W1, b1, w2, b2, w.B)
    label = torch.full((w.B,), 0.5, dtype=torch.float32, device=dev)
    for _ in range(warmup):
        api.svd_length_head(h, W1, b1, w2, b2, w.k, ws=ws)
        trainer.step(h, label)
    torch.cuda.synchronize()
    out = {}
    for name, fn in (("length_head_ms", lambda: api.svd_length_head(h, W1, b1, w2, b2, w.k, ws=ws)),
                     ("length_head_update_ms", lambda: trainer.step(h, label))):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_device(60.0 * steps)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / steps
    print(json.dumps({"profile": "length_head", "workload": w.name, "B": w.B, "H": w.H, "M": w.M, **out}),
          flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seqs", type=int, default=0, help="oracle sample size (0 = auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-vocab-shard", action="store_true", help="skip the vocab-sharded leg")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload (no legs for the other configs)")
    ap.add_argument("--profile-head", action="store_true",
                    help="profiling only: time the length head and its update at the workload's "
                         "shape, without logits, and print their times")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(syn.WORKLOADS),
                    help="profiling only: the reported bench line is the default workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    info = parallel.init_from_env("nccl" if torch.cuda.is_available() else "gloo")
    if args.impl == "reference":
        run_reference(args, info)
        if info.world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA path has no CPU fallback)")
    torch.cuda.set_device(info.local_rank)
    dev = torch.device("cuda", info.local_rank)
    w = syn.WORKLOADS[args.workload]
    if args.profile_head:
        profile_head(w, dev, args.warmup, args.steps)
        return
    headline = run_leg(w, args, info, dev, headline=True)
    legs = {}
    # the other configurations on one GPU only (under torchrun every rank would regenerate them)
    if not args.headline_only and info.world == 1:
        for name in ("greedy_qwen_b32", "stochastic_qwen_b64", "stress_llama_b256"):
            if name == args.workload:
                continue
            sweep = syn.STRESS_SWEEP if name == "stress_llama_b256" else None
            legs[name] = run_leg(syn.WORKLOADS[name], args, info, dev, headline=False, sweep=sweep)
    if info.rank == 0:
        line = headline
        line["legs"] = legs or None
        # the boundary cases of every workload timed, counted on its oracle sample
        cases = {args.workload: line.pop("_cases")}
        for name, leg in legs.items():
            cases[name] = leg.pop("_cases")
        line["boundary_cases"] = cases
        print(json.dumps(line), flush=True)
    if info.world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_leg(w, args, info, dev, *, headline: bool, sweep=None):
    """One workload: the fused step timed over K steps (with clocks on the headline), the row
    pass alone (roofline), the end-to-end rate with host buffers and the CPU oracle sample.
    The headline leg adds the head update, full-k mode, the speedup report and the sharded pass;
    a sweep times the step again for each (c, lambda)."""
    wr, host, d = build_inputs(w, parallel.rank_seed(0, info.rank) if info.rank else 0, dev)
    stream = torch.cuda.current_stream(dev)

    ws = api.Workspace(w.B, w.k, w.kt, w.M, device=dev)
    draft_host = None
    draft = None
    if w.mode == 1:
        draft_host = syn.sample_draft_tokens(host["D"], w.tau, 77)
        draft = draft_host.to(dev)
    head = (d["h"], d["W1"], d["b1"], d["w2"], d["b2"])
    # the product call: length head + row pass in one svd_verify_distill
    fused = api.VerifyDistill(d["D"], d["T"], head=head, draft_tok=draft, mode=w.mode,
                              temperature=w.tau, seed=w.philox_seed, lam=w.lam, clip_c=w.clip_c,
                              ws=ws)
    # the same two kernels launched separately, for per-kernel times (roofline of the row pass)
    bhat = torch.empty(w.B, dtype=torch.float32, device=dev)
    bk = fused.bk
    rows_only = api.VerifyDistill(d["D"], d["T"], bk_in=bk, draft_tok=draft, mode=w.mode,
                                  temperature=w.tau, seed=w.philox_seed, lam=w.lam,
                                  clip_c=w.clip_c, ws=ws)
    rows_only.args.bk = api._ptr(bk)   # read b_k in place: no copy

    def head_only():
        api.lib().svd_length_head(api._ptr(d["h"]), api._ptr(d["W1"]), api._ptr(d["b1"]),
                                  api._ptr(d["w2"]), float(d["b2"]), w.B, w.H, w.M, w.k, 1.0,
                                  api.BK_CEIL, api._ptr(bhat), api._ptr(bk), ws.ptr, ws.nbytes,
                                  api._stream())

    # ---------------------------------------------------------------- warm-up
    for _ in range(args.warmup):
        fused()
        head_only()
        rows_only()
    torch.cuda.synchronize()
    if api.svd_get_device_error(ws) != 0:
        raise SystemExit("device error during warm-up (%s)" % w.name)
    fused()
    torch.cuda.synchronize()
    bk_host = bk.cpu().numpy()
    # boundary cases: gamma * bhat * k within 1e-4 of an integer (ceil / floor decided by rounding)
    bhat_h = fused.bhat.cpu().double().numpy()
    bk_near = int((np.abs(bhat_h * w.k - np.round(bhat_h * w.k)) < 1e-4).sum())
    acc_host = fused.accept_len.cpu().numpy()
    ne_host = fused.n_emitted.cpu().numpy()
    # the step's speedup report (rho = 0: verification-count view of the pages' eta)
    report = api.report_dict(api.svd_speedup_report(fused.accept_len, bk, fused.n_emitted, w.k, 0.0))

    # ---------------------------------------------------------------- timed region (device)
    K = args.steps
    clocks = None if (args.no_clocks or not headline) else ClockSampler(dev.index if dev.index is not None else 0)
    if info.world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(K):
        fused()
    t_end.record(stream)
    torch.cuda.synchronize()
    # per-kernel durations: the same step as two separately timed launches
    KB = 200 if headline else 50   # separate launches for the per-kernel times (outside the timed region)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(KB)]
    for s in range(KB):
        ev[s][0].record(stream)
        head_only()
        ev[s][1].record(stream)
        rows_only()
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    clock_rec = clocks.stop() if clocks else None
    if info.world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    head_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(KB)]
    rows_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(KB)]
    ms_per_step = total_ms / K
    err = api.svd_get_device_error(ws)
    if err != 0:
        raise SystemExit("device error in the timed region (%s): %s" % (w.name, api.STATUS_NAMES.get(err)))
    vd = fused

    verified = float(bk_host.sum())
    accepted = float(acc_host.sum())
    emitted = float(ne_host.sum())
    loss = float(vd.loss_total.cpu()[0])
    red = parallel.reduce_metrics(ms_per_step, verified, accepted, emitted, loss, device=dev)
    value = red["verified"] / (red["ms"] / 1000.0)

    # ---------------------------------------------------------------- roofline of the row pass
    rows_avg_ms = statistics.mean(rows_ms)
    alg = algorithmic_bytes(bk_host, w.k, w.kt, w.V)
    achieved = alg / (rows_avg_ms / 1000.0) / 1e9
    peak, peak_kind = measured_peak()
    traffic = recorded_traffic(w.name)
    n_bonus = int((bk_host < w.kt).sum())

    extra = {}
    if headline:
        # ------------------------------------------------------------ length-head online update
        trainer = api.LengthHeadTrainer(d["W1"], d["b1"], d["w2"], d["b2"], w.B)
        label = (fused.accept_len.float() / bk.float()).contiguous()   # the proxy label a / b_k
        for _ in range(3):
            trainer.step(d["h"], label)
        torch.cuda.synchronize()
        u0 = torch.cuda.Event(enable_timing=True)
        u1 = torch.cuda.Event(enable_timing=True)
        n_upd = 50
        hold_device(60.0 * n_upd)   # the updates then run back to back on the device
        u0.record(stream)
        for _ in range(n_upd):
            trainer.step(d["h"], label)
        u1.record(stream)
        torch.cuda.synchronize()
        extra["length_head_update_ms"] = u0.elapsed_time(u1) / n_upd
        # the update right after a verification step on the same hidden states, reusing that
        # step's head forward (its pre-activations and bhat): only the backward kernel runs
        step_pre = api.VerifyDistill(d["D"], d["T"], head=trainer.head(d["h"]), draft_tok=draft,
                                     mode=w.mode, temperature=w.tau, seed=w.philox_seed,
                                     lam=w.lam, clip_c=w.clip_c, ws=ws, labels=True,
                                     head_preact=True)
        ev_u = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_upd)]
        for j in range(n_upd + 3):
            step_pre()
            if j >= 3:
                ev_u[j - 3][0].record(stream)
            trainer.step(d["h"], step_pre.label_proxy, preact=step_pre.head_preact, bhat=step_pre.bhat)
            if j >= 3:
                ev_u[j - 3][1].record(stream)
        torch.cuda.synchronize()
        extra["length_head_update_after_step_ms"] = statistics.mean(
            e[0].elapsed_time(e[1]) for e in ev_u)
        del step_pre

        # ------------------------------------------------------------ full-k label mode
        # the same step verifying and distilling all k rows (labels a/b_k and a/k both observable)
        fullk = api.VerifyDistill(d["D"], d["T"], head=head, draft_tok=draft, mode=w.mode,
                                  temperature=w.tau, seed=w.philox_seed, lam=w.lam, clip_c=w.clip_c,
                                  ws=ws, full_k=True, labels=True)
        for _ in range(3):
            fullk()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        n_fk = 20
        f0.record(stream)
        for _ in range(n_fk):
            fullk()
        f1.record(stream)
        torch.cuda.synchronize()
        fullk_ms = f0.elapsed_time(f1) / n_fk
        fullk_bytes = algorithmic_bytes(np.full(w.B, w.k, np.int64), w.k, w.kt, w.V)
        extra["full_k_step_ms"] = fullk_ms
        extra["full_k_step_hbm_gbs"] = fullk_bytes / (fullk_ms / 1000.0) / 1e9
        del fullk
        # ------------------------------------------------------------ vocab-sharded variant
        if not args.no_vocab_shard and info.world == 1:
            extra["vocab_sharded"] = time_vocab_shard(w, d, bk, bk_host, draft, 8, stream)

    # ---------------------------------------------------------------- (c, lambda) sweep
    sweep_out = None
    if sweep:
        sweep_out = []
        for c_, lam_ in sweep:
            for v_ in (fused, rows_only):
                v_.args.clip_c, v_.args.lambda_ = float(c_), float(lam_)
            for _ in range(3):
                fused()
            n_sw = min(K, 20)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(n_sw):
                fused()
            s1.record(stream)
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            for _ in range(n_sw):
                rows_only()
            r1.record(stream)
            torch.cuda.synchronize()
            if api.svd_get_device_error(ws) != 0:
                raise SystemExit("device error in the sweep (%s)" % w.name)
            rms = r0.elapsed_time(r1) / n_sw
            sweep_out.append({"clip_c": None if math.isinf(c_) else c_, "lambda": lam_,
                              "ms_per_step": s0.elapsed_time(s1) / n_sw, "row_pass_ms": rms,
                              "frac": alg / (rms / 1000.0) / 1e9 / peak})
        for v_ in (fused, rows_only):
            v_.args.clip_c, v_.args.lambda_ = float(w.clip_c), float(w.lam)

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if args.e2e_steps > 0:
        out_host = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    for n, t in (("accept_len", vd.accept_len), ("emitted", vd.emitted),
                                 ("n_emitted", vd.n_emitted), ("loss_total", vd.loss_total),
                                 ("bk", bk))}
        h2d = host["D"].numel() * 2 + host["T"].numel() * 2 + host["h"].numel() * 2
        if draft_host is not None:
            draft_pin = draft_host.pin_memory()
            h2d += draft_pin.numel() * 4
        d2h = sum(t.numel() * t.element_size() for t in out_host.values())
        if info.world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            d["D"].copy_(host["D"], non_blocking=True)
            d["T"].copy_(host["T"], non_blocking=True)
            d["h"].copy_(host["h"], non_blocking=True)
            if draft_host is not None:
                draft.copy_(draft_pin, non_blocking=True)
            vd()
            for n, t in (("accept_len", vd.accept_len), ("emitted", vd.emitted),
                         ("n_emitted", vd.n_emitted), ("loss_total", vd.loss_total), ("bk", bk)):
                out_host[n].copy_(t, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        red_e = parallel.reduce_metrics(e2e_ms, verified, accepted, emitted, loss, device=dev)
        e2e = {"value": red_e["verified"] / (red_e["ms"] / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "copied_back": "accept_len, emitted, n_emitted, loss_total, b_k; the gradient "
                              "dlogits stays on the device for the drafter's backward"}

    # ---------------------------------------------------------------- CPU oracle baseline
    cpu, cases = None, None
    if info.rank == 0 and not args.no_cpu_baseline and info.world == 1:
        threads = os.cpu_count() or 1
        nseq = args.cpu_seqs or max(4, min(w.B, 2 * threads))
        target = 10.0 if headline else 4.0
        v, ex = cpu_oracle_sample(wr, host, nseq, threads, target, draft=draft_host, bk_gpu=bk_host)
        cases = ex["cases"]
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "first %d of %d sequences x %d passes, fp64 oracle a1-a5 with gradient, "
                         "%.1f s" % (nseq, w.B, ex["reps"], ex["seconds"])}
        if headline:
            # the same sample on one host thread
            n1 = max(2, nseq // 8)
            v1, ex1 = cpu_oracle_sample(wr, host, n1, 1, target, draft=draft_host)
            cpu["single_thread"] = {"value": v1, "unit": UNIT, "cores": 1,
                                    "sample": "first %d sequences x %d passes, %.1f s"
                                              % (n1, ex1["reps"], ex1["seconds"])}
            oracle_threads_reset(threads)
    if cases is None:
        cases = {}
    cases["bk_near_integer"] = bk_near

    bk_hist = np.bincount(bk_host, minlength=w.k + 1)[1:].tolist()
    leg = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": red["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "k": w.k, "kt": w.kt, "V": w.V, "H": w.H,
                   "M": w.M, "mode": "stochastic" if w.mode == 1 else "greedy", "lambda": w.lam,
                   "clip_c": w.clip_c, "tau": w.tau,
                   "storage": "bf16 logits / bf16 gradient, fp32 arithmetic",
                   "l2": "inputs larger than L2 (%.2f GB of logits per step, no flush)"
                         % ((host["D"].numel() + host["T"].numel()) * 2 / 1e9),
                   "parallelism": "dp%d (independent batch per GPU)" % info.world},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "row_pass_kernel", "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": alg,
                     "bytes_breakdown": {"sum_bk": int(bk_host.sum()), "bonus_rows": n_bonus,
                                         "read_bytes": int(bk_host.sum()) * 4 * w.V + n_bonus * 2 * w.V,
                                         "write_bytes": w.B * w.k * 2 * w.V,
                                         "output_bytes": w.B * 4 * (3 + w.k + 1 + w.k)},
                     "avg_launch_ms": rows_avg_ms},
        "cpu_baseline": cpu,
        "e2e": e2e,
        # the row pass (with the length head inside) and the finalize pass per step, plus the
        # stochastic draw
        "gpu_launches": (3 if w.mode == 1 else 2) * K,
        "clocks": clock_rec,
        "accepted_tokens_per_s": red["accepted"] / (red["ms"] / 1000.0),
        "emitted_tokens_per_s": red["emitted"] / (red["ms"] / 1000.0),
        "step_hbm_gbs": (alg + head_bytes(w.B, w.H, w.M)) * info.world / (red["ms"] / 1000.0) / 1e9,
        "length_head_avg_ms": statistics.mean(head_ms),
        "bk_hist": bk_hist,
        "speedup_report": {k_: (None if v_ != v_ else round(v_, 6)) for k_, v_ in report.items()
                           if k_ != "alpha"},
        "_cases": cases,
    }
    if sweep_out is not None:
        leg["sweep"] = sweep_out
    leg.update(extra)
    if not headline:
        # a leg is not a bench line of its own: keep the figures, drop the contract's constants
        for key in ("metric", "unit", "n_gpus", "warmup", "higher_is_better", "scaling",
                    "vs_baseline", "data", "clocks"):
            leg.pop(key, None)
    del fused, rows_only, d, host, ws
    torch.cuda.empty_cache()
    return leg


def oracle_threads_reset(n: int) -> None:
    import oracle
    oracle.set_threads(n)


if __name__ == "__main__":
    main()
