#!/usr/bin/env python
"""Throughput of one GPT-2 pretraining step (forward, backward, global-norm
clip, AdamW) on B200, as training tokens/s and MFU.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...     # the CPU oracle, bounded sample

Default workload: GPT-2 124M (L12 H12 C768, V 50257 padded to 50304, Tmax
1024), B=16 x T=1024 tokens per step, AdamW lr 6e-4 with the 715-step warmup
and cosine schedule, clip 1.0, on a seeded synthetic Zipf(1.1) token stream
(the pages train on FineWeb; no dataset is available here).

For N > 1 (torchrun) every rank runs its own independent replica of the
one-GPU step on its own GPU (the step has no data-path collective); the
value is all ranks' tokens over the slowest rank's device time.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from transformer_lm_pretraining_b200.inputs import ZipfStream, iid_batch  # noqa: E402
from transformer_lm_pretraining_b200.workloads import WORKLOADS  # noqa: E402

PAGES_A100_TOK_S = 16384 / 0.090  # 90 ms per 16x1024 step on 1x A100 SXM 80GB (pages)
SPEC_BF16_DENSE = 2.25e15

# DRAM bytes (read + write) per GEMM launch, averaged over the 147 GEMM
# launches of a gpt2_124m step: each of the step's 15 products captured alone
# at full size, one launch, with ncu's dram__bytes_read.sum +
# dram__bytes_write.sum, weighted by its launches per step
# (profiles/gemm_tc_dram_traffic_gpt2_124m_step.md).  Valid only for the GEMM
# sources it was taken on: reported as null as soon as their hash differs
# (as now: the weight gradients of W_qkv and W_o share one launch since).
GEMM_TRAFFIC = {"bytes_per_launch": 1.6110e8,
                "sources_sha256": "cd62971bde99c52b228bceb93b3b1960d24e535520c1756bfeb342452fa0cfdb"}
GEMM_SOURCES = ("gemm_tc.cu", "gemm_epi.cuh", "tc_util.cuh")


def gemm_traffic(workload):
    import hashlib

    if workload != "gpt2_124m":
        return None
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(HERE, "transformer_lm_pretraining_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return GEMM_TRAFFIC["bytes_per_launch"] if h.hexdigest() == GEMM_TRAFFIC["sources_sha256"] else None


def load_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "power.limit")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                lim = float(parts[9]) if len(parts) > 9 else float("nan")
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9], lim))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "power_limit_w": rows[-1][4],
                "samples": len(loaded), "reasons": reasons}


def make_batches(wl, n_steps, seed):
    """Host token batches for n_steps optimizer steps: [step][micro] -> (tok, tgt)."""
    out = []
    if wl.iid:
        for k in range(n_steps):
            out.append([iid_batch(wl.V, wl.B, wl.T, seed + 1000 * k + j) for j in range(wl.n_micro)])
        return out
    s = ZipfStream(wl.V, seed)
    for _ in range(n_steps):
        out.append([s.next_batch(wl.B, wl.T) for _ in range(wl.n_micro)])
    return out


def metric_name(wl, mode="train"):
    """The metric string both arms print for a workload (so that the two
    lines can be compared)."""
    kind = "evaluation" if mode == "eval" else "training"
    if wl.name == "gpt2_124m":
        return f"{kind} tokens/sec and MFU, GPT-2 124M bf16, B=16×T=1024, 1×B200"
    return f"{kind} tokens/s and MFU, {wl.name} bf16"


def _oracle_row_and_opt(wl, T, openmp):
    """Time the fp32 oracle on one B=1 x T micro-batch forward+backward, and
    on one clip + AdamW over every parameter.  Returns (t_row, t_opt,
    threads, num_params)."""
    import oracle

    cfg = oracle.Config(wl.L, wl.H, wl.C, wl.V, wl.Vp, wl.Tmax)
    o = oracle.Oracle(cfg, np.float32, openmp=openmp)
    p = o.init(0)
    tok, tgt = ZipfStream(wl.V, 0).next_batch(1, T)
    m, v = np.zeros_like(p), np.zeros_like(p)
    t0 = time.perf_counter()
    _, g, _ = o.forward_backward(p, tok, tgt, 1, T, 1.0)
    t1 = time.perf_counter()
    o.clip(g, 1.0)
    o.adamw(p, g, m, v, 1, wl.lr_max)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, (oracle.openmp_threads() if openmp else 1), o.num_params()


def cpu_baseline(wl, sample_T_1core=64):
    """The oracle as it stands on the host cores, on a bounded sample of the
    workload, scaled to one optimizer step of it.

    All cores (the OpenMP build, which parallelises only over independent
    outputs): one full-length B=1 x T row forward+backward and one clip +
    AdamW over every parameter; the step is B*n_micro rows + one clip/AdamW.
    One core (the single-threaded build): a B=1 x sample_T_1core row and the
    clip/AdamW, the row scaled to full length by its FLOP count (6N + 6LCT
    per token, N = 12LC^2 + Vpad C)."""
    rows = wl.B * wl.n_micro
    t_row, t_opt, threads, P = _oracle_row_and_opt(wl, wl.T, True)
    step = rows * t_row + t_opt
    out = {"value": wl.tokens_per_step / step, "unit": "tokens/s", "cores": threads,
           "kind": "oracle",
           "sample": f"fp32 oracle (OpenMP, {threads} threads), {wl.name}: one B=1 x T={wl.T} row "
                     f"forward+backward {t_row:.2f} s and one clip + AdamW over {P} params "
                     f"{t_opt:.2f} s, step extrapolated as {rows} rows + 1 optimizer update = "
                     f"{step:.1f} s"}
    Ts = min(sample_T_1core, wl.T)
    t_row1, t_opt1, _, _ = _oracle_row_and_opt(wl, Ts, False)
    n_mm = 12 * wl.L * wl.C ** 2 + wl.Vp * wl.C

    def row_flops(T):
        return T * (6.0 * n_mm + 6.0 * wl.L * wl.C * T)

    step1 = rows * t_row1 * row_flops(wl.T) / row_flops(Ts) + t_opt1
    out["value_1core"] = wl.tokens_per_step / step1
    out["sample_1core"] = (f"single-threaded fp32 oracle: one B=1 x T={Ts} row forward+backward "
                           f"{t_row1:.2f} s, scaled by FLOP count to a T={wl.T} row, x {rows} rows, "
                           f"+ clip/AdamW {t_opt1:.2f} s = {step1:.0f} s per step (extrapolated)")
    return out


def family_roofline(wl, fam, peaks, distinct_ids, recompute):
    """Per kernel family of one optimizer step: device time, algorithmic
    work and the fraction of the measured peak it reaches.  fam = {family:
    (ms per step, launches per step, flops per step)} from the profiling
    pass.  Algorithmic bytes (bf16 activations, fp32 statistics and
    parameters), per micro-batch of M = B*T tokens unless stated:
      encoder     M(6C + 8) forward + M 2C + (T + distinct ids) 8C backward
      ln_fwd      (2L + 1) M (4C + 8)
      ln_bwd      (2L + 1) M (8C + 8)
      classifier  M (4 Vpad + 8)
      colsum      L M 2 3C + L (M/32) 4C 4   (the bias gradient of W_qkv, a pass
                  over dqkv; that of W_fc, the reduction of the per-32-row
                  sums the GELU-backward GEMM's epilogue writes)
      recompute   L M 4C 4          (read u, write GELU(u))
      optimizer   34 bytes per parameter per step (norm: 4; AdamW: 30)
    gemm and attention are tensor-bound: their algorithmic FLOPs come from
    the profiling pass (2MNK per GEMM; causal 4 B H T(T+1)/2 hd forward and
    10 B H T(T+1)/2 hd backward)."""
    L, C, Vp, T = wl.L, wl.C, wl.Vp, wl.T
    M = wl.B * wl.T
    nm = wl.n_micro
    P = 12 * L * C * C + 13 * L * C + 2 * C + Vp * C + wl.Tmax * C
    hbm = {
        "encoder": nm * (M * (6 * C + 8) + M * 2 * C + (T + distinct_ids) * 8 * C),
        "ln_fwd": nm * (2 * L + 1) * M * (4 * C + 8),
        "ln_bwd": nm * (2 * L + 1) * M * (8 * C + 8),
        "classifier": nm * M * (4 * Vp + 8),
        "colsum": nm * L * (M * 2 * 3 * C + ((M + 31) // 32) * 4 * C * 4),
        "recompute": nm * L * M * 4 * C * 4 if recompute else 0,
        "optimizer": 34 * P,
    }
    out = {}
    for k, (ms, n, fl) in fam.items():
        if ms <= 0:
            continue
        if k in hbm:
            ach = hbm[k] / (ms / 1e3) / 1e9
            out[k] = {"ms": round(ms, 4), "launches": n, "bound": "hbm",
                      "algorithmic": hbm[k], "unit": "GB/s", "achieved": round(ach, 1),
                      "peak": peaks["hbm_gbs"], "frac": round(ach / peaks["hbm_gbs"], 3)}
        else:
            ach = fl / (ms / 1e3) / 1e12
            out[k] = {"ms": round(ms, 4), "launches": n, "bound": "tensor",
                      "algorithmic": fl, "unit": "TFLOP/s", "achieved": round(ach, 1),
                      "peak": peaks["bf16_tflops_sustained"],
                      "frac": round(ach / peaks["bf16_tflops_sustained"], 3)}
    return out


def run_reference(args, wl):
    """Reference arm: the CPU oracle as it stands, timed on the host cores,
    each step a bounded sample (B=1 x T=32 micro-batch + full AdamW)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle

    cfg = oracle.Config(wl.L, wl.H, wl.C, wl.V, wl.Vp, wl.Tmax)
    o = oracle.Oracle(cfg, np.float32, openmp=True)
    p = o.init(0)
    m, v = np.zeros_like(p), np.zeros_like(p)
    T = min(32, wl.T)
    s = ZipfStream(wl.V, 0)
    times = []
    for k in range(args.warmup + args.steps):
        tok, tgt = s.next_batch(1, T)
        t0 = time.perf_counter()
        _, g, _ = o.forward_backward(p, tok, tgt, 1, T, 1.0)
        o.clip(g, 1.0)
        o.adamw(p, g, m, v, k + 1, wl.lr_max)
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = T * len(times) / tot
    return {"impl": "reference", "metric": metric_name(wl, args.mode),
            "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "sample_B": 1, "sample_T": T},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.openmp_threads(),
                             "kind": "oracle",
                             "sample": f"B=1 x T={T} micro-batch forward+backward + clip + AdamW "
                                       f"over all params per step, fp32 oracle, OpenMP"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_ours(args, wl):
    import torch

    from transformer_lm_pretraining_b200 import gpt2 as g2
    from transformer_lm_pretraining_b200.replicas import Replicas

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    reps = Replicas("nccl", timeout_s=120, group=args.mode in ("dp", "zero1"))
    world, rank, local = reps.world, reps.rank, reps.local_rank
    barrier, max_over_ranks = reps.barrier, reps.max

    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    g2.gpt2k_set_programmatic_launch(args.pdl)
    model = g2.GPT2(wl.L, wl.H, wl.C, wl.V, wl.Vp, wl.Tmax, seed=0, precision="bf16",
                    B=wl.B, T=wl.T, recompute=args.recompute)
    evaluate = args.mode == "eval"
    model.set_stream(stream)
    n_steps = args.warmup + args.steps
    host = make_batches(wl, n_steps, seed=reps.data_seed(1))
    # inputs resident in HBM before the timed region
    dev = [[(torch.from_numpy(t).cuda(), torch.from_numpy(y).cuda()) for t, y in st] for st in host]
    scale = 1.0 / wl.n_micro

    def lr(k):
        return g2.gpt2_lr(k, wl.lr_max, 0.1 * wl.lr_max, wl.warmup, wl.max_steps)

    dp_step = None
    if args.mode in ("dp", "zero1"):
        # data-parallel step: each rank its own micro-batches, gradients
        # summed over NCCL (per layer, overlapped with the backward) or
        # reduce-scattered with a sharded AdamW and an all-gather (ZeRO-1)
        import torch.distributed as dist

        from transformer_lm_pretraining_b200.data_parallel import DataParallelStep

        dp_step = DataParallelStep(
            model, world, rank, mode="zero1" if args.mode == "zero1" else "allreduce",
            overlap=args.mode == "dp", sync=False,
            all_reduce=lambda t: dist.all_reduce(t),
            reduce_scatter=lambda out, t: dist.reduce_scatter_tensor(out, t),
            all_gather=lambda out, shard: dist.all_gather_into_tensor(out, shard))

    def step(k, batches):
        if evaluate:  # forward-only evaluation: loss of every micro-batch
            for tok, tgt in batches:
                model.evaluate(tok, tgt, sync_loss=False)
            return
        if dp_step is not None:
            dp_step(batches, lr(k), 1.0, 0.9, 0.95, 1e-8, 0.1)
            return
        model.zero_grad()
        for tok, tgt in batches:
            model.forward(tok, tgt, sync_loss=False)
            model.backward(scale)
        model.grad_norm_clip(1.0, sync=False)
        model.adamw_step(lr(k), 0.9, 0.95, 1e-8, 0.1)

    for k in range(args.warmup):
        step(k, dev[k])
    torch.cuda.synchronize()

    # The training step as one CUDA graph (gpt2_step_graph_capture): its token
    # buffers receive each step's micro-batches, then the graph is replayed;
    # the learning rate follows the schedule from the device step counter.
    use_graph = args.graph and args.mode == "train"
    graph_kernels = None
    if use_graph:
        n_tok = wl.n_micro * wl.B * wl.T
        stok = torch.empty(n_tok, dtype=torch.int32, device="cuda")
        stgt = torch.empty(n_tok, dtype=torch.int32, device="cuda")
        graph_kernels = model.capture_step(stok, stgt, wl.B, wl.T, wl.n_micro, 1.0, wl.lr_max,
                                           0.1 * wl.lr_max, wl.warmup, wl.max_steps)

        def load_tokens(batches):
            for j, (t, y) in enumerate(batches):
                stok[j * wl.B * wl.T:(j + 1) * wl.B * wl.T].copy_(t.view(-1), non_blocking=True)
                stgt[j * wl.B * wl.T:(j + 1) * wl.B * wl.T].copy_(y.view(-1), non_blocking=True)

        def timed_step(k, batches):
            load_tokens(batches)
            model.launch_step()
    else:
        timed_step = step
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    n0 = g2.gpt2_launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for k in range(args.warmup, n_steps):
        timed_step(k, dev[k])
    ev1.record(stream)
    torch.cuda.synchronize()
    launches = graph_kernels if use_graph else (g2.gpt2_launch_count() - n0) // args.steps
    clk = clocks.stop()
    barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1))

    # per-kernel-family device time: a second timed pass over the same
    # batches with CUDA events around every launch on the step's stream
    # (kept out of the headline loop, whose time the events would inflate)
    n_prof = min(args.steps, 20)
    torch.cuda.synchronize()
    model.profile_enable(True)
    for k in range(args.warmup, args.warmup + n_prof):
        step(k, dev[k])
    torch.cuda.synchronize()
    prof = model.profile_read()
    model.profile_enable(False)
    ms_step = ms_total / args.steps
    value = reps.throughput(wl.tokens_per_step * args.steps, ms_total)

    # end to end through the public API: pinned host inputs copied in and the
    # loss read back every step
    e2e = None
    if not args.no_e2e:
        pinned = [[(torch.from_numpy(t).pin_memory(), torch.from_numpy(y).pin_memory()) for t, y in st]
                  for st in host]
        bufs = [(torch.empty_like(a[0][0], device="cuda"), torch.empty_like(a[0][1], device="cuda"))
                for a in [pinned[0]] * wl.n_micro]
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = args.steps
        e0.record(stream)
        for k in range(n_e2e):
            hb = pinned[(args.warmup + k) % n_steps]
            if use_graph:  # pinned host tokens into the graph's buffers, replay, loss back
                load_tokens(hb)
                model.launch_step()
                model.read_loss()
                continue
            if dp_step is not None:
                for j, (t, y) in enumerate(hb):
                    bufs[j][0].copy_(t, non_blocking=True)
                    bufs[j][1].copy_(y, non_blocking=True)
                dp_step([(bufs[j][0], bufs[j][1]) for j in range(wl.n_micro)],
                        lr(args.warmup + k), 1.0, 0.9, 0.95, 1e-8, 0.1)
                model.read_loss()
                continue
            if not evaluate:
                model.zero_grad()
            for j, (t, y) in enumerate(hb):
                bufs[j][0].copy_(t, non_blocking=True)
                bufs[j][1].copy_(y, non_blocking=True)
                if evaluate:
                    model.evaluate(bufs[j][0], bufs[j][1], sync_loss=False)
                else:
                    model.forward(bufs[j][0], bufs[j][1], sync_loss=False)
                    model.backward(scale)
            if not evaluate:
                model.grad_norm_clip(1.0, sync=False)
                model.adamw_step(lr(args.warmup + k), 0.9, 0.95, 1e-8, 0.1)
            model.read_loss()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1))
        e2e = {"value": reps.throughput(wl.tokens_per_step * n_e2e, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": 2 * 4 * wl.B * wl.T * wl.n_micro, "d2h_bytes_per_step": 4}

    # a step that produced a non-finite loss or gradient norm measured nothing
    # (AdamW leaves the parameters alone on a non-finite norm, which would
    # make such a step look fast): one more step, read back and checked
    chk = dev[args.warmup]
    if not evaluate:
        model.zero_grad()
    for tok, tgt in chk:
        if evaluate:
            model.evaluate(tok, tgt, sync_loss=False)
        else:
            model.forward(tok, tgt, sync_loss=False)
            model.backward(scale)
    chk_norm = 0.0 if evaluate else model.grad_norm_clip(1.0)
    chk_loss = model.read_loss()
    if not (math.isfinite(chk_loss) and math.isfinite(chk_norm)):
        print(f"bench: non-finite step (loss {chk_loss}, gradient norm {chk_norm}); no number reported",
              file=sys.stderr)
        sys.exit(3)

    peaks = load_peaks()
    fpt = wl.flops_per_token() / (3.0 if evaluate else 1.0)  # the forward is a third
    mfu_spec = fpt * value / world / SPEC_BF16_DENSE
    peak_mfu = peaks["bf16_tflops"] * 1e12 if peaks["source"] == "measured" else SPEC_BF16_DENSE
    mfu = fpt * value / world / peak_mfu
    gemm_ms, gemm_n, gemm_fl = prof["gemm"]
    achieved = gemm_fl / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    fam_ms = {k: v[0] / n_prof for k, v in prof.items()}
    distinct = float(np.mean([len(np.unique(t)) for st in host[args.warmup:] for t, _ in st]))
    fam_roof = family_roofline(wl, {k: (v[0] / n_prof, v[1] / n_prof, v[2] / n_prof)
                                    for k, v in prof.items()}, peaks, distinct, args.recompute)
    fam_total = sum(fam_ms.values())
    out = {
        "metric": metric_name(wl, args.mode),
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": value / PAGES_A100_TOK_S if wl.name == "gpt2_124m" and not evaluate else None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": wl.B * wl.n_micro * world, "seq_len": wl.T,
                   "micro_batch": wl.B, "n_micro": wl.n_micro,
                   "tokens_per_step": wl.tokens_per_step * world,
                   "parallelism": ({"dp": f"dp{world} (per-layer all-reduce overlapped with "
                                          "the backward)",
                                    "zero1": f"dp{world} ZeRO-1"}.get(args.mode)
                                   or ("replicas" if world > 1 else "single-gpu")),
                   "mode": args.mode, "recompute": args.recompute,
                   "cuda_graph": bool(use_graph),
                   "programmatic_launch": bool(args.pdl),
                   "l2": "no explicit flush: every step streams ~10 GB of activations, logits and "
                         "optimizer state through HBM, far above the 126 MB L2"},
        "mfu": mfu,
        "mfu_spec": mfu_spec,
        "mfu_basis": f"{fpt / 1e6:.2f} MFLOP/token ({'2N + 2LCT' if evaluate else '6N + 6LCT'}, "
                     f"N = 12LC^2 + Vpad C); mfu over "
                     + (f"the measured dense bf16 burst peak {peaks['bf16_tflops']:.0f} TFLOP/s"
                        if peaks["source"] == "measured" else "the 2.25 PFLOP/s dense bf16 spec "
                        "(no measured peak on this box)")
                     + "; mfu_spec over the 2.25 PFLOP/s dense bf16 spec",
        "gpu_launches": int(launches),
        "roofline": {"kernel": "gemm_tc_kernel (all projection GEMM launches of a step)",
                     "bound": "tensor", "achieved": achieved,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops_sustained"] if achieved else None,
                     "peak_source": f"{peaks['source']} sustained bf16",
                     "launches_per_step": gemm_n / n_prof,
                     "timing": f"CUDA events around each GEMM launch on the step's stream, "
                               f"second timed pass of {n_prof} steps",
                     "traffic": gemm_traffic(wl.name),
                     "traffic_unit": "bytes per launch (ncu dram read + write, averaged over the "
                                     "step's GEMM launches)"},
        "kernel_breakdown_ms_per_step": {k: round(v, 4) for k, v in fam_ms.items()},
        "kernel_breakdown_share": {k: round(v / fam_total, 4) for k, v in fam_ms.items()}
        if fam_total > 0 else None,
        "kernel_roofline": fam_roof,
        "kernel_roofline_basis": "device time per family from CUDA events around its launches "
                                 "(second pass); HBM families against the measured copy bandwidth, "
                                 "tensor families against the sustained bf16 peak",
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not evaluate:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_sample_T)
    reps.close()
    model.close()
    return out if reps.is_root else None


def run_generate(args, wl):
    """Autoregressive generation with the key/value cache: B sequences, a
    prompt of T/8 tokens, generated to T/4 (both from the workload's T);
    tokens/s = B * new tokens / device time of one gpt2_generate call."""
    import torch

    from transformer_lm_pretraining_b200 import gpt2 as g2
    from transformer_lm_pretraining_b200.replicas import Replicas

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    reps = Replicas("nccl", timeout_s=120)
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    Tp, Ttot = max(1, wl.T // 8), max(2, wl.T // 4)
    model = g2.GPT2(wl.L, wl.H, wl.C, wl.V, wl.Vp, wl.Tmax, seed=0, precision="bf16", B=wl.B, T=Tp)
    model.set_stream(stream)
    prompt = ZipfStream(wl.V, reps.data_seed(1)).next_batch(wl.B, Tp)[0]
    tok = torch.zeros((wl.B, Ttot), dtype=torch.int32, device="cuda")
    tok[:, :Tp] = torch.from_numpy(prompt).cuda()
    for _ in range(args.warmup):
        model.generate(tok, Tp, 0.8, 40, 7)
    torch.cuda.synchronize()
    reps.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(reps.local_rank)
    clocks.start()
    n0 = g2.gpt2_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        model.generate(tok, Tp, 0.8, 40, 7 + k)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    reps.barrier()
    ms_total = reps.max(e0.elapsed_time(e1))
    ms = ms_total / args.steps
    new = Ttot - Tp
    value = reps.throughput(wl.B * new * args.steps, ms_total)
    launches = (g2.gpt2_launch_count() - n0) // args.steps
    # each decode step streams the bf16 weights once plus the cached keys
    # and values of the positions so far (prefill excluded from the bytes)
    peaks = load_peaks()
    w_bytes = 2.0 * model.P
    kv_bytes = 2.0 * wl.L * wl.B * 2 * wl.C * sum(range(Tp + 1, Ttot))
    step_ms = ms / new
    achieved = (w_bytes * (new - 1) + kv_bytes) / (ms / 1e3) / 1e9
    reps.close()
    model.close()
    if not reps.is_root:
        return None
    return {"metric": f"generation tokens/s (key/value cache), {wl.name} bf16",
            "value": value, "unit": "tokens/s", "n_gpus": reps.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.B, "prompt": Tp, "total": Ttot,
                       "temperature": 0.8, "top_k": 40, "mode": "generate",
                       "l2": "weights (249 MB) stream through HBM every decode step, above L2"},
            "gpu_launches": int(launches),
            "roofline": {"kernel": "whole decode step (weights + key/value cache per step)",
                         "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "peak_source": peaks["source"], "traffic": None},
            "clocks": clk}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gpt2_124m", choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-T", type=int, default=64,
                    help="row length of the single-threaded oracle sample")
    ap.add_argument("--mode", default="train", choices=["train", "eval", "generate", "dp", "zero1"],
                    help="train: the training step; eval: forward-only evaluation (loss); "
                         "generate: autoregressive generation with the key/value cache; "
                         "dp: data-parallel step over the ranks (NCCL all-reduce per layer, "
                         "overlapped with the backward); zero1: data-parallel with the "
                         "optimizer sharded (reduce-scatter, AdamW on a shard, all-gather)")
    ap.add_argument("--graph", type=int, default=1, choices=[0, 1],
                    help="1: time the training step replayed as one captured CUDA graph; "
                         "0: the eager calls")
    ap.add_argument("--pdl", type=int, default=1, choices=[0, 1],
                    help="1: kernels launched with programmatic dependent launch (the "
                         "library's default); 0: plain launches")
    ap.add_argument("--recompute", type=int, default=0, choices=[0, 1],
                    help="1: recompute GELU in the backward instead of keeping it")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        out = run_reference(args, wl)
    elif args.mode == "generate":
        out = run_generate(args, wl)
    else:
        out = run_ours(args, wl)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
