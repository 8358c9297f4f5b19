"""GPT-2 124M training throughput on B200 (fwd + bwd + clip + AdamW), one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload gpt2_124m|gpt2_124m_b64|wide]

Workload: GPT-2 124M (12 blocks, 12 heads, 768 channels, context 1,024,
vocabulary 50,257 padded to 50,304, tied embeddings), micro-batch 19 x 9
accumulation steps = 175,104 tokens per optimizer step, bf16 activations with
fp32 master weights, gradients and Adam state, AdamW with global-norm clip 1.0
and the warmup + cosine schedule ("Pretraining and adapting a language model
on a dependency-free stack", §4.1, §4.3, §4.4). Tokens are a synthetic
Zipf(1.1) stream with end-of-text ids at geometric(mean 1000) document
boundaries, seed 1337 (+ rank), resident in HBM before timing starts.

A step is 9 x gpt2_fwd_bwd + gpt2_clip_adamw. `value` is whole-job tokens/s
from CUDA events over exactly K steps (max over ranks). `e2e` repeats the
measurement through gpt2_train_step_host with pinned host token buffers (the
host->device copies and the loss/norm readback inside the timed region).
With --gpus N the ranks train one model data-parallel (the pages' multi-card
arrangement, §4.4): each rank takes its own micro-batches from its own token
stream and the gradients are averaged across ranks before every update
(gpt_step_b200.dp). --dp-mode zero1 (default): NCCL reduce-scatter of each
gradient bucket as soon as the last backward has finished it (overlapping the
remaining backward), the norm from a scalar all-reduce, each rank's AdamW on
its shards, NCCL all-gather of the bf16 weights; --dp-mode allreduce: one
all-reduce of the fp32 gradients and the full update on every rank. The
weights every rank computes with stay identical (checked after the timed
region). Per-rank work is fixed, so scaling is weak. --parallel replicas
instead trains N independent replicas (no exchange).

--impl reference times the CPU oracle (the fp64 numpy definition of the same
step) on the host cores on a bounded sample of the same workload.

--workload selects one of the configurations the pages' recipe is run at (the
headline is gpt2_124m): gpt2_124m_b64 is the same model at micro-batch 64 x 8
accumulation (524,288 tokens per step), followed by its held-out pass (20
batches of 64 x 1024 from a separately seeded stream, timed on its own and
reported under "eval"); wide is 16 blocks, 24 heads, 1,536 channels,
vocabulary 8,449 padded to 8,576, micro-batch 8 x 8.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "gpt2_124m"
PAGES_TOKENS_PER_S = 43374.0  # the pages' own stack, one card of their 3-card box (numbat §5.4, Table 3)
DATASHEET_BF16_TFLOPS = 2250.0   # dense bf16 per GPU, NVIDIA's figure without 2:4 sparsity


def flops_per_token(args, n_params):
    """6 N (N = parameters over the real vocabulary) + causal attention 6 L C T."""
    return 6.0 * n_params + 6.0 * args["n_layer"] * args["n_embd"] * args["seq_len"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def gemm_traffic_per_launch(name):
    """DRAM bytes (read + written) per GEMM launch, from the committed ncu launch
    list of one micro-step of this workload (profiles/launches_<name>_microstep.md),
    or None when there is none or when the kernel sources have changed since it
    was captured (the summary records their sha256)."""
    import re
    path = os.path.join(ROOT, "profiles", f"launches_{name}_microstep.md")
    if not os.path.exists(path):
        return None, "no launch list committed for this workload"
    from gpt_step_b200.profile_step import kernel_sources_sha256
    text = open(path).read()
    m = re.search(r"kernel_sources_sha256: ([0-9a-f]{64})", text)
    if not m or m.group(1) != kernel_sources_sha256():
        return None, "the kernels changed since the committed launch list was captured"
    n, b = 0, 0.0
    for line in text.splitlines():
        if line.startswith(("| `gemm2::gemm_tc2_kernel", "| `gemm::gemm_tc_kernel")):
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            n += int(cells[1])
            b += (float(cells[4]) + float(cells[5])) * 1e6
    if n == 0:
        return None, "no GEMM launches in the committed launch list"
    return b / n, (f"ncu dram__bytes_read.sum + dram__bytes_write.sum, mean over the {n} GEMM launches of "
                   f"one micro-step + optimizer step ({os.path.relpath(path, ROOT)})")


def workload_desc(w, n_gpus, parallel="dp", dp_mode="zero1", name=WORKLOAD):
    vp = (w["vocab_real"] + 127) // 128 * 128
    title = {"gpt2_124m": "GPT-2 124M", "gpt2_124m_b64": "GPT-2 124M at micro-batch 64",
             "wide": "Wider GPT-2-style"}.get(name, name)
    return {
        "workload": (f"{title} training step: L{w['n_layer']} H{w['n_head']} C{w['n_embd']} "
                     f"T{w['seq_len']} V{w['vocab_real']}->{vp}, micro-batch {w['micro_batch']} x "
                     f"{w['grad_accum']} accumulation"),
        "name": name,
        "global_batch": w["micro_batch"] * w["grad_accum"] * n_gpus,
        "seq_len": w["seq_len"],
        "tokens_per_step": w["micro_batch"] * w["grad_accum"] * w["seq_len"] * n_gpus,
        "parallelism": ("single GPU" if n_gpus == 1 else
                        (f"dp{n_gpus} (ZeRO-1: per-bucket NCCL reduce-scatter overlapped with the last backward, "
                         "sharded AdamW, bf16 all-gather)" if dp_mode == "zero1" else
                         f"dp{n_gpus} (NCCL all-reduce of the fp32 gradients per optimizer step)")
                        if parallel == "dp" else f"replicas x{n_gpus}"),
        "l2": "inputs larger than L2 (each micro-step touches ~8 GB of activations and logits)",
        "inputs": (f"synthetic Zipf(1.1) token stream, geometric({w['mean_doc_len']}) documents, "
                   "seed 1337+rank"),
    }


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * (mx or 1)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """Time the CPU oracle on a bounded sample of the workload (rank 0 only)."""
    if rank != 0:
        return
    from gpt_step_b200 import workloads
    name = args.workload
    w = workloads.WORKLOADS[name]
    res = cpu_baseline(name, target_seconds=max(10.0, 4.0 * args.steps), steps=args.steps, one_core=False)
    tokens_per_step = w["micro_batch"] * w["grad_accum"] * w["seq_len"]
    line = {
        "metric": "GPT-2 124M train tokens/s on 1 B200 (fwd+bwd+AdamW); MFU vs bf16 dense peak",
        "impl": "reference",
        "value": res["value"], "unit": "tokens/s", "n_gpus": 0, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * tokens_per_step / res["value"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_desc(w, 1, name=name),
        "cpu_baseline": res,
        "e2e": {"value": res["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        return os.cpu_count()


def cpu_baseline(name=WORKLOAD, target_seconds=15.0, steps=1, one_core=True):
    """Oracle tokens/s on the host: fwd+bwd of 1 x T tokens plus AdamW amortised over
    a full step, with all the BLAS threads the process has, and (one_core) once
    more with one thread."""
    from gpt_step_b200 import synth, workloads
    from oracle import gpt2 as G
    args = workloads.model_args(name, micro_batch=1)
    cfg = G.Config(**args)
    w = workloads.WORKLOADS[name]
    p = G.init_params(cfg, 1337)
    src = synth.TokenSource(1, cfg.T, cfg.V, 1337, w["mean_doc_len"], 8)
    t_micro = []
    t0 = time.perf_counter()
    n = 0
    while True:
        x, y = src.get()
        a = time.perf_counter()
        _, g = G.fwd_bwd(cfg, p, x, y)
        t_micro.append(time.perf_counter() - a)
        n += 1
        if n >= max(1, steps) and time.perf_counter() - t0 > 0.6 * target_seconds:
            break
        if n >= 4:
            break
    m, v = G.zeros_like_params(cfg), G.zeros_like_params(cfg)
    a = time.perf_counter()
    G.clip_adamw(cfg, p, g, m, v, 0)
    t_adam = time.perf_counter() - a
    seqs_per_step = w["micro_batch"] * w["grad_accum"]
    t_seq = statistics.median(t_micro)
    value = 1.0 / ((t_seq + t_adam / seqs_per_step) / cfg.T)
    cores = _oracle_threads()
    out = {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "omp_num_threads": os.environ.get("OMP_NUM_THREADS", "unset"),
           "host_cpus": os.cpu_count(),
           "sample": (f"{n} oracle micro-steps of 1 x {cfg.T} tokens (fwd+bwd, fp64 numpy, {cores} BLAS threads; "
                      f"median {t_seq:.2f} s) + one clip+AdamW over all parameters ({t_adam:.2f} s) "
                      f"amortised over the {seqs_per_step} sequences of a step")}
    if one_core:
        try:
            from threadpoolctl import threadpool_limits
            x, y = src.get()
            with threadpool_limits(1):
                a = time.perf_counter()
                G.fwd_bwd(cfg, p, x, y)
                t1 = time.perf_counter() - a
                a = time.perf_counter()
                G.clip_adamw(cfg, p, g, m, v, 1)
                ta1 = time.perf_counter() - a
            out["one_core"] = {"value": 1.0 / ((t1 + ta1 / seqs_per_step) / cfg.T), "unit": "tokens/s",
                               "sample": f"one micro-step of 1 x {cfg.T} tokens ({t1:.2f} s) + one AdamW "
                                         f"({ta1:.2f} s) with the BLAS pool limited to 1 thread"}
        except Exception as e:  # threadpoolctl missing: report without the one-thread figure
            out["one_core"] = {"unavailable": str(e)[:100]}
    return out


# --------------------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--parallel", default="dp", choices=["dp", "replicas"])
    ap.add_argument("--dp-mode", default="zero1", choices=["zero1", "allreduce"])
    ap.add_argument("--workload", default=WORKLOAD, choices=["gpt2_124m", "gpt2_124m_b64", "wide"])
    args = ap.parse_args()

    from gpt_step_b200.replicas import job_throughput, max_over_ranks, rank_env, replica_seed
    rank, world, local_rank = rank_env()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import gpt_step_b200 as gs
    from gpt_step_b200 import build, synth, workloads

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    build.build()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    name = args.workload
    w = workloads.WORKLOADS[name]
    B, T, A = w["micro_batch"], w["seq_len"], w["grad_accum"]
    margs = workloads.model_args(name)
    cfg = gs.Config.make(**margs)
    fpt = flops_per_token(margs, gs.num_params(cfg))
    dp_mode = args.parallel == "dp"
    # data parallel: one model (the same initial weights everywhere), per-rank data
    model = gs.GPT2(cfg, 1337 if dp_mode else replica_seed(1337, rank))
    from gpt_step_b200.dp import DataParallel
    par = DataParallel(model, mode=args.dp_mode) if dp_mode else None
    n_steps = args.warmup + args.steps
    n_win = n_steps * A * B
    src = synth.TokenSource(B, T, cfg.vocab_real, replica_seed(1337, rank), w["mean_doc_len"], n_win)
    xs, ys = [], []
    for _ in range(n_steps * A):
        x, y = src.get()
        xs.append(x)
        ys.append(y)
    tok = torch.tensor(np.stack(xs), device="cuda")     # [steps*A, B, T] resident in HBM
    tgt = torch.tensor(np.stack(ys), device="cuda")
    stream = model.stream

    def step(i, sched=None):
        # data of window block i; optimizer step index `sched` (default i)
        for a in range(A):
            j = i * A + a
            model.fwd_bwd(tok[j], tgt[j])
        if par is not None:
            par.update(i if sched is None else sched)   # exchange + (sharded) update; plain update on one rank
        else:
            model.clip_adamw(i if sched is None else sched)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i)
    barrier()
    # timed region: exactly K steps, nothing but the step inside
    launches0 = model.kernel_launches()
    clocks = ClockSampler(local_rank)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.warmup, n_steps):
        step(i)
    ev1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    launches = model.kernel_launches() - launches0
    loss, norm = model.last_step_stats()
    # an identical second pass with CUDA events around every launch group gives the
    # per-kernel-class device times behind the roofline (kept out of the headline
    # number because the extra event records cost ~1-3% of the step)
    model.profile(True)
    for i in range(args.warmup, n_steps):
        step(i, n_steps + i)
    prof = model.profile_read()
    model.profile(False)
    barrier()
    # every rank's weights must still be identical after the data-parallel steps
    agree = par.replicas_agree() if (par is not None and world > 1) else None
    t_max = max_over_ranks(ms, device="cuda")
    tokens = args.steps * A * B * T * world
    value = job_throughput(args.steps * A * B * T, world, t_max)

    # end to end through the host-buffer C-ABI call
    e2e = None
    if not args.no_e2e:
        htok = torch.empty((A, B, T), dtype=torch.int32, pin_memory=True)
        htgt = torch.empty((A, B, T), dtype=torch.int32, pin_memory=True)
        host_batches = [(np.stack(xs[i * A:(i + 1) * A]), np.stack(ys[i * A:(i + 1) * A]))
                        for i in range(args.warmup, n_steps)]
        multi = par is not None and world > 1
        if multi:   # the step needs the exchange between backward and update: dp's host path
            dtok, dtgt = torch.empty((A, B, T), dtype=torch.int32, device="cuda"), torch.empty(
                (A, B, T), dtype=torch.int32, device="cuda")
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k, (hx, hy) in enumerate(host_batches):
            htok.numpy()[...] = hx
            htgt.numpy()[...] = hy
            if multi:
                par.step_host(htok, htgt, dtok, dtgt, 2 * n_steps + k)
            else:
                model.train_step_host_ptr(htok.data_ptr(), htgt.data_ptr(), A, 2 * n_steps + k)
        e1.record(stream)
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), device="cuda")
        e2e = {"value": job_throughput(args.steps * A * B * T, world, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": 2 * A * B * T * 4, "d2h_bytes_per_step": 8,
               "api": ("DataParallel.step_host (pinned host tokens/targets, NCCL gradient average)" if multi
                       else "gpt2_train_step_host (pinned host tokens/targets)")}

    # the held-out pass of the large-micro-batch workload: 20 batches of 64 x 1024
    # from a separately seeded stream, losses only (no logits stored), timed alone
    ev = None
    if "eval_batches" in w:
        eb, nb = w["eval_batch"], w["eval_batches"]
        esrc = synth.TokenSource(eb, T, cfg.vocab_real, w["eval_seed"] + rank, w["mean_doc_len"], eb * nb)
        etok, etgt = [], []
        for _ in range(nb):
            x, y = esrc.get()
            etok.append(torch.tensor(x, device="cuda"))
            etgt.append(torch.tensor(y, device="cuda"))
        model.eval_loss(etok[0], etgt[0])          # warm-up
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        eloss = [model.eval_loss(a, b) for a, b in zip(etok, etgt)]
        e1.record(stream)
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), device="cuda")
        ev = {"batches": nb, "batch": eb, "loss": round(float(np.mean(eloss)), 5),
              "tokens_per_s": job_throughput(nb * eb * T, world, ems), "ms": round(ems, 3),
              "seed": w["eval_seed"], "note": "eval_loss per batch includes its host read of the loss"}

    peaks = load_peaks()
    roof = None
    if prof and prof.get("gemm", {}).get("ms", 0) > 0:
        g = prof["gemm"]
        ach = g["flops"] / (g["ms"] / 1000.0) / 1e12
        pk = peaks["bf16_tflops_sustained"]
        traffic, tsrc = gemm_traffic_per_launch(name)
        roof = {"bound": "tensor", "kernel": "gemm_tc2_kernel / gemm_tc_kernel (every tcgen05 GEMM launch)",
                "achieved": round(ach, 1), "peak": pk, "unit": "TFLOP/s", "frac": round(ach / pk, 4),
                "peak_kind": f"bf16 dense, sustained, {peaks['source']}",
                "traffic": None if traffic is None else round(traffic), "traffic_source": tsrc,
                "launches": g["launches"], "share_of_step": round(g["ms"] / ms, 4),
                "timing": "CUDA events around each launch in a second pass of K steps"}

    if rank == 0:
        mfu = value / world * fpt / (peaks["bf16_tflops"] * 1e12)
        line = {
            "metric": "GPT-2 124M train tokens/s on 1 B200 (fwd+bwd+AdamW); MFU vs bf16 dense peak",
            "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_max / args.steps, 3),
            "higher_is_better": True, "scaling": "weak",
            # the pages' figure is for this model at micro-batch 19 x 9 only
            "vs_baseline": round(value / PAGES_TOKENS_PER_S, 3) if name == WORKLOAD else None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_desc(w, world, args.parallel, args.dp_mode, name),
            "mfu": round(mfu, 4), "mfu_peak": f"{peaks['bf16_tflops']} TFLOP/s bf16 dense ({peaks['source']})",
            "mfu_datasheet": round(value / world * fpt / (DATASHEET_BF16_TFLOPS * 1e12), 4),
            "mfu_datasheet_peak": f"{DATASHEET_BF16_TFLOPS} TFLOP/s bf16 dense (datasheet)",
            "flops_per_token": fpt,
            "loss": round(loss, 4), "grad_norm": round(norm, 4),
            "gpu_launches": int(launches), "clocks": clk, "roofline": roof, "e2e": e2e,
            "kernels": prof,
        }
        if ev is not None:
            line["eval"] = ev
        if agree is not None:
            line["replicas_agree"] = agree
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(name)
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
