"""Profiling driver: one training micro-step, or one GEMM shape, in isolation.

  python -m gpt_step_b200.profile_step step --workload gpt2_124m [--micro-batch B]
      Creates the model, runs one warm-up optimizer step (1 micro-step), then
      one micro-step (fwd_bwd) plus clip_adamw inside an NVTX range named
      "profiled" (use `ncu --nvtx --nvtx-include "profiled/"`), and prints the
      kernel launch count of that range and per-class event timings.

  python -m gpt_step_b200.profile_step gemm --kind fwd|dgrad|wgrad --shape M,N,K [--iters n]
      Times one tcgen05 GEMM arrangement through the op-level C ABI with CUDA
      events (bf16 inputs, fp32 accumulation) and prints TFLOP/s. M, N, K are the
      GEMM's own dimensions: output M x N, reduction K.

  python -m gpt_step_b200.profile_step attn --dir fwd|bwd --shape B,T,H [--iters n]
      Times the causal attention forward or backward (head size 64) through the
      op-level C ABI and prints TFLOP/s (causal FLOPs: the T(T+1)/2 visible pairs).

  python -m gpt_step_b200.profile_step head --shape N,C,Vp [--iters n]
      Times the tied lm_head + softmax-CE: the plain GEMM followed by the
      two-pass CE, the GEMM whose epilogue leaves the row partials followed by
      the one-pass CE (real vocabulary Vp - 47), each alone and together, and
      the logits-free loss (partials and target logit only, nothing stored),
      in milliseconds.

  python -m gpt_step_b200.profile_step bw --kernel ln_fwd|ln_bwd|ce|colsum|embed_fwd|embed_bwd --shape rows,C [--iters n]
      Times a bandwidth-bound kernel alone and prints GB/s of algorithmic bytes
      (for ce, C is the padded vocabulary and the real one is C - 47; for the
      embeddings, rows is B * 1024 tokens over a 50,257-id vocabulary).

  python -m gpt_step_b200.profile_step launches --csv LIST.csv
      Summarises an ncu launch list (the --csv log of a capture with the metrics
      gpu__time_duration.sum, dram__bytes_read.sum and dram__bytes_write.sum) as
      a markdown table per kernel: launches, total time, share, DRAM MB read and
      written. It also prints the hash of the kernel sources as they are now
      (`kernel_sources_sha256`), so that a summary records which kernels it
      describes; needs no GPU.
"""
from __future__ import annotations

import argparse
import json

import numpy as np


def run_step(args):
    import torch

    import gpt_step_b200 as gs
    from gpt_step_b200 import build, synth, workloads
    build.build()
    over = {}
    if args.micro_batch:
        over["micro_batch"] = args.micro_batch
    margs = workloads.model_args(args.workload, **over)
    w = workloads.WORKLOADS[args.workload]
    m = gs.GPT2(gs.Config.make(**margs), 1337)
    B, T, V = margs["micro_batch"], margs["seq_len"], margs["vocab_real"]
    src = synth.TokenSource(B, T, V, 1337, w["mean_doc_len"], 4 * B)
    batches = [src.get() for _ in range(2)]
    tok = [torch.tensor(x, device="cuda") for x, _ in batches]
    tgt = [torch.tensor(y, device="cuda") for _, y in batches]
    m.fwd_bwd(tok[0], tgt[0])
    m.clip_adamw(0)
    torch.cuda.synchronize()
    n0 = m.kernel_launches()
    m.profile(True)
    torch.cuda.nvtx.range_push("profiled")
    m.fwd_bwd(tok[1], tgt[1])
    m.clip_adamw(1)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    prof = m.profile_read()
    print(json.dumps({"workload": args.workload, "micro_batch": B,
                      "launches_in_range": m.kernel_launches() - n0, "classes": prof}))


def kernel_sources_sha256() -> str:
    """sha256 over the CUDA sources of the library: file names in sorted order and
    their contents with comments removed and every run of whitespace collapsed
    to one space, so that a change of comments or layout alone keeps the hash."""
    import hashlib
    import os
    import re
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            with open(os.path.join(d, name), "rb") as f:
                text = re.sub(rb"/\*.*?\*/", b" ", f.read(), flags=re.S)
                text = re.sub(rb"//[^\n]*", b" ", text)
                h.update(re.sub(rb"\s+", b" ", text).strip())
    return h.hexdigest()


def launch_table(csv_path):
    """Per-kernel (launches, microseconds, DRAM MB read, DRAM MB written) of an ncu launch list."""
    import collections
    import csv
    rows = list(csv.reader(open(csv_path)))
    hi = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    hdr, data = rows[hi], rows[hi + 1:]
    ki, mi, vi, ui, ii = (hdr.index(k) for k in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit", "ID"))
    scale_t = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3}
    scale_b = {"byte": 1e-6, "Kbyte": 1e-3, "Mbyte": 1.0, "Gbyte": 1e3}
    per = collections.OrderedDict()
    for r in data:
        if len(r) > vi:
            per.setdefault((int(r[ii]), r[ki]), {})[r[mi]] = (float(r[vi].replace(",", "")), r[ui])
    agg = collections.OrderedDict()
    for (_, k), m in sorted(per.items()):
        name = k.split("(")[0].replace("void ", "")
        a = agg.setdefault(name, [0, 0.0, 0.0, 0.0])
        t, u = m["gpu__time_duration.sum"]
        a[0] += 1
        a[1] += t * scale_t[u]
        if "dram__bytes_read.sum" in m:
            v, u = m["dram__bytes_read.sum"]
            a[2] += v * scale_b[u]
            v, u = m["dram__bytes_write.sum"]
            a[3] += v * scale_b[u]
    return agg


def run_launches(args):
    agg = launch_table(args.csv)
    tot = sum(v[1] for v in agg.values())
    print(f"kernel_sources_sha256: {kernel_sources_sha256()}\n")
    print("| kernel | launches | total us | share | DRAM read MB | DRAM write MB |")
    print("|---|---:|---:|---:|---:|---:|")
    for n, v in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        print(f"| `{n}` | {v[0]} | {v[1]:.0f} | {100 * v[1] / tot:.1f}% | {v[2]:.1f} | {v[3]:.1f} |")
    print(f"| total | {sum(v[0] for v in agg.values())} | {tot:.0f} | | "
          f"{sum(v[2] for v in agg.values()):.0f} | {sum(v[3] for v in agg.values()):.0f} |")


def run_gemm(args):
    import torch

    import gpt_step_b200 as gs
    from gpt_step_b200 import build
    build.build()
    M, N, K = (int(v) for v in args.shape.split(","))
    rng = np.random.default_rng(0)
    bf = lambda *s: torch.tensor(rng.standard_normal(s).astype(np.float32) * 0.1).to(torch.bfloat16).cuda()
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    if args.kind == "fwd":
        a, b, out = bf(M, K), bf(N, K), torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        fn = lambda: gs.linear_fwd(a, b, None, None, out, err)
    elif args.kind == "dgrad":
        # din[M, N] = dout[M, K] . w[K, N]   (the op names the reduction N)
        a, b, out = bf(M, K), bf(K, N), torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        fn = lambda: gs.linear_dgrad(a, b, None, out, err)
    else:
        # dw[M, N] += dout[K, M]^T . inp[K, N]
        a, b = bf(K, M), bf(K, N)
        out = torch.zeros(M, N, device="cuda")
        fn = lambda: gs.linear_wgrad(a, b, out, err, splits=args.splits)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.iters
    tf = 2.0 * M * N * K / (ms / 1000.0) / 1e12
    print(json.dumps({"kind": args.kind, "M": M, "N": N, "K": K, "ms": ms, "tflops": tf,
                      "err": int(err.sum())}))


def run_attn(args):
    import torch

    import gpt_step_b200 as gs
    from gpt_step_b200 import build
    build.build()
    B, T, H = (int(v) for v in args.shape.split(","))
    hd = 64
    C = H * hd
    rng = np.random.default_rng(0)
    qkv = torch.tensor(rng.standard_normal((B, T, 3 * C)).astype(np.float32)).to(torch.bfloat16).cuda()
    out = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, T, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    gs.attention_fwd(qkv, out, lse, H, err)
    if args.dir == "fwd":
        fn = lambda: gs.attention_fwd(qkv, out, lse, H, err)
        flops = 2.0 * B * H * T * (T + 1) * hd   # causal: T(T+1)/2 visible pairs
    else:
        dout = torch.tensor(rng.standard_normal((B, T, C)).astype(np.float32)).to(torch.bfloat16).cuda()
        dqkv = torch.empty_like(qkv)
        ws = torch.empty(gs.attention_bwd_workspace(B, T, H, hd), dtype=torch.uint8, device="cuda")
        dbias = torch.zeros(3 * C, device="cuda")   # the model's form: the qkv bias gradient added too
        fn = lambda: gs.attention_bwd(qkv, out, dout, lse, dqkv, H, ws, err, dbias=dbias)
        flops = 5.0 * B * H * T * (T + 1) * hd
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.iters
    print(json.dumps({"dir": args.dir, "B": B, "T": T, "H": H, "ms": ms,
                      "tflops": flops / (ms / 1000.0) / 1e12, "err": int(err.sum())}))


def run_bw(args):
    """Bandwidth-bound kernels alone: LayerNorm fwd/bwd, softmax-CE (GB/s of algorithmic bytes)."""
    import torch

    import gpt_step_b200 as gs
    from gpt_step_b200 import build
    build.build()
    rows, C = (int(v) for v in args.shape.split(","))
    rng = np.random.default_rng(0)
    bf = lambda *s: torch.tensor(rng.standard_normal(s).astype(np.float32)).to(torch.bfloat16).cuda()
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    if args.kernel in ("ln_fwd", "ln_bwd"):
        x, w, b = bf(rows, C), torch.ones(C, device="cuda"), torch.zeros(C, device="cuda")
        y = torch.empty_like(x)
        mean, rstd = torch.empty(rows, device="cuda"), torch.empty(rows, device="cuda")
        gs.layernorm_fwd(x, w, b, y, mean, rstd)
        if args.kernel == "ln_fwd":
            fn = lambda: gs.layernorm_fwd(x, w, b, y, mean, rstd)
            nbytes = rows * (4.0 * C + 8)
        else:
            dy, dres = bf(rows, C), bf(rows, C)
            dx = torch.empty_like(x)
            dw, db = torch.zeros(C, device="cuda"), torch.zeros(C, device="cuda")
            # the model's form: column sums by atomics, no workspace, one launch
            fn = lambda: gs.layernorm_bwd(dy, x, mean, rstd, w, dres, dx, dw, db, None)
            nbytes = rows * (8.0 * C + 8)
    elif args.kernel in ("embed_fwd", "embed_bwd"):  # rows = B * T tokens (T = 1024), vocabulary 50,257
        T, V = 1024, 50257
        Bt = rows // T
        tok = torch.tensor(rng.integers(0, V, (Bt, T)), dtype=torch.int32, device="cuda")
        wte, wpe = bf(V + 47, C), bf(T, C)
        out = torch.empty(Bt, T, C, dtype=torch.bfloat16, device="cuda")
        if args.kernel == "embed_fwd":
            fn = lambda: gs.embedding_fwd(tok, wte, wpe, out, V, err)
            nbytes = rows * (6.0 * C + 4)
        else:
            dx = bf(Bt, T, C)
            dwte, dwpe = torch.zeros(V + 47, C, device="cuda"), torch.zeros(T, C, device="cuda")
            fn = lambda: gs.embedding_bwd(tok, dx, dwte, dwpe, V)
            nbytes = rows * (2.0 * C + 4) + 2.0 * rows * C * 4 + 8.0 * T * C
    elif args.kernel == "colsum":  # bias gradient: column sums of a rows x C bf16 matrix
        a = bf(rows, C)
        db = torch.zeros(C, device="cuda")
        fn = lambda: gs.bias_grad(a, db, None)   # the model's form (atomics, one launch)
        nbytes = rows * C * 2.0
    else:  # ce: rows x C logits (C = padded vocabulary), real vocabulary C - 47
        z0 = bf(rows, C)
        z = torch.empty_like(z0)
        t = torch.tensor(rng.integers(0, C - 47, rows), dtype=torch.int32, device="cuda")
        losses = torch.empty(rows, device="cuda")
        def fn():
            gs.softmax_ce(z, t, losses, C - 47, 1.0 / rows, err)
        nbytes = rows * C * 4.0
        z.copy_(z0)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.iters
    print(json.dumps({"kernel": args.kernel, "rows": rows, "C": C, "us": ms * 1000,
                      "gbs": nbytes / (ms / 1000.0) / 1e9}))


def _time(fn, iters):
    import torch
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def run_head(args):
    import torch

    import gpt_step_b200 as gs
    from gpt_step_b200 import build
    build.build()
    N, C, Vp = (int(v) for v in args.shape.split(","))
    V = Vp - 47
    rng = np.random.default_rng(0)
    bf = lambda s, sc: torch.tensor(rng.standard_normal(s).astype(np.float32) * sc).to(torch.bfloat16).cuda()
    h, w = bf((N, C), 1.0), bf((Vp, C), 0.05)
    t = torch.tensor(rng.integers(0, V, N), dtype=torch.int32, device="cuda")
    logits = torch.empty(N, Vp, dtype=torch.bfloat16, device="cuda")
    losses = torch.empty(N, device="cuda")
    ws = torch.empty(gs.lm_head_ce_workspace(N, Vp), dtype=torch.uint8, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    gemm = lambda: gs.linear_fwd(h, w, None, None, logits, err)
    ce2 = lambda: gs.softmax_ce(logits, t, losses, V, 1.0 / N, err)
    out = {"N": N, "C": C, "Vp": Vp}
    out["gemm_store_ms"] = _time(gemm, args.iters)
    out["gemm_lse_plus_loss_only_ms"] = _time(
        lambda: gs.lm_head_ce(h, w, t, logits, losses, V, 1.0 / N, False, ws, err), args.iters)
    # logits never stored: the GEMM keeps the row partials and the target logit only
    out["logits_free_loss_ms"] = _time(lambda: gs.lm_head_loss(h, w, t, losses, V, ws, err), args.iters)
    out["ce_two_pass_ms"] = _time(lambda: (gemm(), ce2()), args.iters) - out["gemm_store_ms"]
    out["unfused_total_ms"] = out["gemm_store_ms"] + out["ce_two_pass_ms"]
    out["fused_total_ms"] = _time(lambda: gs.lm_head_ce(h, w, t, logits, losses, V, 1.0 / N, True, ws, err),
                                  args.iters)
    out["err"] = int(err.sum())
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="mode", required=True)
    s = sub.add_parser("step")
    s.add_argument("--workload", default="gpt2_124m")
    s.add_argument("--micro-batch", type=int, default=0)
    g = sub.add_parser("gemm")
    g.add_argument("--kind", choices=["fwd", "dgrad", "wgrad"], default="fwd")
    g.add_argument("--shape", default="19456,3072,768")
    g.add_argument("--iters", type=int, default=20)
    g.add_argument("--splits", type=int, default=0)
    a = sub.add_parser("attn")
    a.add_argument("--dir", choices=["fwd", "bwd"], default="fwd")
    a.add_argument("--shape", default="19,1024,12")
    a.add_argument("--iters", type=int, default=20)
    hp = sub.add_parser("head")
    hp.add_argument("--shape", default="19456,768,50304")
    hp.add_argument("--iters", type=int, default=20)
    w = sub.add_parser("bw")
    w.add_argument("--kernel", choices=["ln_fwd", "ln_bwd", "ce", "colsum", "embed_fwd", "embed_bwd"],
                   default="ln_fwd")
    w.add_argument("--shape", default="19456,768")
    w.add_argument("--iters", type=int, default=20)
    ls = sub.add_parser("launches")
    ls.add_argument("--csv", required=True)
    args = ap.parse_args()
    {"step": run_step, "gemm": run_gemm, "attn": run_attn, "bw": run_bw, "head": run_head,
     "launches": run_launches}[args.mode](args)


if __name__ == "__main__":
    main()
