"""The small configuration's 20-step loss curve against the oracle.

Small GPT-2 (6 blocks, 12 heads, 384 channels, T 1024, vocabulary 4,353 padded
to 4,480), micro-batch 16, 20 optimizer steps with warmup 5 on the Zipf
document stream (seed 1337): the loss and the pre-clip gradient norm of every
step against the oracle's, which runs the 16 sequences of each step in a pool
of CPU processes (the mean-loss gradient of the micro-batch is the mean of the
single-sequence gradients) and takes the same clipped AdamW step.

The oracle needs about 320 sequence passes here, minutes of CPU time, so this
test runs only with GPT2_RUN_SLOW=1 in the environment.
"""
import math
import multiprocessing as mp
import os

import numpy as np
import pytest

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

RUN = os.environ.get("GPT2_RUN_SLOW") == "1"

_W = {}


def _views(buf, shapes):
    out, o = {}, 0
    for name, shape in shapes:
        n = int(np.prod(shape))
        out[name] = buf[o:o + n].reshape(shape)
        o += n
    return out


def _worker_init(args, ppath, gpath, total):
    from oracle import gpt2 as G
    cfg = G.Config(**args)
    shapes = [(k, s) for k, s, _ in G.param_shapes(cfg)]
    _W.update(cfg=cfg, shapes=shapes, ppath=ppath, gpath=gpath, total=total)


def _chunk_grad(task):
    """Sequences [a, b) of the step: the oracle's summed gradient into slot `slot` of
    the shared gradient file; returns the summed loss."""
    from oracle import gpt2 as G
    slot, x, y = task
    p = _views(np.memmap(_W["ppath"], np.float64, "r", shape=(_W["total"],)), _W["shapes"])
    p = {k: np.array(v) for k, v in p.items()}
    out = np.memmap(_W["gpath"], np.float64, "r+", shape=(_W["total"],), offset=slot * _W["total"] * 8)
    g_all = None
    loss = 0.0
    for b in range(x.shape[0]):
        lb, gb = G.fwd_bwd(_W["cfg"], p, x[b:b + 1], y[b:b + 1])
        loss += lb
        g_all = gb if g_all is None else {k: g_all[k] + gb[k] for k in gb}
    gv = _views(out, _W["shapes"])
    for k, v in g_all.items():
        gv[k][...] = v
    out.flush()
    return loss


@pytest.mark.skipif(not RUN, reason="set GPT2_RUN_SLOW=1 (the oracle takes minutes)")
def test_small_config_20_step_loss_curve(tmp_path_factory):
    from gpu_util import i32, rel_l2, require_gpu
    require_gpu()
    import gpt_step_b200 as gs
    from gpt_step_b200 import synth, workloads
    from oracle import gpt2 as G

    w = workloads.WORKLOADS["small"]
    args = workloads.model_args("small")
    B, T, V, steps = args["micro_batch"], args["seq_len"], args["vocab_real"], w["steps"]
    assert (B, steps, args["warmup_steps"], args["total_steps"]) == (16, 20, 5, 20)
    m = gs.GPT2(gs.Config.make(**args), 1337)
    ocfg = G.Config(**args)
    p = G.init_params(ocfg, 1337)
    om, ov = G.zeros_like_params(ocfg), G.zeros_like_params(ocfg)
    src = synth.TokenSource(B, T, V, 1337, w["mean_doc_len"], steps * B)
    batches = [src.get() for _ in range(steps)]
    # the pool starts before this process has more GPU work than the model above;
    # spawn, never fork, after CUDA is initialised
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ.setdefault(v, "1")
    one = dict(args, micro_batch=1)
    shapes = [(k, s) for k, s, _ in G.param_shapes(ocfg)]
    total = sum(int(np.prod(s)) for _, s in shapes)
    nw = min(B, os.cpu_count() or 1)
    chunks = np.array_split(np.arange(B), nw)
    tmp = tmp_path_factory.mktemp("curve")
    ppath, gpath = str(tmp / "params.f64"), str(tmp / "grads.f64")
    pbuf = np.memmap(ppath, np.float64, "w+", shape=(total,))
    np.memmap(gpath, np.float64, "w+", shape=(len(chunks) * total,)).flush()
    ctx = mp.get_context("spawn")   # never fork a process that has initialised CUDA
    gl, ol, gn, on = [], [], [], []
    with ctx.Pool(nw, initializer=_worker_init, initargs=(one, ppath, gpath, total)) as pool:
        for step, (x, y) in enumerate(batches):
            m.fwd_bwd(i32(x), i32(y))
            m.clip_adamw(step)
            loss, norm = m.last_step_stats()
            pv = _views(pbuf, shapes)
            for k, _ in shapes:
                pv[k][...] = p[k]
            pbuf.flush()
            losses = pool.map(_chunk_grad, [(i, x[c], y[c]) for i, c in enumerate(chunks)])
            gbuf = np.memmap(gpath, np.float64, "r", shape=(len(chunks), total))
            gsum = np.asarray(gbuf).sum(axis=0) / B
            g = {k: np.array(v) for k, v in _views(gsum, shapes).items()}
            oloss = float(sum(losses) / B)
            onorm = G.clip_adamw(ocfg, p, g, om, ov, step)
            gl.append(loss); ol.append(oloss); gn.append(norm); on.append(onorm)
            print(f"step {step:2d}: loss {loss:.5f} (oracle {oloss:.5f})  norm {norm:.4f} (oracle {onorm:.4f})")
    dl = max(abs(a - b) for a, b in zip(gl, ol))
    dn = max(abs(a - b) / b for a, b in zip(gn, on))
    print(f"20-step curve: max |loss diff| {dl:.2e}, max relative norm diff {dn:.2e}")
    assert all(math.isfinite(v) for v in gl)
    assert dl <= 2e-2, dl
    assert dn <= 3e-2, dn
    assert gl[-1] < gl[0] - 0.5               # the curve descends
    names = [t.name for t in m.tensors()]
    got = m.read_all(gs.GPT2_PARAMS)
    ref = G.split_named(ocfg, p)
    err = rel_l2(np.concatenate([got[n].ravel() for n in names]),
                 np.concatenate([np.asarray(ref[n]).ravel() for n in names]))
    print(f"weights after 20 steps: relative L2 {err:.2e}")
    assert err <= 1e-2, err
    m.close()
