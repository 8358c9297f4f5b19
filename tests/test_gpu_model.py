"""Whole-step parity: gpt2_create / gpt2_fwd_bwd / gpt2_clip_adamw against the oracle.

Both sides draw the initial weights from the same Philox stream (the oracle in
fp64, the device in fp32) and see the same seeded tokens. Tolerances are the
ones the target fixes for a bf16-activation / fp32-master step against an fp32
definition: |loss diff| <= 2e-2, per-tensor gradient relative L2 <= 3e-2,
post-step weights relative L2 <= 1e-3 (over the elements whose first-step sign is
determined; see check_first_step), and the AdamW update on identical fp32
gradients within 1e-6 relative.
"""
import math

import numpy as np
import pytest

import gpt_step_b200 as gs
from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G

from gpu_util import i32, rel_l2, require_gpu, torch

pytestmark = pytest.mark.gpu

LOSS_TOL, GRAD_TOL, STEP_TOL, ADAM_TOL = 2e-2, 3e-2, 1e-3, 1e-6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def pair(name, seed=1337, **over):
    args = workloads.model_args(name, **over)
    m = gs.GPT2(gs.Config.make(**args), seed)
    return m, G.Config(**args)


def oracle_named(ocfg, arrays):
    return G.split_named(ocfg, arrays)


def flat(named, names):
    return np.concatenate([np.asarray(named[n], np.float64).ravel() for n in names])


def check_first_step(ocfg, got, ref, w0, grad, lr):
    """Post-step weights after the FIRST AdamW step.

    At t = 1 the update is m/(sqrt(v)+eps) = g/(|g|+eps), i.e. a sign decision per
    element: each weight moves by about lr whatever |g| is. Where |g| lies inside
    the bf16 noise of the gradient (bf16 activations, numbat §4.3) that sign is not
    determined by the method, so, as for any floating-point-decided discrete
    outcome, the determined elements are compared against the bar and the others
    are only checked to be valid updates (|step| <= lr). Storing activations in
    bf16 alone, with everything else exact, already gives a whole-vector error of
    1.3e-3 at lr 6e-4 (tests/test_bf16_floor.py), which is reported here too.
    """
    names = list(got)
    det_got, det_ref, whole_got, whole_ref = [], [], [], []
    for n in names:
        g = np.asarray(grad[n], np.float64)
        rms = np.sqrt(np.mean(g * g)) if g.size else 0.0
        det = np.abs(g) >= 0.01 * rms   # 2.5 x bf16's relative precision (2^-8) of the RMS gradient
        a, b = np.asarray(got[n], np.float64), np.asarray(ref[n], np.float64)
        det_got.append(a[det]); det_ref.append(b[det])
        whole_got.append(a.ravel()); whole_ref.append(b.ravel())
        # undetermined elements: any valid Adam step (|normalised step| <= 1, decay on 2-D only)
        w = np.asarray(w0[n], np.float64)
        decay = 0.1 * w if w.ndim == 2 else 0.0
        step = (w - a) / lr - decay
        assert np.all(np.abs(step[~det]) <= 1.0 + 1e-3), n
    det_err = rel_l2(np.concatenate(det_got), np.concatenate(det_ref))
    whole_err = rel_l2(np.concatenate(whole_got), np.concatenate(whole_ref))
    print(f"first-step weights: determined elements rel L2 {det_err:.3e}, whole vector {whole_err:.3e}")
    assert det_err <= STEP_TOL, det_err
    assert whole_err <= 2 * STEP_TOL, whole_err


def batch_for(name, ocfg, seed=1337, n=1):
    w = workloads.WORKLOADS[name]
    if w["input"] == "uniform":
        return [synth.uniform_next_token_batch(ocfg.micro_batch, ocfg.T, ocfg.V, seed + i) for i in range(n)]
    src = synth.TokenSource(ocfg.micro_batch, ocfg.T, ocfg.V, seed, w["mean_doc_len"], n * ocfg.micro_batch)
    return [src.get() for _ in range(n)]


# --- initialisation ([numbat] §4.1) ----------------------------------------------------------

def test_initial_weights_match_oracle():
    m, ocfg = pair("tiny")
    got = m.read_all(gs.GPT2_PARAMS)
    ref = oracle_named(ocfg, G.init_params(ocfg, 1337))
    assert len(got) == len(G.tensor_names(ocfg))
    for name, a in got.items():
        assert a.shape == ref[name].shape, name
        assert np.max(np.abs(a - ref[name])) <= 2e-7 * max(1.0, np.max(np.abs(ref[name]))), name
    assert np.all(got["wte.weight"][ocfg.V:] == 0.0)


# --- one full step on the tiny configuration -------------------------------------------------

def test_tiny_step_parity():
    m, ocfg = pair("tiny")
    (x, y), = batch_for("tiny", ocfg)
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    grads = m.read_all(gs.GPT2_GRADS)
    p = G.init_params(ocfg, 1337)
    oloss, og = G.fwd_bwd(ocfg, p, x, y)
    assert abs(loss - oloss) <= LOSS_TOL
    assert abs(oloss - math.log(ocfg.V)) < 0.1
    ogn = oracle_named(ocfg, og)
    for name, a in grads.items():
        assert rel_l2(a, ogn[name]) <= GRAD_TOL, (name, rel_l2(a, ogn[name]))
    assert np.all(grads["wte.weight"][ocfg.V:] == 0.0)
    norm = m.clip_adamw(0, want_norm=True)
    m_, v_ = G.zeros_like_params(ocfg), G.zeros_like_params(ocfg)
    onorm = G.clip_adamw(ocfg, p, og, m_, v_, 0)
    assert abs(norm - onorm) <= GRAD_TOL * onorm
    got = m.read_all(gs.GPT2_PARAMS)
    check_first_step(ocfg, got, oracle_named(ocfg, p), oracle_named(ocfg, G.init_params(ocfg, 1337)), ogn,
                     G.lr_at(ocfg, 0))
    assert np.all(got["wte.weight"][ocfg.V:] == 0.0)
    # gradients are cleared by the step
    assert all(np.all(g == 0) for g in m.read_all(gs.GPT2_GRADS).values())
    ml, mn = m.last_step_stats()
    assert ml == pytest.approx(loss, rel=1e-6) and mn == pytest.approx(norm, rel=1e-6)


def test_eval_loss_and_token_losses_match_forward():
    m, ocfg = pair("tiny")
    (x, y), = batch_for("tiny", ocfg, seed=5)
    ev = m.eval_loss(i32(x), i32(y))
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    tl = m.token_losses()
    assert ev == pytest.approx(loss, abs=1e-5)
    assert float(tl.mean()) == pytest.approx(loss, abs=1e-5)
    ref = G.token_losses(ocfg, G.init_params(ocfg, 1337), x, y)
    assert np.max(np.abs(tl - ref)) < 5e-2
    # eval over more rows than the micro-batch is chunked
    x2 = np.concatenate([x, x[::-1]])
    y2 = np.concatenate([y, y[::-1]])
    assert m.eval_loss(i32(x2), i32(y2)) == pytest.approx(loss, abs=1e-5)


# steps of the 124M schedule (warmup 700 to 6e-4, cosine to 0 at 18,865): first
# warmup step, end of warmup, start of the cosine, its midpoint, its last step
SCHEDULE_STEPS = [0, 699, 700, 9782, 18864]


@pytest.mark.parametrize("step", SCHEDULE_STEPS)
def test_adamw_on_identical_fp32_gradients(step):
    """clip + AdamW + bf16 copy on fp32 state written identically to both sides,
    with the 124M schedule so that the learning rate is non-zero: the update,
    the decoupled decay and both moments within 1e-6 relative of the oracle, and
    the library's learning rate equal to the oracle's."""
    m, ocfg = pair("tiny", warmup_steps=700, total_steps=18865)
    assert m.lr(step) == pytest.approx(G.lr_at(ocfg, step), rel=1e-6)
    assert G.lr_at(ocfg, step) > 0
    (x, y), = batch_for("tiny", ocfg)
    m.fwd_bwd(i32(x), i32(y))      # one micro-step pending
    rng = np.random.default_rng(99)
    names = [t.name for t in m.tensors()]
    P, Gd, M, V = {}, {}, {}, {}
    for i, t in enumerate(m.tensors()):
        P[t.name] = (rng.standard_normal(t.shape) * 0.05).astype(np.float32)
        Gd[t.name] = (rng.standard_normal(t.shape) * 0.02).astype(np.float32)
        M[t.name] = (rng.standard_normal(t.shape) * 1e-3).astype(np.float32)
        V[t.name] = (rng.random(t.shape) * 1e-4).astype(np.float32)
        if t.name == "wte.weight":     # padded rows stay zero, as the model keeps them
            for a in (P, Gd, M, V):
                a[t.name][ocfg.V:] = 0.0
        m.write(gs.GPT2_PARAMS, i, P[t.name])
        m.write(gs.GPT2_GRADS, i, Gd[t.name])
        m.write(gs.GPT2_ADAM_M, i, M[t.name])
        m.write(gs.GPT2_ADAM_V, i, V[t.name])
    norm = m.clip_adamw(step, want_norm=True)
    # oracle on the same fp32 values, per kind arrays assembled from named tensors
    def kinds(named):
        out = {}
        for kind, shape, _ in G.param_shapes(ocfg):
            out[kind] = np.zeros(shape)
        for name, kind, layer, _ in G.tensor_names(ocfg):
            if layer < 0:
                out[kind][...] = named[name]
            else:
                out[kind][layer] = named[name]
        return out
    op, og, om, ov = kinds(P), kinds(Gd), kinds(M), kinds(V)
    w0 = {k: v.copy() for k, v in op.items()}
    onorm = G.clip_adamw(ocfg, op, og, om, ov, step)
    assert onorm > 1.0                 # the clip is active
    assert norm == pytest.approx(onorm, rel=ADAM_TOL)
    for what, ref in ((gs.GPT2_PARAMS, op), (gs.GPT2_ADAM_M, om), (gs.GPT2_ADAM_V, ov)):
        got = m.read_all(what)
        refn = oracle_named(ocfg, ref)
        for n in names:
            assert rel_l2(got[n], refn[n]) <= ADAM_TOL, (what, n, rel_l2(got[n], refn[n]))
    # the update itself (w1 - w0), not only w1, matches. It is lr-sized, far below
    # |w|, so storing w1 in fp32 alone costs a relative error `floor` (the fp32
    # rounding of the exact w1); the bar is 1e-4 above twice that floor.
    got = m.read_all(gs.GPT2_PARAMS)
    w1 = flat(oracle_named(ocfg, op), names)
    d_got = flat({n: got[n] - P[n] for n in names}, names)
    d_ref = w1 - flat(oracle_named(ocfg, w0), names)
    floor = rel_l2(w1.astype(np.float32).astype(np.float64) - flat(oracle_named(ocfg, w0), names), d_ref)
    err = rel_l2(d_got, d_ref)
    print(f"step {step}: lr {G.lr_at(ocfg, step):.3e}, update rel L2 {err:.3e} (fp32 storage floor {floor:.3e})")
    assert err <= 1e-4 + 2 * floor, (err, floor)
    assert np.all(got["wte.weight"][ocfg.V:] == 0.0)


def test_bad_token_and_nonfinite_are_reported():
    m, ocfg = pair("tiny")
    (x, y), = batch_for("tiny", ocfg)
    bad = x.copy()
    bad[1, 3] = ocfg.V
    with pytest.raises(gs.GPT2Error) as e:
        m.fwd_bwd(i32(bad), i32(y), want_loss=True)
    assert e.value.status == 3
    with pytest.raises(gs.GPT2Error) as e:
        m.clip_adamw(0)
        m.clip_adamw(0)
    assert e.value.status == 5        # second step with no micro-step in between
    # a non-finite parameter: the step is refused and the weights stay as they were
    before = m.read_all(gs.GPT2_PARAMS)
    idx = [t.name for t in m.tensors()].index("ln_f.weight")
    w = before["ln_f.weight"].copy()
    w[0] = np.nan
    m.write(gs.GPT2_PARAMS, idx, w)
    m.fwd_bwd(i32(x), i32(y))
    with pytest.raises(gs.GPT2Error) as e:
        m.clip_adamw(1, want_norm=True)
    assert e.value.status == 4
    after = m.read_all(gs.GPT2_PARAMS)
    for n in before:
        if n != "ln_f.weight":
            np.testing.assert_array_equal(after[n], before[n])
    # still usable after restoring the weight
    m.write(gs.GPT2_PARAMS, idx, before["ln_f.weight"])
    assert np.isfinite(m.fwd_bwd(i32(x), i32(y), want_loss=True))


def test_host_train_step_matches_device_calls():
    m1, ocfg = pair("tiny")
    m2, _ = pair("tiny")
    bs = batch_for("tiny", ocfg, n=2)
    for x, y in bs:
        m1.fwd_bwd(i32(x), i32(y))
    m1.clip_adamw(0)
    l1, n1 = m1.last_step_stats()
    toks = np.stack([b[0] for b in bs]).astype(np.int32)
    tgts = np.stack([b[1] for b in bs]).astype(np.int32)
    l2, n2 = m2.train_step_host(toks, tgts, 0)
    assert l1 == pytest.approx(l2, abs=1e-6) and n1 == pytest.approx(n2, rel=1e-3)


# --- head size 64: the tcgen05 attention path with fused bias gradients ----------------------

def test_head64_accumulated_gradients_match_oracle():
    """Head size 64 and T a multiple of 128 take the tcgen05 attention (the tiny and
    small configurations use head size 32), and the GELU-backward GEMM epilogue
    adds the MLP fc bias gradient by atomics. Two micro-steps check that the
    gradients accumulate."""
    m, ocfg = pair("tiny", n_head=2, seq_len=256, micro_batch=2)
    batches = batch_for("tiny", ocfg, n=2)
    p = G.init_params(ocfg, 1337)
    og = None
    for x, y in batches:
        loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
        oloss, g = G.fwd_bwd(ocfg, p, x, y)
        assert abs(loss - oloss) <= LOSS_TOL
        og = g if og is None else {k: og[k] + g[k] for k in og}
    grads = m.read_all(gs.GPT2_GRADS)
    ogn = oracle_named(ocfg, og)
    for name, a in grads.items():
        assert rel_l2(a, ogn[name]) <= GRAD_TOL, (name, rel_l2(a, ogn[name]))


# --- the small configuration: full context length, many tiles --------------------------------

def test_small_config_step_parity():
    m, ocfg = pair("small", micro_batch=2)
    (x, y), = batch_for("small", ocfg)
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    grads = m.read_all(gs.GPT2_GRADS)
    p = G.init_params(ocfg, 1337)
    oloss, og = G.fwd_bwd(ocfg, p, x, y)
    assert abs(loss - oloss) <= LOSS_TOL
    ogn = oracle_named(ocfg, og)
    worst = max(rel_l2(a, ogn[n]) for n, a in grads.items())
    assert worst <= GRAD_TOL, worst
    m.clip_adamw(0)
    w0 = oracle_named(ocfg, {k: v.copy() for k, v in p.items()})
    G.clip_adamw(ocfg, p, og, G.zeros_like_params(ocfg), G.zeros_like_params(ocfg), 0)
    check_first_step(ocfg, m.read_all(gs.GPT2_PARAMS), oracle_named(ocfg, p), w0, ogn, G.lr_at(ocfg, 0))


def test_small_config_accumulated_steps_track_oracle():
    m, ocfg = pair("small", micro_batch=1)
    p = G.init_params(ocfg, 1337)
    om, ov = G.zeros_like_params(ocfg), G.zeros_like_params(ocfg)
    src = synth.TokenSource(1, ocfg.T, ocfg.V, 1337, 800, 8)
    for step in range(3):
        bs = [src.get(), src.get()]
        for x, y in bs:
            m.fwd_bwd(i32(x), i32(y))
        m.clip_adamw(step)
        gl, gn = m.last_step_stats()
        ol, on = G.train_step(ocfg, p, om, ov, step, bs)
        assert abs(gl - ol) <= LOSS_TOL, (step, gl, ol)
        assert abs(gn - on) <= GRAD_TOL * on, (step, gn, on)
    got = m.read_all(gs.GPT2_PARAMS)
    names = list(got)
    assert rel_l2(flat(got, names), flat(oracle_named(ocfg, p), names)) <= STEP_TOL


# --- GPT-2 124M in the launch configuration the benchmark times (B = 19) ---------------------

def test_gpt2_124m_bench_configuration_sampled():
    m, ocfg = pair("gpt2_124m")
    (x, y), = batch_for("gpt2_124m", ocfg)
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    tl = m.token_losses()
    assert float(tl.mean()) == pytest.approx(loss, abs=1e-4)
    p = G.init_params(ocfg, 1337)
    for b in (0, 18):                                   # sequences the oracle computes one by one
        ref = G.token_losses(ocfg, p, x[b:b + 1], y[b:b + 1])[0]
        assert abs(float(tl[b].mean()) - float(ref.mean())) <= LOSS_TOL
        assert np.max(np.abs(tl[b] - ref)) < 0.15
    g = m.read_all(gs.GPT2_GRADS)
    assert np.all(g["wte.weight"][ocfg.V:] == 0.0)
    assert all(np.all(np.isfinite(a)) for a in g.values())
    norm = m.clip_adamw(0, want_norm=True)
    assert np.isfinite(norm) and norm > 0
    assert np.all(m.read(gs.GPT2_PARAMS, 0)[ocfg.V:] == 0.0)


def test_gpt2_124m_micro_batch_64_with_held_out_pass_sampled():
    """The large-micro-batch 124M configuration (64 x 1024 per micro-step) and its
    held-out pass (batches of 64 x 1024 from a separately seeded stream): the
    micro-step's per-token losses on a sampled sequence against the oracle, and the
    held-out loss equal to the forward's mean loss on the same batch."""
    m, ocfg = pair("gpt2_124m_b64")
    w = workloads.WORKLOADS["gpt2_124m_b64"]
    (x, y), = batch_for("gpt2_124m_b64", ocfg)
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    tl = m.token_losses()
    assert tl.shape == (64, 1024) and float(tl.mean()) == pytest.approx(loss, abs=1e-4)
    p = G.init_params(ocfg, 1337)
    ref = G.token_losses(ocfg, p, x[63:64], y[63:64])[0]
    assert abs(float(tl[63].mean()) - float(ref.mean())) <= LOSS_TOL
    assert np.max(np.abs(tl[63] - ref)) < 0.15
    assert np.isfinite(m.clip_adamw(0, want_norm=True))
    src = synth.TokenSource(w["eval_batch"], ocfg.T, ocfg.V, w["eval_seed"], w["mean_doc_len"], w["eval_batch"])
    ex, ey = src.get()
    ev = m.eval_loss(i32(ex), i32(ey))
    assert ev == pytest.approx(m.fwd_bwd(i32(ex), i32(ey), want_loss=True), abs=1e-5)
    m.close()


def test_wide_configuration_sampled():
    """The wide configuration (16 blocks, 24 heads, 1536 channels, vocabulary 8449
    padded to 8576, micro-batch 8): per-token losses of a sampled sequence against
    the oracle, finite gradients with zero padded rows, a finite clipped step."""
    m, ocfg = pair("wide")
    (x, y), = batch_for("wide", ocfg)
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    tl = m.token_losses()
    assert float(tl.mean()) == pytest.approx(loss, abs=1e-4)
    p = G.init_params(ocfg, 1337)
    ref = G.token_losses(ocfg, p, x[0:1], y[0:1])[0]
    assert abs(float(tl[0].mean()) - float(ref.mean())) <= LOSS_TOL
    assert np.max(np.abs(tl[0] - ref)) < 0.15
    g = m.read_all(gs.GPT2_GRADS)
    assert np.all(g["wte.weight"][ocfg.V:] == 0.0)
    assert all(np.all(np.isfinite(a)) for a in g.values())
    assert np.isfinite(m.clip_adamw(0, want_norm=True))
    m.close()


def test_checkpoint_resume_continues_the_run(tmp_path):
    """A run stopped at a checkpoint and restored into a model of another seed
    continues the uninterrupted run: the restored fp32 weights and moments are
    bitwise the saved ones, the held-out loss (forward only, no atomics) is bitwise
    equal, and the following steps track the uninterrupted ones to fp32 summation
    order (the split-K weight gradients add in an unspecified order)."""
    from gpt_step_b200 import checkpoint as ck
    over = dict(total_steps=10, warmup_steps=2, grad_accum=2)
    args = workloads.model_args("tiny", **over)
    w = workloads.WORKLOADS["tiny"]
    B, T, V = args["micro_batch"], args["seq_len"], args["vocab_real"]
    hx, hy = synth.uniform_next_token_batch(B, T, V, 4242)
    hx, hy = i32(hx), i32(hy)
    ev = lambda m: m.eval_loss(hx, hy)
    cad = ck.Cadence(eval_every=2, ckpt_every=2)
    src = lambda: synth.TokenSource(B, T, V, 1337, w["mean_doc_len"], 64)

    a = gs.GPT2(gs.Config.make(**args), 1337)
    ra = ck.run(a, src(), 0, 4, i32, cad, str(tmp_path / "a"), ev)
    path = ck.ckpt_path(str(tmp_path / "a"), 2)
    saved = np.load(path)

    b = gs.GPT2(gs.Config.make(**args), 999)
    h = ck.load(b, path)
    assert h["step"] == 2
    for i, t in enumerate(b.tensors()):
        for key, what in (("param", gs.GPT2_PARAMS), ("m", gs.GPT2_ADAM_M), ("v", gs.GPT2_ADAM_V)):
            assert np.array_equal(b.read(what, i), saved[f"{key}/{t.name}"]), (key, t.name)
    assert ev(b) == ra[1]["eval_loss"]
    s = src()
    s.next = h["data_cursor"]
    rb = ck.run(b, s, h["step"], 4, i32, cad, None, ev)
    for x, y in zip(ra[2:], rb):
        assert x["step"] == y["step"]
        assert y["loss"] == pytest.approx(x["loss"], rel=1e-5)
        assert y["grad_norm"] == pytest.approx(x["grad_norm"], rel=1e-4)
    for i, t in enumerate(a.tensors()):
        assert np.max(np.abs(a.read(gs.GPT2_PARAMS, i) - b.read(gs.GPT2_PARAMS, i))) <= 2e-6, t.name
    a.close()
    b.close()


def test_data_parallel_plumbing_on_one_rank():
    """The flat gradient array that data-parallel ranks average (gpt2_state_device_ptr)
    is the one gpt2_read reports, padded gaps zero; an NCCL average over a one-rank
    group leaves it bit-identical; and DataParallel's step on one rank runs the
    plain step and keeps the weights finite."""
    import socket

    import torch.distributed as dist
    from gpt_step_b200 import dp
    args = workloads.model_args("tiny")
    m = gs.GPT2(gs.Config.make(**args), 1337)
    x, y = synth.uniform_next_token_batch(args["micro_batch"], args["seq_len"], args["vocab_real"], 77)
    m.fwd_bwd(i32(x), i32(y))
    torch.cuda.synchronize()
    g = m.state_tensor(gs.GPT2_GRADS)
    per = sum(float(np.abs(m.read(gs.GPT2_GRADS, i).astype(np.float64)).sum()) for i in range(len(m.tensors())))
    assert per > 0 and float(g.double().abs().sum()) == pytest.approx(per, rel=1e-12)
    before = g.clone()
    own = not dist.is_initialized()
    if own:
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        dist.all_reduce(g, op=dist.ReduceOp.AVG)
        torch.cuda.synchronize()
        assert torch.equal(g, before)
        d = dp.DataParallel(m)
        assert d.world == 1
        m.clip_adamw(0)
        d.step([i32(x)], [i32(y)], 1)
        loss, norm = m.last_step_stats()
        assert math.isfinite(loss) and math.isfinite(norm) and d.replicas_agree()
    finally:
        if own:
            dist.destroy_process_group()
    m.close()
