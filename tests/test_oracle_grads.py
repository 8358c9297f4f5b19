"""The oracle's forward and backward pinned by finite differences, brute force,
invariants, special cases and an independent library computation. No GPU.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as TF

from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G

MICRO = dict(n_layer=2, n_head=2, n_embd=16, seq_len=8, vocab_real=37, micro_batch=2)


def perturbed_params(cfg, seed, scale=0.3):
    """Arbitrary (not initialisation) weights large enough to exercise every nonlinearity."""
    p = G.init_params(cfg, seed)
    rng = np.random.default_rng(seed)
    for k in p:
        p[k] = p[k] + rng.standard_normal(p[k].shape) * (scale if p[k].ndim > 1 else 0.2)
    p["wte"][cfg.V:] = rng.standard_normal(p["wte"][cfg.V:].shape)  # padded rows: must not matter
    return p


def micro_batch(cfg, seed):
    return synth.uniform_next_token_batch(cfg.micro_batch, cfg.T, cfg.V, seed)


# --- central finite differences in fp64 ---------------------------------------------------

@pytest.mark.parametrize("cfgkw", [MICRO, dict(MICRO, n_layer=1, n_head=4, seq_len=5, vocab_real=130)])
def test_finite_differences_every_kind(cfgkw):
    cfg = G.Config(**cfgkw)
    p = perturbed_params(cfg, 7)
    x, y = micro_batch(cfg, 8)
    loss, g = G.fwd_bwd(cfg, p, x, y)
    rng = np.random.default_rng(9)
    h = 1e-5
    for kind in G.KIND_NAMES:
        a = p[kind]
        flat_idx = list(rng.choice(a.size, size=min(12, a.size), replace=False))
        if kind == "wte":
            flat_idx += [int(x[0, 0]) * cfg.C + 3, int(y[1, 2]) * cfg.C + 5, (cfg.V + 1) * cfg.C]
        fd, an = [], []
        for fi in flat_idx:
            idx = np.unravel_index(fi, a.shape)
            old = a[idx]
            a[idx] = old + h
            lp, _, _ = G.forward(cfg, p, x, y)
            a[idx] = old - h
            lm, _, _ = G.forward(cfg, p, x, y)
            a[idx] = old
            fd.append((lp - lm) / (2 * h))
            an.append(g[kind][idx])
        fd, an = np.array(fd), np.array(an)
        err = np.linalg.norm(fd - an)
        assert err <= 1e-6 * np.linalg.norm(an) + 1e-9, (kind, fd, an)


def test_finite_differences_tiny_config():
    cfg = G.Config(**workloads.model_args("tiny"))
    p = G.init_params(cfg, 1337)
    x, y = synth.uniform_next_token_batch(cfg.micro_batch, cfg.T, cfg.V, 1337)
    loss, g = G.fwd_bwd(cfg, p, x, y)
    rng = np.random.default_rng(1)
    h = 1e-4
    for kind in ("wte", "qkvw", "fcprojw", "ln2w", "lnfb", "qkvb"):
        a = p[kind]
        # pick the largest-gradient elements so the check is not dominated by roundoff
        cand = rng.choice(a.size, size=min(2000, a.size), replace=False)
        pick = cand[np.argsort(-np.abs(g[kind].ravel()[cand]))[:3]]
        for fi in pick:
            idx = np.unravel_index(fi, a.shape)
            old = a[idx]
            a[idx] = old + h
            lp, _, _ = G.forward(cfg, p, x, y)
            a[idx] = old - h
            lm, _, _ = G.forward(cfg, p, x, y)
            a[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[kind][idx]) <= 1e-6 * abs(g[kind][idx]) + 1e-10, (kind, fd, g[kind][idx])


# --- an independent implementation with library autograd ----------------------------------

def torch_reference(cfg, p, x, y):
    """GPT-2 written with torch's own layer_norm / gelu / sdpa / cross_entropy in fp64."""
    P = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p.items()}
    B, T = x.shape
    C, H = cfg.C, cfg.H
    tok = torch.tensor(x, dtype=torch.long)
    h = P["wte"][tok] + P["wpe"][:T]
    for l in range(cfg.L):
        a = TF.layer_norm(h, (C,), P["ln1w"][l], P["ln1b"][l], eps=1e-5)
        qkv = TF.linear(a, P["qkvw"][l], P["qkvb"][l])
        q, k, v = (t.view(B, T, H, C // H).transpose(1, 2) for t in qkv.split(C, dim=-1))
        o = TF.scaled_dot_product_attention(q, k, v, is_causal=True)
        h = h + TF.linear(o.transpose(1, 2).reshape(B, T, C), P["attprojw"][l], P["attprojb"][l])
        b = TF.layer_norm(h, (C,), P["ln2w"][l], P["ln2b"][l], eps=1e-5)
        u = TF.gelu(TF.linear(b, P["fcw"][l], P["fcb"][l]), approximate="tanh")
        h = h + TF.linear(u, P["fcprojw"][l], P["fcprojb"][l])
    f = TF.layer_norm(h, (C,), P["lnfw"], P["lnfb"], eps=1e-5)
    z = f @ P["wte"].T
    loss = TF.cross_entropy(z[..., : cfg.V].reshape(-1, cfg.V), torch.tensor(y, dtype=torch.long).reshape(-1))
    loss.backward()
    return float(loss.detach()), {k: t.grad.numpy() for k, t in P.items()}


@pytest.mark.parametrize("cfgkw", [MICRO, workloads.model_args("tiny")])
def test_matches_torch_autograd(cfgkw):
    cfg = G.Config(**cfgkw)
    p = perturbed_params(cfg, 11, scale=0.1)
    x, y = micro_batch(cfg, 12)
    loss, g = G.fwd_bwd(cfg, p, x, y)
    tl, tg = torch_reference(cfg, p, x, y)
    assert loss == pytest.approx(tl, rel=1e-12)
    for k in G.KIND_NAMES:
        np.testing.assert_allclose(g[k], tg[k], rtol=1e-9, atol=1e-13, err_msg=k)


# --- padded vocabulary (numbat §4.1) -----------------------------------------------------

def test_padded_vocab_gets_no_probability_or_gradient():
    cfg = G.Config(**MICRO)
    p = perturbed_params(cfg, 13)
    x, y = micro_batch(cfg, 14)
    loss, losses, cache = G.forward(cfg, p, x, y)
    g = G.backward(cfg, p, cache)
    assert np.all(g["wte"][cfg.V:] == 0.0)
    dz = cache["dz"]
    assert np.all(dz[:, cfg.V:] == 0.0)
    np.testing.assert_allclose(dz.sum(axis=1), 0.0, atol=1e-15)
    # the padded logits do not influence the loss at all
    z = cache["logits"].copy()
    z[:, cfg.V:] += 1e3
    l2, _ = G.softmax_ce(z, y.reshape(-1), cfg.V)
    np.testing.assert_array_equal(l2, losses.reshape(-1))


def test_softmax_ce_matches_library():
    rng = np.random.default_rng(3)
    N, V, Vp = 6, 50, 128
    z = rng.standard_normal((N, Vp)) * 3
    t = rng.integers(0, V, N)
    losses, dz = G.softmax_ce(z, t, V)
    ref = scipy.special.logsumexp(z[:, :V], axis=1) - z[np.arange(N), t]
    np.testing.assert_allclose(losses, ref, rtol=1e-13)
    sm = scipy.special.softmax(z[:, :V], axis=1)
    sm[np.arange(N), t] -= 1
    np.testing.assert_allclose(dz[:, :V], sm / N, rtol=1e-12, atol=1e-16)


def test_initial_loss_near_log_vocab():
    for name, kw in (("tiny", {}), ("small", dict(micro_batch=1))):
        cfg = G.Config(**workloads.model_args(name, **kw))
        p = G.init_params(cfg, 1337)
        if name == "tiny":
            x, y = synth.uniform_next_token_batch(cfg.micro_batch, cfg.T, cfg.V, 1337)
        else:
            s = synth.zipf_document_stream(cfg.T + 1, cfg.V, cfg.V - 1, 800, 1337)
            x, y = synth.windows(s, 1, cfg.T)
        loss, _, _ = G.forward(cfg, p, x, y)
        expected = math.log(cfg.V) + 0.5 * (0.02 ** 2) * cfg.C
        assert abs(loss - expected) < 0.1, (name, loss, expected)


# --- building blocks against brute force and invariants ------------------------------------

def test_attention_brute_force():
    rng = np.random.default_rng(4)
    T, hd = 5, 3
    q, k, v = (rng.standard_normal((T, hd)) for _ in range(3))
    o, lse = G.attention_fwd(q, k, v)
    for i in range(T):
        s = [sum(q[i, d] * k[j, d] for d in range(hd)) / math.sqrt(hd) for j in range(i + 1)]
        mx = max(s)
        e = [math.exp(a - mx) for a in s]
        tot = sum(e)
        assert lse[i] == pytest.approx(mx + math.log(tot), rel=1e-13)
        for d in range(hd):
            assert o[i, d] == pytest.approx(sum(e[j] / tot * v[j, d] for j in range(i + 1)), rel=1e-12, abs=1e-14)


def test_attention_single_position_returns_v_and_is_causal():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((2, 3, 1, 8)) for _ in range(3))
    o, _ = G.attention_fwd(q, k, v)
    np.testing.assert_allclose(o, v, rtol=1e-15)
    q, k, v = (rng.standard_normal((1, 2, 7, 4)) for _ in range(3))
    o1, _ = G.attention_fwd(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[..., 4:, :] += 5.0
    v2[..., 4:, :] -= 3.0
    o2, _ = G.attention_fwd(q, k2, v2)
    np.testing.assert_array_equal(o1[..., :4, :], o2[..., :4, :])


def test_attention_backward_matches_torch():
    rng = np.random.default_rng(6)
    q, k, v, do = (rng.standard_normal((2, 3, 9, 4)) for _ in range(4))
    dq, dk, dv = G.attention_bwd(do, q, k, v)
    Q, K, Vt = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    TF.scaled_dot_product_attention(Q, K, Vt, is_causal=True).backward(torch.tensor(do))
    for a, b in ((dq, Q), (dk, K), (dv, Vt)):
        np.testing.assert_allclose(a, b.grad.numpy(), rtol=1e-10, atol=1e-13)


def test_attention_bias_gradient_identities():
    """The column sums that the fused QKV bias gradient uses: over all queries,
    dk sums to zero (a shift shared by a query's scores cancels in its softmax)
    and dv sums to do (every causal softmax row sums to one); checked against
    the oracle's gradients and against finite differences of the loss in a bias
    added to every key or value row."""
    rng = np.random.default_rng(16)
    q, k, v, do = (rng.standard_normal((2, 3, 11, 4)) for _ in range(4))
    dq, dk, dv = G.attention_bwd(do, q, k, v)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=1e-12, atol=1e-12)
    loss = lambda kk, vv: float((G.attention_fwd(q, kk, vv)[0] * do).sum())
    e = 1e-6
    bk = rng.standard_normal(4)
    assert abs(loss(k + e * bk, v) - loss(k - e * bk, v)) / (2 * e) < 1e-7
    bv = rng.standard_normal(4)
    fd = (loss(k, v + e * bv) - loss(k, v - e * bv)) / (2 * e)
    assert fd == pytest.approx(float((do.sum(axis=(0, 2)) * bv).sum()), rel=1e-6)


def test_layernorm_brute_force_and_invariants():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 10)) * 2 + 1
    w, b = np.ones(10), np.zeros(10)
    y, mean, rstd = G.layernorm_fwd(x, w, b)
    for r in range(3):
        mu = sum(x[r]) / 10
        var = sum((a - mu) ** 2 for a in x[r]) / 10
        for c in range(10):
            assert y[r, c] == pytest.approx((x[r, c] - mu) / math.sqrt(var + 1e-5), rel=1e-13)
    dy = rng.standard_normal((3, 10))
    dx, dw, db = G.layernorm_bwd(dy, x, mean, rstd, w)
    np.testing.assert_allclose(dx.sum(axis=1), 0.0, atol=1e-13)
    # sum_c dx * xhat = 0 holds up to eps / var; with var ~ 4e4 that is ~1e-9 relative
    xs = x * 200.0
    ys, ms, rs = G.layernorm_fwd(xs, w, b)
    dxs, _, _ = G.layernorm_bwd(dy, xs, ms, rs, w)
    np.testing.assert_allclose((dxs * ys).sum(axis=1) / np.abs(dxs * ys).sum(axis=1), 0.0, atol=1e-8)
    np.testing.assert_allclose(db, dy.sum(0), rtol=1e-14)


def test_gelu_matches_library():
    u = np.linspace(-6, 6, 101)
    ut = torch.tensor(u, requires_grad=True)
    gt = TF.gelu(ut, approximate="tanh")
    gt.backward(torch.ones_like(ut))
    np.testing.assert_allclose(G.gelu_fwd(u), gt.detach().numpy(), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(G.gelu_bwd(u, np.ones_like(u)), ut.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert G.gelu_fwd(np.array([0.0]))[0] == 0.0


def test_model_is_causal():
    cfg = G.Config(**MICRO)
    p = perturbed_params(cfg, 15)
    x, y = micro_batch(cfg, 16)
    _, l1, _ = G.forward(cfg, p, x, y)
    x2 = x.copy()
    x2[:, 5] = (x2[:, 5] + 1) % cfg.V
    _, l2, _ = G.forward(cfg, p, x2, y)
    np.testing.assert_array_equal(l1[:, :5], l2[:, :5])
    assert not np.allclose(l1[:, 5:], l2[:, 5:])


def test_zero_layer_model_is_logistic_regression():
    cfg = G.Config(**dict(MICRO, n_layer=0))
    p = perturbed_params(cfg, 17)
    x, y = micro_batch(cfg, 18)
    loss, g = G.fwd_bwd(cfg, p, x, y)
    f, _, _ = G.layernorm_fwd(p["wte"][x] + p["wpe"][: cfg.T], p["lnfw"], p["lnfb"])
    F = f.reshape(-1, cfg.C)
    probs = scipy.special.softmax(F @ p["wte"][: cfg.V].T, axis=1)
    nll = -np.log(probs[np.arange(F.shape[0]), y.reshape(-1)]).mean()
    assert loss == pytest.approx(nll, rel=1e-12)
    # head part of the tied gradient: (P - Y)^T F / N; embedding part adds only at input ids
    Y = np.zeros_like(probs)
    Y[np.arange(F.shape[0]), y.reshape(-1)] = 1
    head = (probs - Y).T @ F / F.shape[0]
    untouched = np.setdiff1d(np.arange(cfg.V), x.reshape(-1))
    np.testing.assert_allclose(g["wte"][untouched], head[untouched], rtol=1e-11, atol=1e-15)


def test_equal_shards_average_to_the_whole_batch():
    """The mean loss over a batch is the mean of its equal-sized shards' mean
    losses, so its gradient is the mean of theirs. Gradient accumulation
    ("Pretraining and adapting a language model on a dependency-free stack"
    §4.3, 9 micro-steps per optimizer step) and the average across cards (§4.4)
    both rely on this. So one optimizer step over 4 sequences must equal one
    step accumulated over two shards of 2, with the same pre-clip norm."""
    cfg = G.Config(**dict(MICRO, micro_batch=4))
    p = perturbed_params(cfg, 23)
    x, y = micro_batch(cfg, 24)
    loss, g = G.fwd_bwd(cfg, p, x, y)
    l0, g0 = G.fwd_bwd(cfg, p, x[:2], y[:2])
    l1, g1 = G.fwd_bwd(cfg, p, x[2:], y[2:])
    assert loss == pytest.approx(0.5 * (l0 + l1), rel=1e-13)
    for k in g:
        np.testing.assert_allclose(g[k], 0.5 * (g0[k] + g1[k]), rtol=1e-10, atol=1e-15)
    pa, pb = {k: v.copy() for k, v in p.items()}, {k: v.copy() for k, v in p.items()}
    ma, va, mb, vb = (G.zeros_like_params(cfg) for _ in range(4))
    la, na = G.train_step(cfg, pa, ma, va, 3, [(x, y)])
    lb, nb = G.train_step(cfg, pb, mb, vb, 3, [(x[:2], y[:2]), (x[2:], y[2:])])
    assert la == pytest.approx(lb, rel=1e-13) and na == pytest.approx(nb, rel=1e-10)
    for k in pa:
        np.testing.assert_allclose(pa[k], pb[k], rtol=0, atol=1e-12)
