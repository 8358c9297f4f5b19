"""Pins of the CPU oracle against values the pages print and closed forms.

Runs without a GPU. The oracle is test infrastructure; these tests are what let
the GPU parity tests trust it.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy import stats

from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G
from oracle import philox

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")))


def cfg_of(name, **over):
    return G.Config(**workloads.model_args(name, **over))


# --- architecture and counts (numbat §4.1, §4.4, §5.1) ------------------------------------

def test_param_count_gpt2_124m():
    cfg = cfg_of("gpt2_124m")
    assert (cfg.L, cfg.H, cfg.C, cfg.T) == tuple(GOLD["gpt2_124m_layers_heads_channels_context"]["value"])
    assert G.count_params(cfg) == GOLD["gpt2_124m_param_count"]["value"]
    # padded storage holds 47 extra vocabulary rows
    assert G.count_params(cfg, padded=True) - G.count_params(cfg) == (cfg.Vp - cfg.V) * cfg.C


def test_vocab_padding():
    V, Vp = GOLD["vocab_real_padded"]["value"]
    cfg = cfg_of("gpt2_124m")
    assert cfg.V == V and cfg.Vp == Vp and Vp % 128 == 0 and Vp - V < 128


def test_named_tensor_count_and_names():
    cfg = cfg_of("gpt2_124m")
    names = G.tensor_names(cfg)
    assert len(names) == GOLD["gpt2_124m_named_gradients"]["value"]
    assert GOLD["worst_gradient_tensor_name"]["value"] in [n for n, *_ in names]
    total = sum(int(np.prod(s)) for *_, s in names)
    assert total == G.count_params(cfg, padded=True)


def test_small_family_count_matches_table():
    g = GOLD["andrea_12m_params_millions"]
    sh = g["shape"]
    cfg = G.Config(n_layer=sh["layers"], n_head=sh["heads"], n_embd=sh["d_model"],
                   seq_len=sh["context"], vocab_real=sh["vocab"])
    assert round(G.count_params(cfg, padded=True) / 1e6, 1) == g["value"]


def test_batch_geometry_matches_pages():
    w = workloads.WORKLOADS["gpt2_124m"]
    b, t, a, tot = GOLD["tokens_per_step_per_card"]["value"]
    assert (w["micro_batch"], w["seq_len"], w["grad_accum"]) == (b, t, a)
    assert b * t * a == tot and 3 * tot == GOLD["tokens_per_step_three_cards"]["value"]
    (n1, b1, t1, c1, e1), (n2, b2, t2, c2, e2) = GOLD["eval_tokens"]["value"]
    assert n1 * b1 * t1 * c1 == e1 and n2 * b2 * t2 * c2 == e2
    w4 = workloads.WORKLOADS["gpt2_124m_b64"]
    assert w4["eval_batches"] * w4["eval_batch"] * w4["seq_len"] * 8 == e1
    for loss, ppl in GOLD["perplexity_pairs"]["value"]:
        assert abs(math.exp(loss) - ppl) < 5e-3


# --- Philox and the normals drawn from it -------------------------------------------------

@pytest.mark.parametrize("case", GOLD["philox4x32_10_kat"]["value"])
def test_philox_known_answers(case):
    c = [int(x, 16) for x in case["ctr"]]
    k = [int(x, 16) for x in case["key"]]
    out = philox.philox4x32_10(*c, *k)
    assert [int(np.asarray(o)) for o in out] == [int(x, 16) for x in case["out"]]


def test_normals_are_standard_normal():
    z = philox.normals(3, 200_000, 1337)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.01
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # streams for different kinds and seeds are uncorrelated
    z2 = philox.normals(4, 200_000, 1337)
    z3 = philox.normals(3, 200_000, 1338)
    assert abs(np.corrcoef(z, z2)[0, 1]) < 0.01 and abs(np.corrcoef(z, z3)[0, 1]) < 0.01
    # element order: element 4c+j is the j-th normal of counter block c
    assert np.array_equal(philox.normals(3, 10, 1337), z[:10])


def test_uniform_mapping_endpoints():
    u = philox.uniform_from_bits(np.array([0, 0xFFFFFFFF], dtype=np.uint32))
    assert u[0] == 0.5 / 2 ** 23 and u[1] == 1.0 - 0.5 / 2 ** 23
    # every value is exactly representable in fp32 (the CUDA side computes it in fp32)
    x = np.random.default_rng(0).integers(0, 2 ** 32, 10000, dtype=np.uint64).astype(np.uint32)
    uu = philox.uniform_from_bits(x)
    assert np.array_equal(uu.astype(np.float32).astype(np.float64), uu)


def test_init_statistics():
    cfg = cfg_of("small")
    p = G.init_params(cfg, 1337)
    assert np.all(p["wte"][cfg.V:] == 0.0)
    for name, std in (("wte", 0.02), ("wpe", 0.02), ("qkvw", 0.02), ("fcw", 0.02),
                      ("attprojw", 0.02 / math.sqrt(2 * cfg.L)),
                      ("fcprojw", 0.02 / math.sqrt(2 * cfg.L))):
        a = p[name][: cfg.V] if name == "wte" else p[name]
        assert abs(a.std() / std - 1.0) < 0.02, name
        assert abs(a.mean()) < 0.05 * std, name
    for name in ("ln1w", "ln2w", "lnfw"):
        assert np.all(p[name] == 1.0)
    for name in ("ln1b", "ln2b", "lnfb", "qkvb", "attprojb", "fcb", "fcprojb"):
        assert np.all(p[name] == 0.0)


# --- schedule (numbat §4.3) ----------------------------------------------------------------

def test_lr_schedule_closed_form():
    cfg = cfg_of("gpt2_124m")
    s = GOLD["lr_schedule"]["value"]
    assert (cfg.warmup_steps, cfg.max_lr, cfg.total_steps) == (s["warmup"], s["max_lr"], s["total"])
    assert G.lr_at(cfg, 0) == pytest.approx(6e-4 / 700, rel=1e-12)
    assert G.lr_at(cfg, 349) == pytest.approx(3e-4, rel=1e-12)
    assert G.lr_at(cfg, 699) == pytest.approx(6e-4, rel=1e-12)
    assert G.lr_at(cfg, 700) == pytest.approx(6e-4, rel=1e-12)
    span = 18865 - 700
    # cosine is symmetric about the midpoint: lr(700 + x) + lr(18865 - x) = max
    for x in (1, 100, 5000, 9000):
        assert G.lr_at(cfg, 700 + x) + G.lr_at(cfg, 18865 - x) == pytest.approx(6e-4, rel=1e-12)
    # midpoint of the decay is half the peak
    assert G.lr_at(cfg, 700 + span // 2) == pytest.approx(3e-4, abs=1e-7)
    assert G.lr_at(cfg, 18864) < 1e-10
    lrs = [G.lr_at(cfg, s) for s in range(700, 18865, 97)]
    assert all(a >= b for a, b in zip(lrs, lrs[1:]))
    tiny = cfg_of("tiny")
    assert G.lr_at(tiny, 0) == 6e-4


# --- clip and AdamW closed forms (numbat §4.3) ---------------------------------------------

def _rand_state(cfg, seed, gscale):
    rng = np.random.default_rng(seed)
    p = {k: rng.standard_normal(s) * 0.05 for k, s, _ in G.param_shapes(cfg)}
    g = {k: rng.standard_normal(s) * gscale for k, s, _ in G.param_shapes(cfg)}
    return p, g


def _flat(d):
    return np.concatenate([np.asarray(d[k], np.float64).ravel() for k in G.KIND_NAMES])


MICRO = dict(n_layer=2, n_head=2, n_embd=16, seq_len=8, vocab_real=37, micro_batch=2,
             warmup_steps=10, total_steps=100)


@pytest.mark.parametrize("gscale", [1e-4, 1.0])
def test_adamw_first_step_closed_form(gscale):
    cfg = G.Config(**MICRO)
    p0, g = _rand_state(cfg, 1, gscale)
    p = {k: a.copy() for k, a in p0.items()}
    m, v = G.zeros_like_params(cfg), G.zeros_like_params(cfg)
    accum, step = 3, 0
    norm = G.clip_adamw(cfg, p, g, m, v, step, accum=accum)
    gbar = _flat(g) / accum
    assert norm == pytest.approx(np.linalg.norm(gbar), rel=1e-12)
    k = min(1.0, 1.0 / np.linalg.norm(gbar))
    lr = G.lr_at(cfg, step)
    for name, _, is2d in G.param_shapes(cfg):
        gh = g[name] / accum * k
        exp = p0[name] - lr * (gh / (np.abs(gh) + cfg.eps) + (cfg.weight_decay * p0[name] if is2d else 0))
        np.testing.assert_allclose(p[name], exp, rtol=1e-12, atol=1e-15)
    if gscale == 1.0:
        # clipped: the first moment is (1 - beta1) times a unit-norm gradient
        assert np.linalg.norm(_flat(m)) == pytest.approx(1.0 - cfg.beta1, rel=1e-12)


def test_adamw_epsilon_regime():
    cfg = G.Config(**MICRO)
    p0, _ = _rand_state(cfg, 2, 1.0)
    g = {k: np.full(s, 1e-9) for k, s, _ in G.param_shapes(cfg)}
    p = {k: a.copy() for k, a in p0.items()}
    G.clip_adamw(cfg, p, g, G.zeros_like_params(cfg), G.zeros_like_params(cfg), 0)
    lr = G.lr_at(cfg, 0)
    # |g| = 1e-9 against eps 1e-8: the normalised step is 1e-9 / 1.1e-8
    np.testing.assert_allclose(p["ln1b"], p0["ln1b"] - lr * (1e-9 / 1.1e-8), rtol=1e-9)


def test_adamw_second_step_closed_form():
    cfg = G.Config(**MICRO)
    p0, g1 = _rand_state(cfg, 3, 1e-4)
    _, g2 = _rand_state(cfg, 4, 1e-4)
    p = {k: a.copy() for k, a in p0.items()}
    m, v = G.zeros_like_params(cfg), G.zeros_like_params(cfg)
    G.clip_adamw(cfg, p, g1, m, v, 0)
    p1 = {k: a.copy() for k, a in p.items()}
    G.clip_adamw(cfg, p, g2, m, v, 1)
    b1, b2, lr2 = cfg.beta1, cfg.beta2, G.lr_at(cfg, 1)
    for name, _, is2d in G.param_shapes(cfg):
        mh = (b1 * g1[name] + g2[name]) / (1 + b1)
        vh = (b2 * g1[name] ** 2 + g2[name] ** 2) / (1 + b2)
        exp = p1[name] - lr2 * (mh / (np.sqrt(vh) + cfg.eps) + (cfg.weight_decay * p1[name] if is2d else 0))
        np.testing.assert_allclose(p[name], exp, rtol=1e-10, atol=1e-14)


def test_decay_only_on_2d_weights():
    cfg = G.Config(**MICRO)
    p0, _ = _rand_state(cfg, 5, 1.0)
    zero = G.zeros_like_params(cfg)
    p = {k: a.copy() for k, a in p0.items()}
    G.clip_adamw(cfg, p, zero, G.zeros_like_params(cfg), G.zeros_like_params(cfg), 3)
    lr = G.lr_at(cfg, 3)
    for name, _, is2d in G.param_shapes(cfg):
        exp = p0[name] * (1 - lr * cfg.weight_decay) if is2d else p0[name]
        np.testing.assert_allclose(p[name], exp, rtol=1e-14)
    assert {n for n, _, d in G.param_shapes(cfg) if d} == {"wte", "wpe", "qkvw", "attprojw", "fcw", "fcprojw"}


# --- synthetic inputs --------------------------------------------------------------------

def test_zipf_stream_statistics():
    V = 50257
    s = synth.zipf_document_stream(400_000, V, V - 1, 1000, 1337)
    assert s.min() >= 0 and s.max() == V - 1
    frac_eot = np.mean(s == V - 1)
    assert abs(frac_eot - 1 / 1001) < 3e-4
    doc = s[s != V - 1]
    H = np.sum(np.arange(1, V, dtype=np.float64) ** -1.1)
    assert abs(np.mean(doc == 0) - 1 / H) < 3e-3
    assert abs(np.mean(doc == 1) - 2 ** -1.1 / H) < 3e-3
    x, y = synth.windows(s, 4, 1024)
    assert np.array_equal(x[:, 1:], y[:, :-1])


# --- masked-target cross-entropy (an ignore index per target) -------------------------------

def test_masked_ce_without_ignored_rows_is_plain_ce():
    rng = np.random.default_rng(7)
    z = rng.standard_normal((5, 24))
    t = rng.integers(0, 20, 5)
    l0, d0 = G.softmax_ce(z, t, 20)
    l1, d1, n = G.softmax_ce_masked(z, t, 20)
    assert n == 5
    np.testing.assert_allclose(l1, l0, rtol=0, atol=0)
    np.testing.assert_allclose(d1, d0, rtol=0, atol=0)


def test_masked_ce_all_ignored_is_zero():
    z = np.random.default_rng(8).standard_normal((3, 8))
    l, d, n = G.softmax_ce_masked(z, np.full(3, -1), 6)
    assert n == 0 and not l.any() and not d.any()


def test_masked_ce_gradient_by_finite_differences():
    """The gradient is that of the mean loss over the kept rows (central
    differences in fp64); ignored rows and padded columns get exactly zero."""
    rng = np.random.default_rng(9)
    N, V, Vp = 6, 10, 16
    z = rng.standard_normal((N, Vp))
    t = np.array([2, -1, 7, -1, 0, 9])
    _, dz, n = G.softmax_ce_masked(z, t, V)
    assert n == 4
    keep = t != -1

    def mean_loss(zz):
        zr = zz[:, :V]
        m = zr.max(axis=1)
        lse = m + np.log(np.exp(zr - m[:, None]).sum(axis=1))
        return np.mean((lse - zz[np.arange(N), np.where(keep, t, 0)])[keep])

    h = 1e-6
    num = np.zeros_like(z)
    for i in range(N):
        for j in range(Vp):
            zp, zm = z.copy(), z.copy()
            zp[i, j] += h
            zm[i, j] -= h
            num[i, j] = (mean_loss(zp) - mean_loss(zm)) / (2 * h)
    np.testing.assert_allclose(dz, num, atol=1e-8)
    assert not dz[~keep].any() and not dz[:, V:].any()
