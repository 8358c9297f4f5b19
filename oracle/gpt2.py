"""CPU oracle for one GPT-2 training step -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this module. The CUDA product path never calls it, and the two share no
code: the only common dependency is the seeded input generator
``gpt_step_b200.synth`` (which holds none of the method's arithmetic).

What it computes is the plain definition of the step the pages fix, written as
direct numpy in fp64 (a matrix product is the only library primitive used):

* model -- "Pretraining and adapting a language model on a dependency-free
  stack" (arXiv 2609.28568; cited below as [numbat]), §4.1 and Fig. 1: GPT-2
  decoder, pre-LayerNorm blocks with residuals around attention and MLP, tied
  input/output embeddings, learned token and position embeddings, causal
  scaled dot-product multi-head attention (grow_a_language_model_intro,
  activities 4-7), final LayerNorm before the tied head (the 148 named
  gradient tensors of [numbat] §5.1 include it);
* vocabulary padded to a multiple of 128, softmax and its gradient over the
  real ids only ([numbat] §4.1);
* N(0, 0.02) initialisation, residual-writing projections scaled by
  1/sqrt(2L) ([numbat] §4.1), drawn from the Philox generator in
  ``oracle.philox``;
* cross-entropy loss, mean over positions ([numbat] §4.3, §5.6);
* global-norm clip 1.0 and AdamW (0.9, 0.95), eps 1e-8, weight decay 0.1 on
  2-D weights only, linear warmup then cosine decay ([numbat] §4.3).

Readings where the pages are silent (each listed in the repository's design
notes): tanh-approximation GELU; LayerNorm eps 1e-5 with biased variance;
LayerNorm gains 1 and all biases 0 at init; padded embedding rows start at 0;
attention scale 1/sqrt(head_dim) with the diagonal visible; no dropout; loss
averaged over all positions of a micro-step and gradients averaged over
micro-steps; clip scale min(1, clip / ||g||) with no epsilon; bias-corrected
AdamW with t = step + 1 and decoupled decay on the pre-update weight.

Everything is fp64 unless a caller passes fp32 arrays to the AdamW helper.
Parity unpinned: nothing -- every function here is checked by a test in
tests/test_oracle_*.py against finite differences, closed forms, invariants,
brute force or an independent library computation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import philox

F64 = np.float64
LN_EPS = 1e-5

# The 16 parameter kinds in storage order, each stored as one tensor-major
# array ([L, ...] for per-layer kinds). "2-D" marks the weights that take
# weight decay ([numbat] §4.3: decay on two-dimensional weights only).
KINDS = [
    # name,        shape fn,                                2-D,  init
    ("wte",      lambda c: (c.Vp, c.C),               True,  "normal"),
    ("wpe",      lambda c: (c.T, c.C),                True,  "normal"),
    ("ln1w",     lambda c: (c.L, c.C),                False, "ones"),
    ("ln1b",     lambda c: (c.L, c.C),                False, "zeros"),
    ("qkvw",     lambda c: (c.L, 3 * c.C, c.C),       True,  "normal"),
    ("qkvb",     lambda c: (c.L, 3 * c.C),            False, "zeros"),
    ("attprojw", lambda c: (c.L, c.C, c.C),           True,  "scaled"),
    ("attprojb", lambda c: (c.L, c.C),                False, "zeros"),
    ("ln2w",     lambda c: (c.L, c.C),                False, "ones"),
    ("ln2b",     lambda c: (c.L, c.C),                False, "zeros"),
    ("fcw",      lambda c: (c.L, 4 * c.C, c.C),       True,  "normal"),
    ("fcb",      lambda c: (c.L, 4 * c.C),            False, "zeros"),
    ("fcprojw",  lambda c: (c.L, c.C, 4 * c.C),       True,  "scaled"),
    ("fcprojb",  lambda c: (c.L, c.C),                False, "zeros"),
    ("lnfw",     lambda c: (c.C,),                    False, "ones"),
    ("lnfb",     lambda c: (c.C,),                    False, "zeros"),
]
KIND_NAMES = [k[0] for k in KINDS]

# Per-layer tensor names in the order the pages' 148-gradient count implies
# (wte, wpe, 12 per block, final LayerNorm weight and bias).
_LAYER_NAMES = [
    ("ln1w", "ln_1.weight"), ("ln1b", "ln_1.bias"),
    ("qkvw", "attn.c_attn.weight"), ("qkvb", "attn.c_attn.bias"),
    ("attprojw", "attn.c_proj.weight"), ("attprojb", "attn.c_proj.bias"),
    ("ln2w", "ln_2.weight"), ("ln2b", "ln_2.bias"),
    ("fcw", "mlp.c_fc.weight"), ("fcb", "mlp.c_fc.bias"),
    ("fcprojw", "mlp.c_proj.weight"), ("fcprojb", "mlp.c_proj.bias"),
]


@dataclass
class Config:
    """Model and optimiser configuration (names follow GPT-2 and [numbat] §4.1, §4.3)."""
    n_layer: int
    n_head: int
    n_embd: int
    seq_len: int
    vocab_real: int
    vocab_padded: int = 0          # 0: round vocab_real up to a multiple of 128
    micro_batch: int = 1
    grad_accum: int = 1
    max_lr: float = 6e-4
    min_lr: float = 0.0
    warmup_steps: int = 700
    total_steps: int = 18865
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    weight_decay: float = 0.1
    grad_clip: float = 1.0
    extra: dict = field(default_factory=dict)

    @property
    def L(self): return self.n_layer

    @property
    def H(self): return self.n_head

    @property
    def C(self): return self.n_embd

    @property
    def T(self): return self.seq_len

    @property
    def V(self): return self.vocab_real

    @property
    def Vp(self):
        if self.vocab_padded:
            return self.vocab_padded
        return ((self.vocab_real + 127) // 128) * 128

    @property
    def hd(self): return self.n_embd // self.n_head


def param_shapes(cfg: Config):
    """[(kind, shape, is_2d)] in storage order."""
    return [(name, fn(cfg), is2d) for name, fn, is2d, _ in KINDS]


def tensor_names(cfg: Config):
    """The named tensors ([numbat] §4.5/§5.1 count 148 for 12 blocks): (name, kind, layer, shape)."""
    out = [("wte.weight", "wte", -1, (cfg.Vp, cfg.C)), ("wpe.weight", "wpe", -1, (cfg.T, cfg.C))]
    shapes = {k: s[1:] for k, s, _ in param_shapes(cfg)}
    for l in range(cfg.L):
        for kind, nm in _LAYER_NAMES:
            out.append((f"h.{l}.{nm}", kind, l, shapes[kind]))
    out.append(("ln_f.weight", "lnfw", -1, (cfg.C,)))
    out.append(("ln_f.bias", "lnfb", -1, (cfg.C,)))
    return out


def count_params(cfg: Config, padded: bool = False) -> int:
    """Parameter count; the pages' 124,439,808 counts real vocabulary rows only."""
    n = 0
    for name, shape, _ in param_shapes(cfg):
        sz = int(np.prod(shape))
        if name == "wte" and not padded:
            sz = cfg.V * cfg.C
        n += sz
    return n


# ----------------------------------------------------------------------------
# initialisation ([numbat] §4.1)
# ----------------------------------------------------------------------------

def init_params(cfg: Config, seed: int) -> dict:
    """N(0, 0.02) weights, residual-writing projections x 1/sqrt(2L), LN 1/0, biases 0.

    Kind index k of KINDS selects Philox stream k; padded vocabulary rows are 0.
    """
    p = {}
    for k, (name, fn, _, init) in enumerate(KINDS):
        shape = fn(cfg)
        n = int(np.prod(shape))
        if init == "ones":
            a = np.ones(shape, F64)
        elif init == "zeros":
            a = np.zeros(shape, F64)
        else:
            std = 0.02 if init == "normal" else 0.02 / math.sqrt(2 * max(1, cfg.L))
            a = (philox.normals(k, n, seed) * std).reshape(shape)
            if name == "wte":
                a[cfg.V:, :] = 0.0
        p[name] = a
    return p


def zeros_like_params(cfg: Config) -> dict:
    return {name: np.zeros(fn(cfg), F64) for name, fn, _, _ in KINDS}


# ----------------------------------------------------------------------------
# building blocks
# ----------------------------------------------------------------------------

def layernorm_fwd(x, w, b):
    """LayerNorm over the last axis; fp64 statistics, biased variance, eps 1e-5."""
    mean = x.mean(axis=-1, keepdims=True)
    xc = x - mean
    var = (xc * xc).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + LN_EPS)
    xhat = xc * rstd
    return xhat * w + b, mean[..., 0], rstd[..., 0]


def layernorm_bwd(dy, x, mean, rstd, w):
    """Gradient of layernorm_fwd: returns dx, dw, db (dw, db summed over rows)."""
    xhat = (x - mean[..., None]) * rstd[..., None]
    dxhat = dy * w
    C = x.shape[-1]
    m1 = dxhat.sum(axis=-1, keepdims=True) / C
    m2 = (dxhat * xhat).sum(axis=-1, keepdims=True) / C
    dx = (dxhat - m1 - xhat * m2) * rstd[..., None]
    red = tuple(range(dy.ndim - 1))
    return dx, (dy * xhat).sum(axis=red), dy.sum(axis=red)


GELU_K = math.sqrt(2.0 / math.pi)


def gelu_fwd(u):
    """GPT-2's tanh-approximation GELU."""
    return 0.5 * u * (1.0 + np.tanh(GELU_K * (u + 0.044715 * u ** 3)))


def gelu_bwd(u, dg):
    """dg * GELU'(u) for the tanh approximation."""
    t = np.tanh(GELU_K * (u + 0.044715 * u ** 3))
    d = 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * GELU_K * (1.0 + 3.0 * 0.044715 * u * u)
    return dg * d


def attention_fwd(q, k, v):
    """Causal softmax(q k^T / sqrt(hd)) v, explicit O(T^2); q, k, v [..., T, hd].

    Returns the output and the per-row log-sum-exp of the scaled, masked scores.
    """
    T, hd = q.shape[-2], q.shape[-1]
    s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(hd)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)      # key j > query i is hidden
    s = np.where(mask, -np.inf, s)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    p = e / z
    return p @ v, (m + np.log(z))[..., 0]


def attention_bwd(do, q, k, v):
    """Gradients of attention_fwd w.r.t. q, k, v (probabilities recomputed)."""
    T, hd = q.shape[-2], q.shape[-1]
    scale = 1.0 / math.sqrt(hd)
    s = (q @ np.swapaxes(k, -1, -2)) * scale
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    s = np.where(mask, -np.inf, s)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    p /= p.sum(axis=-1, keepdims=True)
    dv = np.swapaxes(p, -1, -2) @ do
    dp = do @ np.swapaxes(v, -1, -2)
    ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
    dq = (ds @ k) * scale
    dk = (np.swapaxes(ds, -1, -2) @ q) * scale
    return dq, dk, dv


def softmax_ce(z, targets, V):
    """Vocabulary-masked cross-entropy ([numbat] §4.1): softmax over ids < V only.

    z [N, Vp] logits, targets [N]. Returns per-row losses [N] and the gradient of
    the MEAN loss w.r.t. z (exactly zero in the padded columns >= V).
    """
    N = z.shape[0]
    zr = z[:, :V]
    m = zr.max(axis=1, keepdims=True)
    e = np.exp(zr - m)
    ssum = e.sum(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(ssum[:, 0])
    losses = lse - z[np.arange(N), targets]
    dz = np.zeros_like(z)
    dz[:, :V] = e / ssum
    dz[np.arange(N), targets] -= 1.0
    dz /= N
    return losses, dz


def softmax_ce_masked(z, targets, V, ignore_index=-1):
    """Cross-entropy with an ignore index per target: the loss is taken only on
    chosen positions ("Pretraining and adapting a language model on a
    dependency-free stack" takes the adapter's loss on answers rather than
    questions). Rows whose target equals `ignore_index` contribute loss 0 and a
    gradient of exactly zero; the others are softmax_ce's rows, and the mean is
    over the kept rows only.

    z [N, Vp], targets [N]. Returns (per-row losses [N], dz of the mean loss over
    kept rows, number of kept rows).
    """
    keep = targets != ignore_index
    n_keep = int(keep.sum())
    losses = np.zeros(z.shape[0])
    dz = np.zeros_like(z)
    if n_keep:
        lk, dk = softmax_ce(z[keep], targets[keep], V)
        losses[keep] = lk
        dz[keep] = dk           # softmax_ce of the kept rows already divides by n_keep
    return losses, dz, n_keep


# ----------------------------------------------------------------------------
# forward / backward of the whole model
# ----------------------------------------------------------------------------

def forward(cfg: Config, p: dict, tokens: np.ndarray, targets: np.ndarray | None = None):
    """Forward pass; returns (mean loss or None, per-position losses or None, cache)."""
    B, T = tokens.shape
    C, H, hd = cfg.C, cfg.H, cfg.hd
    if tokens.min() < 0 or tokens.max() >= cfg.V:
        raise ValueError("token id out of range")
    x = p["wte"][tokens] + p["wpe"][:T][None]
    cache = {"tokens": tokens, "layers": []}
    for l in range(cfg.L):
        lc = {"x_in": x}
        a, lc["ln1_mean"], lc["ln1_rstd"] = layernorm_fwd(x, p["ln1w"][l], p["ln1b"][l])
        lc["ln1"] = a
        qkv = a @ p["qkvw"][l].T + p["qkvb"][l]
        q, k, v = (qkv[..., i * C:(i + 1) * C].reshape(B, T, H, hd).transpose(0, 2, 1, 3)
                   for i in range(3))
        o, lse = attention_fwd(q, k, v)
        lc["q"], lc["k"], lc["v"], lc["lse"] = q, k, v, lse
        y = o.transpose(0, 2, 1, 3).reshape(B, T, C)
        lc["atty"] = y
        x = x + y @ p["attprojw"][l].T + p["attprojb"][l]
        lc["x_mid"] = x
        b, lc["ln2_mean"], lc["ln2_rstd"] = layernorm_fwd(x, p["ln2w"][l], p["ln2b"][l])
        lc["ln2"] = b
        u = b @ p["fcw"][l].T + p["fcb"][l]
        g = gelu_fwd(u)
        lc["fch"], lc["fchg"] = u, g
        x = x + g @ p["fcprojw"][l].T + p["fcprojb"][l]
        cache["layers"].append(lc)
    cache["x_final"] = x
    f, cache["lnf_mean"], cache["lnf_rstd"] = layernorm_fwd(x, p["lnfw"], p["lnfb"])
    cache["lnf"] = f
    z = f.reshape(B * T, C) @ p["wte"].T               # tied head over all Vp rows
    cache["logits"] = z
    if targets is None:
        return None, None, cache
    losses, dz = softmax_ce(z, targets.reshape(-1), cfg.V)
    cache["dz"] = dz
    return float(losses.mean()), losses.reshape(B, T), cache


def backward(cfg: Config, p: dict, cache: dict) -> dict:
    """Gradients of the mean loss w.r.t. every parameter kind."""
    g = zeros_like_params(cfg)
    tokens = cache["tokens"]
    B, T = tokens.shape
    C, H, hd = cfg.C, cfg.H, cfg.hd
    dz = cache["dz"]
    f = cache["lnf"].reshape(B * T, C)
    g["wte"] += dz.T @ f
    df = (dz @ p["wte"]).reshape(B, T, C)
    dx, g["lnfw"], g["lnfb"] = layernorm_bwd(df, cache["x_final"], cache["lnf_mean"],
                                             cache["lnf_rstd"], p["lnfw"])
    for l in reversed(range(cfg.L)):
        lc = cache["layers"][l]
        # MLP branch: x_out = x_mid + GELU(LN2(x_mid) Wfc^T + bfc) Wfp^T + bfp
        dflat = dx.reshape(B * T, C)
        g["fcprojw"][l] = dflat.T @ lc["fchg"].reshape(B * T, 4 * C)
        g["fcprojb"][l] = dflat.sum(0)
        dgl = dx @ p["fcprojw"][l]
        du = gelu_bwd(lc["fch"], dgl)
        duf = du.reshape(B * T, 4 * C)
        g["fcw"][l] = duf.T @ lc["ln2"].reshape(B * T, C)
        g["fcb"][l] = duf.sum(0)
        db_ = du @ p["fcw"][l]
        dxm, g["ln2w"][l], g["ln2b"][l] = layernorm_bwd(db_, lc["x_mid"], lc["ln2_mean"],
                                                        lc["ln2_rstd"], p["ln2w"][l])
        dx = dx + dxm
        # attention branch: x_mid = x_in + Attn(LN1(x_in)) Wap^T + bap
        dflat = dx.reshape(B * T, C)
        g["attprojw"][l] = dflat.T @ lc["atty"].reshape(B * T, C)
        g["attprojb"][l] = dflat.sum(0)
        dy = dx @ p["attprojw"][l]
        do = dy.reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        dq, dk, dv = attention_bwd(do, lc["q"], lc["k"], lc["v"])
        dqkv = np.concatenate([t.transpose(0, 2, 1, 3).reshape(B, T, C) for t in (dq, dk, dv)],
                              axis=-1)
        dqf = dqkv.reshape(B * T, 3 * C)
        g["qkvw"][l] = dqf.T @ lc["ln1"].reshape(B * T, C)
        g["qkvb"][l] = dqf.sum(0)
        da = dqkv @ p["qkvw"][l]
        dxi, g["ln1w"][l], g["ln1b"][l] = layernorm_bwd(da, lc["x_in"], lc["ln1_mean"],
                                                        lc["ln1_rstd"], p["ln1w"][l])
        dx = dx + dxi
    # embeddings: x0 = wte[tok] + wpe[t]
    np.add.at(g["wte"], tokens.reshape(-1), dx.reshape(B * T, C))
    g["wpe"][:T] += dx.sum(axis=0)
    return g


def fwd_bwd(cfg: Config, p: dict, tokens, targets):
    """Mean loss of one micro-batch and the gradient of that mean loss."""
    loss, _, cache = forward(cfg, p, tokens, targets)
    return loss, backward(cfg, p, cache)


def token_losses(cfg: Config, p: dict, tokens, targets):
    """Per-position losses [B, T] (forward only)."""
    _, losses, _ = forward(cfg, p, tokens, targets)
    return losses


# ----------------------------------------------------------------------------
# optimiser ([numbat] §4.3)
# ----------------------------------------------------------------------------

def lr_at(cfg: Config, step: int) -> float:
    """Linear warmup over warmup_steps to max_lr, then cosine to min_lr at total_steps.

    Step is 0-based: warmup gives max_lr * (step + 1) / warmup_steps.
    """
    if step < cfg.warmup_steps:
        return cfg.max_lr * (step + 1) / cfg.warmup_steps
    span = max(1, cfg.total_steps - cfg.warmup_steps)
    ratio = min(1.0, (step - cfg.warmup_steps) / span)
    coeff = 0.5 * (1.0 + math.cos(math.pi * ratio))
    return cfg.min_lr + coeff * (cfg.max_lr - cfg.min_lr)


def global_norm(grads: dict, accum: int = 1) -> float:
    """||g / accum||_2 over every parameter of every kind."""
    s = 0.0
    for name in KIND_NAMES:
        a = np.asarray(grads[name], dtype=F64) / accum
        s += float((a * a).sum())
    return math.sqrt(s)


def clip_adamw(cfg: Config, params: dict, grads: dict, m: dict, v: dict, step: int,
               accum: int = 1) -> float:
    """One clipped AdamW step in place (fp64 arithmetic); returns the pre-clip norm.

    g_bar = g / accum; scale = min(1, clip / ||g_bar||); m, v are Adam's moment
    estimates with bias correction at t = step + 1; decay lambda * w is added
    (times lr) for 2-D weights only.
    """
    norm = global_norm(grads, accum)
    scale = min(1.0, cfg.grad_clip / norm) if norm > 0 else 1.0
    lr = lr_at(cfg, step)
    t = step + 1
    bc1 = 1.0 - cfg.beta1 ** t
    bc2 = 1.0 - cfg.beta2 ** t
    for name, _, is2d, _ in KINDS:
        gk = np.asarray(grads[name], dtype=F64) / accum * scale
        mk = cfg.beta1 * np.asarray(m[name], F64) + (1.0 - cfg.beta1) * gk
        vk = cfg.beta2 * np.asarray(v[name], F64) + (1.0 - cfg.beta2) * gk * gk
        w = np.asarray(params[name], F64)
        upd = (mk / bc1) / (np.sqrt(vk / bc2) + cfg.eps)
        if is2d:
            upd = upd + cfg.weight_decay * w
        params[name] = w - lr * upd
        m[name] = mk
        v[name] = vk
    return norm


def train_step(cfg: Config, params: dict, m: dict, v: dict, step: int, batches):
    """accum micro-steps of fwd_bwd then clip_adamw; returns (mean loss, norm)."""
    acc = zeros_like_params(cfg)
    losses = []
    for tokens, targets in batches:
        loss, g = fwd_bwd(cfg, params, tokens, targets)
        losses.append(loss)
        for k in KIND_NAMES:
            acc[k] += g[k]
    norm = clip_adamw(cfg, params, acc, m, v, step, accum=len(losses))
    return float(np.mean(losses)), norm


def split_named(cfg: Config, arrays: dict) -> dict:
    """View kind arrays as the named tensors of tensor_names()."""
    out = {}
    for name, kind, layer, _ in tensor_names(cfg):
        out[name] = arrays[kind] if layer < 0 else arrays[kind][layer]
    return out
