"""How close any bf16-activation implementation can come to the fp64 definition.

The recipe stores activations in bfloat16 ("Pretraining and adapting a language
model on a dependency-free stack", §4.3). This test re-runs the oracle's tiny
step with every activation and activation gradient rounded to bf16 at the
tensor boundaries where the CUDA path stores them (all math otherwise fp64) and
measures how far its first-step weights land from the exact oracle. That floor
(~1.3e-3 relative L2 at lr 6e-4) is above 1e-3 because the first Adam step is a
sign decision per element; the GPU parity test therefore applies the 1e-3 bar to
the sign-determined elements. No GPU needed.
"""
import numpy as np
import torch

from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G


def R(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


def fwd_bwd_bf16_storage(cfg, p, x, y):
    B, T = x.shape
    C, H, hd = cfg.C, cfg.H, cfg.hd
    W = {k: (R(v) if k in ("wte", "wpe", "qkvw", "attprojw", "fcw", "fcprojw") else v) for k, v in p.items()}
    h = R(W["wte"][x] + W["wpe"][:T][None])
    cache = []
    for l in range(cfg.L):
        c = {"x": h}
        a, c["m1"], c["s1"] = G.layernorm_fwd(h, p["ln1w"][l], p["ln1b"][l])
        c["a"] = a = R(a)
        qkv = R(a @ W["qkvw"][l].T + p["qkvb"][l])
        c["q"], c["k"], c["v"] = (qkv[..., i * C:(i + 1) * C].reshape(B, T, H, hd).transpose(0, 2, 1, 3) for i in range(3))
        o, _ = G.attention_fwd(c["q"], c["k"], c["v"])
        c["y"] = R(o.transpose(0, 2, 1, 3).reshape(B, T, C))
        c["hm"] = hm = R(h + c["y"] @ W["attprojw"][l].T + p["attprojb"][l])
        b, c["m2"], c["s2"] = G.layernorm_fwd(hm, p["ln2w"][l], p["ln2b"][l])
        c["b"] = b = R(b)
        u = b @ W["fcw"][l].T + p["fcb"][l]
        c["g"], c["u"] = R(G.gelu_fwd(u)), R(u)
        h = R(hm + c["g"] @ W["fcprojw"][l].T + p["fcprojb"][l])
        cache.append(c)
    f, mf, sf = G.layernorm_fwd(h, p["lnfw"], p["lnfb"])
    f = R(f)
    z = R(f.reshape(B * T, C) @ W["wte"].T)
    losses, dz = G.softmax_ce(z, y.reshape(-1), cfg.V)
    dz = R(dz)
    g = G.zeros_like_params(cfg)
    g["wte"] += dz.T @ f.reshape(B * T, C)
    dx, g["lnfw"], g["lnfb"] = G.layernorm_bwd(R(dz @ W["wte"]).reshape(B, T, C), h, mf, sf, p["lnfw"])
    dx = R(dx)
    for l in reversed(range(cfg.L)):
        c = cache[l]
        d2 = dx.reshape(B * T, C)
        g["fcprojw"][l], g["fcprojb"][l] = d2.T @ c["g"].reshape(B * T, 4 * C), d2.sum(0)
        du = R(G.gelu_bwd(c["u"], dx @ W["fcprojw"][l]))
        g["fcw"][l], g["fcb"][l] = du.reshape(B * T, 4 * C).T @ c["b"].reshape(B * T, C), du.reshape(B * T, 4 * C).sum(0)
        dxm, g["ln2w"][l], g["ln2b"][l] = G.layernorm_bwd(R(du @ W["fcw"][l]), c["hm"], c["m2"], c["s2"], p["ln2w"][l])
        dx = R(dx + dxm)
        d2 = dx.reshape(B * T, C)
        g["attprojw"][l], g["attprojb"][l] = d2.T @ c["y"].reshape(B * T, C), d2.sum(0)
        dy = R(dx @ W["attprojw"][l]).reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        dq, dk, dv = G.attention_bwd(dy, c["q"], c["k"], c["v"])
        dqkv = R(np.concatenate([t.transpose(0, 2, 1, 3).reshape(B, T, C) for t in (dq, dk, dv)], -1))
        g["qkvw"][l], g["qkvb"][l] = dqkv.reshape(B * T, 3 * C).T @ c["a"].reshape(B * T, C), dqkv.reshape(B * T, 3 * C).sum(0)
        dxi, g["ln1w"][l], g["ln1b"][l] = G.layernorm_bwd(R(dqkv @ W["qkvw"][l]), c["x"], c["m1"], c["s1"], p["ln1w"][l])
        dx = R(dx + dxi)
    np.add.at(g["wte"], x.reshape(-1), dx.reshape(B * T, C))
    g["wpe"][:T] += dx.sum(0)
    return float(losses.mean()), g


def test_bf16_storage_floor_of_the_first_step():
    cfg = G.Config(**workloads.model_args("tiny"))
    p = G.init_params(cfg, 1337)
    x, y = synth.uniform_next_token_batch(cfg.micro_batch, cfg.T, cfg.V, 1337)
    l_ref, g_ref = G.fwd_bwd(cfg, p, x, y)
    l_bf, g_bf = fwd_bwd_bf16_storage(cfg, p, x, y)
    assert abs(l_bf - l_ref) < 1e-3
    rels = [np.linalg.norm(g_bf[k] - g_ref[k]) / np.linalg.norm(g_ref[k]) for k in G.KIND_NAMES]
    assert 1e-3 < float(np.median(rels)) < 2e-2       # bf16 noise, well inside the 3e-2 bar

    def after_step(g):
        q = {k: v.copy() for k, v in p.items()}
        G.clip_adamw(cfg, q, g, G.zeros_like_params(cfg), G.zeros_like_params(cfg), 0)
        return np.concatenate([q[k].ravel() for k in G.KIND_NAMES])
    a, b = after_step(g_bf), after_step(g_ref)
    floor = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < floor < 2e-3, floor
