"""Parity at the sizes the benchmark runs: GPT-2 124M, micro-batch 19, T = 1024.

The launch configuration is the one `bench.py` times, so the code paths that
only run at full size are compared with the oracle here:

* the persistent attention backward, whose CTAs take many (key block, head)
  work items each (19 x 12 heads x 8 key blocks = 1,824 items over the SMs),
  with every output compared element by element;
* the tied lm_head's input gradient (a 50,304-long reduction) and the wte
  weight gradient over 19,456 rows, and the grouped input + weight gradient
  launches of the four linear layers of a block with the reduction splits the
  host chooses at this size, on sampled output rows the oracle computes one by
  one; their inputs are small multiples of 1/4, so every fp32 partial sum is
  exact and the expected value is known exactly;
* all 148 gradients of the whole 124M step at micro-batch 19 against the
  oracle. The batch holds three distinct sequences, repeated; the gradient of
  the batch-mean loss is then the count-weighted mean of the three
  single-sequence gradients (linearity of the mean), which the oracle computes
  in three passes of one sequence each.
"""
import numpy as np
import pytest

import gpt_step_b200 as gs
from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G

from gpu_util import bf16, err_word, host, i32, rel_l2, require_gpu, rounded, torch

pytestmark = pytest.mark.gpu

B, T, H, HD, C, V, VP = 19, 1024, 12, 64, 768, 50257, 50304
M = B * T


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


# --- a4: attention with many work items per persistent CTA -------------------------------------

@pytest.mark.parametrize("Bt,HDt", [(3, 64), (4, 64), (19, 64), (16, 32)])
def test_attention_many_items_per_cta(Bt, HDt):
    """(Bt, 1024, 12, 64): 288, 384 and 1,824 backward work items against 148
    SMs, so most CTAs run the cross-item K/V prefetch and accumulator hand-over
    (288 = 148 + 140 ends on a partial pass taken in reversed order); and
    head size 32 at (16, 1024, 12) (the small configuration's attention, the
    forward on the tensor cores with 64-byte rows). The forward's persistent
    CTAs take 2 to 7 query tiles each. Every dQ, dK, dV element, the output,
    the lse and the qkv bias gradient are compared."""
    HD = HDt
    C = H * HD
    rng = np.random.default_rng(40 + Bt)
    qkv = rng.standard_normal((Bt, T, 3 * C)).astype(np.float32)
    do = rng.standard_normal((Bt, T, C)).astype(np.float32)
    qd = bf16(qkv)
    out = torch.empty(Bt, T, C, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(Bt, H, T, device="cuda")
    err = err_word()
    gs.attention_fwd(qd, out, lse, H, err)
    dqkv = torch.empty_like(qd)
    ws = torch.empty(gs.attention_bwd_workspace(Bt, T, H, HD), dtype=torch.uint8, device="cuda")
    dbias = torch.zeros(3 * C, device="cuda")
    gs.attention_bwd(qd, out, bf16(do), lse, dqkv, H, ws, err, dbias=dbias)
    got_o, got_l, got_d, got_b = host(out), host(lse), host(dqkv), host(dbias)
    assert int(err.sum()) == 0
    qr, dr = rounded(qkv), rounded(do)
    worst = {"o": 0.0, "dq": 0.0, "dk": 0.0, "dv": 0.0, "lse": 0.0}
    sums = np.zeros(3 * C)   # the qkv bias gradient: column sums of dq | dk | dv over all rows
    for b in range(Bt):     # the oracle one sequence at a time (its score matrices are T x T per head)
        q, k, v = (qr[b, :, i * C:(i + 1) * C].reshape(T, H, HD).transpose(1, 0, 2) for i in range(3))
        o, l = G.attention_fwd(q, k, v)
        dq, dk, dv = G.attention_bwd(dr[b].reshape(T, H, HD).transpose(1, 0, 2), q, k, v)
        worst["o"] = max(worst["o"], rel_l2(got_o[b], o.transpose(1, 0, 2).reshape(T, C)))
        worst["lse"] = max(worst["lse"], float(np.max(np.abs(got_l[b] - l))))
        for i, (name, ref) in enumerate((("dq", dq), ("dk", dk), ("dv", dv))):
            ref = ref.transpose(1, 0, 2).reshape(T, C)
            e = rel_l2(got_d[b, :, i * C:(i + 1) * C], ref)
            worst[name] = max(worst[name], e)
            sums[i * C:(i + 1) * C] += ref.sum(axis=0)
    print("attention worst per-sequence errors:", worst)
    assert worst["o"] < 1e-2 and worst["lse"] < 2e-3
    assert worst["dq"] < 2e-2 and worst["dk"] < 2e-2 and worst["dv"] < 2e-2
    assert rel_l2(got_b[:C], sums[:C]) < 2e-2
    assert np.all(got_b[C:2 * C] == 0.0) and np.max(np.abs(sums[C:2 * C])) < 1e-9 * np.max(np.abs(sums[:C]))
    assert rel_l2(got_b[2 * C:], sums[2 * C:]) < 1e-5


# --- a10, a3/a5/a7/a8 backward: full-size GEMMs on exact inputs -----------------------------------

def quarters(rng, shape):
    """int8 values in {-2..2}: the bf16 operand is value / 4 (exact)."""
    return rng.integers(-2, 3, size=shape, dtype=np.int8)


def dev_quarters(a):
    return (torch.from_numpy(a).cuda().to(torch.bfloat16) * 0.25).contiguous()


def sample_rows(n, k=40, seed=0):
    rng = np.random.default_rng(seed)
    r = np.concatenate([[0, 1, 255, 256, n // 2, n - 257, n - 2, n - 1], rng.choice(n, k, replace=False)])
    return np.unique(r)


def assert_bf16_of_exact(got, exact):
    """bf16 round-to-nearest of an exactly known value: within half a unit in the
    last place (bf16 keeps 8 significant bits: half an ulp is 2^(e - 8) for
    2^e <= |x| < 2^(e+1)), and exact zeros stay zero."""
    a = np.abs(exact)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8), 0.0)
    assert np.all(np.abs(got - exact) <= half_ulp), float(np.max(np.abs(got - exact) - half_ulp))


def test_lm_head_backward_full_size():
    """dlnf = dlogits . wte (K = 50,304, 786 k-blocks) and dwte += dlogits^T . lnf
    over 19,456 rows, exactly as the tied head's backward launches them."""
    rng = np.random.default_rng(50)
    dz = quarters(rng, (M, VP))
    wte = quarters(rng, (VP, C))
    h = quarters(rng, (M, C))
    dzd, wd, hd = dev_quarters(dz), dev_quarters(wte), dev_quarters(h)
    err = err_word()
    din = torch.empty(M, C, dtype=torch.bfloat16, device="cuda")
    gs.linear_dgrad(dzd, wd, None, din, err)
    dw0 = rng.standard_normal((VP, C)).astype(np.float32)
    dw = torch.tensor(dw0).cuda()
    gs.linear_wgrad(dzd, hd, dw, err)
    assert int(err.sum()) == 0
    rows = sample_rows(M, seed=51)
    exact = (dz[rows].astype(np.float64) @ wte.astype(np.float64)) / 16.0
    assert_bf16_of_exact(host(din[torch.tensor(rows).cuda()]), exact)
    vrows = sample_rows(VP, seed=52)
    exact_w = dw0[vrows].astype(np.float64) + (dz[:, vrows].astype(np.float64).T @ h.astype(np.float64)) / 16.0
    got_w = host(dw[torch.tensor(vrows).cuda()])
    # fp32 accumulation of exact partial sums onto an fp32 start value: one rounding per add at most
    assert rel_l2(got_w, exact_w) < 1e-6
    assert np.max(np.abs(got_w - exact_w)) <= 1e-5 * np.max(np.abs(exact_w))


# the four linear layers of a block in the backward: (name, N = output width of the layer, K = its input width, GELU')
LAYERS = [("mlp_proj", C, 4 * C, True), ("mlp_fc", 4 * C, C, False), ("attn_proj", C, C, False),
          ("qkv", 3 * C, C, False)]


@pytest.mark.parametrize("name,N,K,gelu", LAYERS)
def test_grouped_linear_backward_full_size(name, N, K, gelu):
    """One grouped launch of a layer's input gradient and weight gradient at
    M = 19,456 rows, with the weight gradient's reduction split the host picks
    for this size (the launch gpt2_fwd_bwd makes)."""
    rng = np.random.default_rng(60 + N + K)
    dout = quarters(rng, (M, N))
    w = quarters(rng, (N, K))
    inp = quarters(rng, (M, K))
    dd, wd, xd = dev_quarters(dout), dev_quarters(w), dev_quarters(inp)
    pre = rng.standard_normal((M, K)).astype(np.float32) if gelu else None
    pred = bf16(pre) if gelu else None
    din = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dw0 = rng.standard_normal((N, K)).astype(np.float32)
    dw = torch.tensor(dw0).cuda()
    cs0 = rng.standard_normal(K).astype(np.float32) if gelu else None
    cs = torch.tensor(cs0).cuda() if gelu else None
    err = err_word()
    splits = gs.linear_bwd(dd, wd, xd, pred, din, dw, cs, err)
    torch.cuda.synchronize()
    print(f"{name}: dw reduction split {splits}")
    assert splits >= 1 and int(err.sum()) == 0
    rows = sample_rows(M, seed=61)
    acc = (dout[rows].astype(np.float64) @ w.astype(np.float64)) / 16.0
    got = host(din[torch.tensor(rows).cuda()])
    if gelu:
        ref = G.gelu_bwd(rounded(pre[rows]), acc)
        assert rel_l2(got, ref) < 6e-3
        # the fused column sum (the MLP fc bias gradient) adds the stored bf16
        # values: against the exact sum it carries their rounding, and it equals
        # the column sums of what was stored up to fp32 addition order
        full = G.gelu_bwd(rounded(pre), (dout.astype(np.float64) @ w.astype(np.float64)) / 16.0)
        got_cs = host(cs) - cs0.astype(np.float64)
        assert rel_l2(got_cs, full.sum(0)) < 3e-3
        assert rel_l2(got_cs, host(din).sum(0)) < 1e-5
    else:
        assert_bf16_of_exact(got, acc)
    nrows = sample_rows(N, k=24, seed=62)
    exact_w = dw0[nrows].astype(np.float64) + (dout[:, nrows].astype(np.float64).T @ inp.astype(np.float64)) / 16.0
    got_w = host(dw[torch.tensor(nrows).cuda()])
    assert rel_l2(got_w, exact_w) < 1e-6
    assert np.max(np.abs(got_w - exact_w)) <= 1e-5 * np.max(np.abs(exact_w))


# --- the whole 124M step at micro-batch 19: every gradient ---------------------------------------

def test_gpt2_124m_all_gradients_at_micro_batch_19():
    args = workloads.model_args("gpt2_124m")
    assert args["micro_batch"] == B
    m = gs.GPT2(gs.Config.make(**args), 1337)
    ocfg = G.Config(**args)
    w = workloads.WORKLOADS["gpt2_124m"]
    src = synth.TokenSource(1, T, V, 1337, w["mean_doc_len"], 3)
    seqs = [src.get() for _ in range(3)]
    pattern = [0, 1, 2, 0, 0, 1, 2, 2, 1, 0, 2, 1, 0, 1, 2, 0, 2, 1, 0]    # 7 / 6 / 6, not periodic
    counts = np.bincount(pattern, minlength=3)
    x = np.concatenate([seqs[i][0] for i in pattern])
    y = np.concatenate([seqs[i][1] for i in pattern])
    loss = m.fwd_bwd(i32(x), i32(y), want_loss=True)
    grads = m.read_all(gs.GPT2_GRADS)
    cfg1 = G.Config(**workloads.model_args("gpt2_124m", micro_batch=1))
    p = G.init_params(cfg1, 1337)
    oloss, og = 0.0, None
    for i, (sx, sy) in enumerate(seqs):
        li, gi = G.fwd_bwd(cfg1, p, sx, sy)
        oloss += counts[i] * li / B
        og = {k: counts[i] * gi[k] / B for k in gi} if og is None else {k: og[k] + counts[i] * gi[k] / B for k in og}
    assert abs(loss - oloss) <= 2e-2, (loss, oloss)
    ogn = G.split_named(ocfg, og)
    assert len(grads) == 148
    errs = {n: rel_l2(a, ogn[n]) for n, a in grads.items()}
    worst = max(errs, key=errs.get)
    print(f"124M B=19: loss {loss:.5f} (oracle {oloss:.5f}); worst gradient {worst} rel L2 {errs[worst]:.3e}")
    assert errs[worst] <= 3e-2, (worst, errs[worst])
    assert np.all(grads["wte.weight"][V:] == 0.0)
    norm = m.clip_adamw(0, want_norm=True)
    onorm = G.global_norm(og)
    assert abs(norm - onorm) <= 3e-2 * onorm, (norm, onorm)
    m.close()
