"""Per-step parity: each CUDA kernel (called through the C ABI) against the oracle.

Inputs are seeded; the oracle sees the same bf16-rounded values the device
reads, and computes in fp64. Tolerances follow from the arithmetic: a bf16
output carries a relative rounding error of 2^-9, fp32 accumulations far less.
"""
import numpy as np
import pytest

import gpt_step_b200 as gs
from oracle import gpt2 as G

from gpu_util import bf16, err_word, f32, host, i32, rel_l2, require_gpu, rounded, torch

pytestmark = pytest.mark.gpu

BF16_TOL = 6e-3  # relative L2 for bf16-stored results of fp32 math


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --- a3/a5/a7/a8/a10: the tcgen05 GEMM in its three arrangements ---------------------------

GEMM_SHAPES = [(128, 256, 64), (256, 128, 128), (300, 384, 192), (1000, 768, 768),
               (77, 512, 1024), (512, 2304, 768), (640, 3200, 128)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_linear_fwd(M, N, K):
    x, w, b, r = rnd((M, K), 1), rnd((N, K), 2, 0.05), rnd(N, 3, 0.1), rnd((M, N), 4)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    err = err_word()
    gs.linear_fwd(bf16(x), bf16(w), f32(b), None, out, err)
    ref = rounded(x) @ rounded(w).T + b.astype(np.float32)
    assert rel_l2(host(out), ref) < BF16_TOL
    gs.linear_fwd(bf16(x), bf16(w), f32(b), bf16(r), out, err)
    ref = rounded(x) @ rounded(w).T + b.astype(np.float32) + rounded(r)
    assert rel_l2(host(out), ref) < BF16_TOL
    gs.linear_fwd(bf16(x), bf16(w), None, None, out, err)
    assert rel_l2(host(out), rounded(x) @ rounded(w).T) < BF16_TOL
    assert int(err.sum()) == 0


@pytest.mark.parametrize("M,N,K", [(256, 512, 128), (333, 1536, 384)])
def test_linear_fwd_gelu(M, N, K):
    x, w, b = rnd((M, K), 5), rnd((N, K), 6, 0.1), rnd(N, 7, 0.5)
    pre = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    g = torch.empty_like(pre)
    gs.linear_fwd_gelu(bf16(x), bf16(w), f32(b), pre, g, err_word())
    u = rounded(x) @ rounded(w).T + b.astype(np.float32)
    assert rel_l2(host(pre), u) < BF16_TOL
    assert rel_l2(host(g), G.gelu_fwd(u)) < BF16_TOL


@pytest.mark.parametrize("M,N,K", [(128, 64, 128), (300, 768, 256), (1024, 2304, 768), (192, 4480, 256)])
def test_linear_dgrad(M, N, K):
    dy, w, pre = rnd((M, N), 8), rnd((N, K), 9, 0.05), rnd((M, K), 10)
    din = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    gs.linear_dgrad(bf16(dy), bf16(w), None, din, err_word())
    ref = rounded(dy) @ rounded(w)
    assert rel_l2(host(din), ref) < BF16_TOL
    gs.linear_dgrad(bf16(dy), bf16(w), bf16(pre), din, err_word())
    assert rel_l2(host(din), G.gelu_bwd(rounded(pre), ref)) < BF16_TOL


@pytest.mark.parametrize("M,N,K,splits", [(128, 64, 64, 1), (256, 384, 128, 1), (2048, 768, 768, 0),
                                          (4096, 768, 3072, 0), (1024, 1024, 128, 4)])
def test_linear_wgrad(M, N, K, splits):
    dy, x = rnd((M, N), 11), rnd((M, K), 12)
    dw0 = rnd((N, K), 13)
    dw = f32(dw0)
    gs.linear_wgrad(bf16(dy), bf16(x), dw, err_word(), splits=splits)
    ref = dw0.astype(np.float32) + rounded(dy).T @ rounded(x)
    assert rel_l2(host(dw), ref) < 1e-5


@pytest.mark.parametrize("atomic", [False, True])
def test_bias_grad(atomic):
    """Column sums: deterministic two-pass with a workspace, one launch with fp32
    atomics without (the form the model uses)."""
    M, N = 3000, 2304
    dy = rnd((M, N), 14)
    db0 = rnd(N, 15)
    db = f32(db0)
    ws = None if atomic else torch.empty(gs.bias_grad_workspace(M, N), dtype=torch.uint8, device="cuda")
    gs.bias_grad(bf16(dy), db, ws)
    assert rel_l2(host(db), db0.astype(np.float32) + rounded(dy).sum(0)) < 1e-6


# --- a2/a6/a9: LayerNorm -------------------------------------------------------------------

@pytest.mark.parametrize("C,atomic", [(128, False), (256, False), (384, False), (512, False), (768, False),
                                      (1024, False), (1536, False), (2048, False), (128, True), (512, True),
                                      (768, True), (1024, True), (1536, True), (2048, True)])
def test_layernorm_fwd_bwd(C, atomic):
    """LayerNorm forward and backward; the backward's column sums both ways: a
    fixed-order second pass over a workspace, or fp32 atomics in one launch."""
    rows = 1000
    x = rnd((rows, C), 16, 2.0) + 0.5
    w, b = 1.0 + rnd(C, 17, 0.1), rnd(C, 18, 0.1)
    y = torch.empty(rows, C, dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(rows, device="cuda")
    rstd = torch.empty(rows, device="cuda")
    xd = bf16(x)
    gs.layernorm_fwd(xd, f32(w), f32(b), y, mean, rstd)
    xr = rounded(x)
    w32, b32 = w.astype(np.float32).astype(np.float64), b.astype(np.float32).astype(np.float64)
    yr, mr, rr = G.layernorm_fwd(xr, w32, b32)
    assert rel_l2(host(y), yr) < BF16_TOL
    assert rel_l2(host(mean), mr) < 1e-6 and rel_l2(host(rstd), rr) < 1e-5
    dy, dres = rnd((rows, C), 19), rnd((rows, C), 20)
    dx = torch.empty_like(y)
    dw0, db0 = rnd(C, 21), rnd(C, 22)
    dw, db = f32(dw0), f32(db0)
    ws = None if atomic else torch.empty(gs.layernorm_bwd_workspace(rows, C), dtype=torch.uint8, device="cuda")
    gs.layernorm_bwd(bf16(dy), xd, mean, rstd, f32(w), bf16(dres), dx, dw, db, ws)
    rdx, rdw, rdb = G.layernorm_bwd(rounded(dy), xr, mr, rr, w32)
    assert rel_l2(host(dx), rdx + rounded(dres)) < BF16_TOL
    assert rel_l2(host(dw), dw0.astype(np.float32) + rdw) < 1e-5
    assert rel_l2(host(db), db0.astype(np.float32) + rdb) < 1e-5


@pytest.mark.parametrize("rows,C", [(1, 768), (999, 768), (4737, 768), (999, 128), (333, 1024)])
def test_layernorm_fwd_row_counts(rows, C):
    """The forward takes rows in pairs for C <= 768, so an odd count leaves the
    last pair with one row: a single row, 999 rows, and 4,737 rows (one more
    than a whole pass of the resident grid on 148 SMs). Wider rows go one at a
    time. Every output row and statistic is compared; rows past the end are
    never written."""
    x = rnd((rows, C), 30, 1.5) - 0.25
    w, b = 1.0 + rnd(C, 31, 0.1), rnd(C, 32, 0.1)
    y = torch.full((rows + 2, C), 7.0, dtype=torch.bfloat16, device="cuda")
    mean = torch.full((rows + 2,), 7.0, device="cuda")
    rstd = torch.full((rows + 2,), 7.0, device="cuda")
    gs.layernorm_fwd(bf16(x), f32(w), f32(b), y[:rows], mean[:rows], rstd[:rows])
    w32, b32 = w.astype(np.float32).astype(np.float64), b.astype(np.float32).astype(np.float64)
    yr, mr, rr = G.layernorm_fwd(rounded(x), w32, b32)
    got = host(y)
    assert rel_l2(got[:rows], yr) < BF16_TOL
    assert rel_l2(host(mean)[:rows], mr) < 1e-6 and rel_l2(host(rstd)[:rows], rr) < 1e-5
    assert np.all(got[rows:] == 7.0) and np.all(host(mean)[rows:] == 7.0) and np.all(host(rstd)[rows:] == 7.0)


# --- a4: causal attention ------------------------------------------------------------------

@pytest.mark.parametrize("B,T,H,hd", [(2, 64, 2, 32), (2, 192, 3, 64), (1, 1024, 2, 64), (2, 256, 4, 32),
                                      (2, 256, 2, 64), (1, 512, 3, 64), (3, 128, 1, 64)])
def test_attention_fwd_bwd(B, T, H, hd):
    C = H * hd
    qkv = rnd((B, T, 3 * C), 23)
    out = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, T, device="cuda")
    qd = bf16(qkv)
    err = err_word()
    gs.attention_fwd(qd, out, lse, H, err)
    qr = rounded(qkv)
    q, k, v = (qr[..., i * C:(i + 1) * C].reshape(B, T, H, hd).transpose(0, 2, 1, 3) for i in range(3))
    o, l = G.attention_fwd(q, k, v)
    assert rel_l2(host(out), o.transpose(0, 2, 1, 3).reshape(B, T, C)) < 1e-2
    assert np.max(np.abs(host(lse) - l)) < 2e-3
    do = rnd((B, T, C), 24)
    dqkv = torch.empty_like(qd)
    ws = torch.empty(gs.attention_bwd_workspace(B, T, H, hd), dtype=torch.uint8, device="cuda")
    db0 = rnd(3 * C, 27).astype(np.float32)
    dbias = f32(db0)
    gs.attention_bwd(qd, out, bf16(do), lse, dqkv, H, ws, err, dbias=dbias)
    dor = rounded(do).reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    dq, dk, dv = G.attention_bwd(dor, q, k, v)
    got = host(dqkv)
    for i, ref in enumerate((dq, dk, dv)):
        assert rel_l2(got[..., i * C:(i + 1) * C], ref.transpose(0, 2, 1, 3).reshape(B, T, C)) < 2e-2, "qkv"[i]
    # the qkv bias gradient: column sums of dq | dk | dv over the B*T rows
    sq, sk, sv = (r.transpose(0, 2, 1, 3).reshape(B * T, C).sum(0) for r in (dq, dk, dv))
    assert np.max(np.abs(sk)) < 1e-9 * np.max(np.abs(sq))      # the oracle: the key bias has no gradient
    gb = host(dbias).astype(np.float64) - db0
    tc = T % 128 == 0
    assert rel_l2(gb[:C], sq) < 2e-2
    if tc:
        assert np.all(host(dbias)[C:2 * C] == db0[C:2 * C])      # nothing added to the key third
        assert rel_l2(gb[2 * C:], sv) < 1e-5                     # dV's column sums are dO's
    else:                                                        # column sums of the stored bf16 dqkv
        assert np.max(np.abs(gb[C:2 * C])) < 2e-2 * np.max(np.abs(sq))
        assert rel_l2(gb[2 * C:], sv) < 2e-2
    assert int(err.sum()) == 0


# --- a11: vocabulary-masked softmax cross-entropy ------------------------------------------

@pytest.mark.parametrize("N,V,Vp", [(64, 1000, 1024), (37, 4353, 4480), (16, 50257, 50304), (8, 129, 256)])
def test_softmax_ce(N, V, Vp):
    z = rnd((N, Vp), 25, 2.0)
    z[:, V:] = 50.0  # padded columns must be ignored however large
    t = np.random.default_rng(26).integers(0, V, N)
    zd = bf16(z)
    losses = torch.empty(N, device="cuda")
    err = err_word()
    gs.softmax_ce(zd, i32(t), losses, V, 1.0 / N, err)
    lr, dzr = G.softmax_ce(rounded(z), t, V)
    assert np.max(np.abs(host(losses) - lr)) < 1e-4
    dz = host(zd)
    assert np.all(dz[:, V:] == 0.0)
    assert rel_l2(dz[:, :V], dzr[:, :V]) < BF16_TOL
    assert int(err.sum()) == 0
    t2 = t.copy()
    t2[3] = V  # out of range
    gs.softmax_ce(bf16(z), i32(t2), losses, V, 1.0 / N, err)
    assert int(err[0]) & 1


@pytest.mark.parametrize("N,C,V,Vp,pair", [(700, 256, 50257, 50304, True), (512, 768, 50257, 50304, True),
                                            (1024, 384, 4353, 4480, True), (300, 256, 1000, 1024, False),
                                            (128, 128, 4353, 4480, False)])
def test_lm_head_ce(N, C, V, Vp, pair):
    """Tied lm_head GEMM + softmax-CE. The first three shapes run the GEMM on CTA
    pairs, whose epilogue leaves per-row (max, sum) partials so that the CE reads
    the logits once (700 rows: a ragged last row tile); the last two take the
    single-CTA GEMM and the two-pass CE. Losses agree with the oracle's CE of the stored bf16 logits
    to fp32 rounding, padded columns (given large logits here) are left out, and
    the gradient matches the oracle's."""
    h, w = rnd((N, C), 29), rnd((Vp, C), 30, 0.05)
    w[V:] = rnd((Vp - V, C), 31, 0.5)   # padded ids: large logits that must not count
    t = np.random.default_rng(32).integers(0, V, N)
    hd, wd, td = bf16(h), bf16(w), i32(t)
    ws_bytes = gs.lm_head_ce_workspace(N, Vp)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    logits = torch.empty(N, Vp, dtype=torch.bfloat16, device="cuda")
    losses = torch.empty(N, device="cuda")
    err = err_word()
    gs.lm_head_ce(hd, wd, td, logits, losses, V, 1.0 / N, False, ws, err)
    z = host(logits)
    assert rel_l2(z, rounded(h) @ rounded(w).T) < BF16_TOL
    lr, dzr = G.softmax_ce(z, t, V)
    l0 = host(losses)
    assert np.max(np.abs(l0 - lr)) < 1e-4
    # the logits-free evaluation form: the same partials and target logit, no logits stored
    lf = torch.empty(N, device="cuda")
    if pair:
        gs.lm_head_loss(hd, wd, td, lf, V, ws, err)
        assert np.array_equal(host(lf), l0)
    else:
        with pytest.raises(gs.GPT2Error):
            gs.lm_head_loss(hd, wd, td, lf, V, ws, err)
    gs.lm_head_ce(hd, wd, td, logits, losses, V, 1.0 / N, True, ws, err)
    assert np.array_equal(host(losses), l0)
    dz = host(logits)
    assert np.all(dz[:, V:] == 0.0)
    assert rel_l2(dz[:, :V], dzr[:, :V]) < BF16_TOL
    assert int(err.sum()) == 0
    with pytest.raises(gs.GPT2Error):
        gs.lm_head_ce(hd, wd, td, logits, losses, V, 1.0 / N, True, ws[: ws_bytes - 8], err)


@pytest.mark.parametrize("N,V,Vp,ignore", [(64, 1000, 1024, -100), (37, 4353, 4480, -1), (16, 50257, 50304, -1)])
def test_softmax_ce_masked(N, V, Vp, ignore):
    """Ignore index per target: ignored rows give loss 0 and an exactly zero
    gradient row and raise no error; kept rows match the oracle's mean over kept rows."""
    z = rnd((N, Vp), 27, 2.0)
    t = np.random.default_rng(28).integers(0, V, N)
    t[::3] = ignore
    zd = bf16(z)
    losses = torch.empty(N, device="cuda")
    err = err_word()
    n_keep = int((t != ignore).sum())
    gs.softmax_ce_masked(zd, i32(t), losses, V, ignore, 1.0 / n_keep, err)
    lr, dzr, n = G.softmax_ce_masked(rounded(z), t, V, ignore)
    assert n == n_keep
    assert np.max(np.abs(host(losses) - lr)) < 1e-4
    dz = host(zd)
    assert np.all(dz[t == ignore] == 0.0) and np.all(dz[:, V:] == 0.0)
    assert rel_l2(dz, dzr) < BF16_TOL
    assert int(err.sum()) == 0


# --- a1: embeddings -----------------------------------------------------------------------

def test_embedding_fwd_bwd():
    B, T, C, V, Vp = 3, 128, 384, 1000, 1024
    wte, wpe = rnd((Vp, C), 27, 0.02), rnd((T, C), 28, 0.02)
    tok = np.random.default_rng(29).integers(0, V, (B, T))
    tok[0, :10] = 7  # repeated ids exercise the accumulation
    out = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    err = err_word()
    gs.embedding_fwd(i32(tok), bf16(wte), bf16(wpe), out, V, err)
    ref = rounded(wte)[tok] + rounded(wpe)[None]
    assert rel_l2(host(out), ref) < BF16_TOL and int(err.sum()) == 0
    dx = rnd((B, T, C), 30)
    dwte, dwpe = torch.zeros(Vp, C, device="cuda"), torch.zeros(T, C, device="cuda")
    gs.embedding_bwd(i32(tok), bf16(dx), dwte, dwpe, V)
    rw = np.zeros((Vp, C))
    np.add.at(rw, tok.reshape(-1), rounded(dx).reshape(-1, C))
    assert rel_l2(host(dwte), rw) < 1e-6
    assert rel_l2(host(dwpe), rounded(dx).sum(0)) < 1e-6
    bad = tok.copy()
    bad[1, 5] = V + 3
    gs.embedding_fwd(i32(bad), bf16(wte), bf16(wpe), out, V, err)
    assert int(err[0]) & 1


# --- failure handling: the bounded device wait -----------------------------------------------

def test_bounded_wait_times_out_and_the_context_stays_usable():
    """A wait on a barrier that nothing completes gives up after its limit: the
    kernel records the timeout flag (4) in the device error word and returns,
    the call maps it to GPT2_ERR_TIMEOUT (6), and the GPU keeps working."""
    import time
    err = err_word()
    t0 = time.perf_counter()
    st = gs.wait_selftest(50_000_000, err)       # 50 ms
    dt = time.perf_counter() - t0
    assert st == 6, st
    assert int(err[0]) == 4
    assert 0.04 <= dt < 5.0, dt
    # the context is intact: an ordinary op still runs and is correct
    x, w = rnd((256, 128), 70), rnd((256, 128), 71, 0.05)
    out = torch.empty(256, 256, dtype=torch.bfloat16, device="cuda")
    err2 = err_word()
    gs.linear_fwd(bf16(x), bf16(w), None, None, out, err2)
    assert rel_l2(host(out), rounded(x) @ rounded(w).T) < BF16_TOL and int(err2.sum()) == 0
