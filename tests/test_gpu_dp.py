"""Data parallelism in the sharded (ZeRO-1) form on one GPU: two model
instances stand in for two ranks.

"Pretraining and adapting a language model on a dependency-free stack" §4.4
averages the gradients of every card once per optimizer step. Here rank r's
model takes half of the micro-batches; the exchange the collectives would make
is done with plain tensor arithmetic on the models' flat state arrays (the
reduce-scatter average of each bucket into its owner's shard, the all-reduce
of region 0 and of the norm partials, the all-gather of the bf16 shards), and
the library's sharded update (gpt2_grad_sumsq, gpt2_clip_adamw_ranges) runs on
each model for its own ranges. The result must be the step of one model that
took every micro-batch, and the oracle's step over the union batch.
"""
import numpy as np
import pytest

import gpt_step_b200 as gs
from gpt_step_b200 import synth, workloads
from oracle import gpt2 as G

from gpu_util import i32, rel_l2, require_gpu, torch

pytestmark = pytest.mark.gpu

WORLD = 2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def shards(m, rank):
    out = []
    for b in range(m.num_buckets()):
        lo, hi = m.bucket_range(b)
        n = (hi - lo) // WORLD
        assert (hi - lo) % (64 * WORLD) == 0
        out.append((lo + rank * n, lo + (rank + 1) * n))
    return out


def emulated_sharded_step(models, step):
    """The collectives of the sharded step, done with tensor arithmetic on one GPU."""
    r0 = models[0].bucket_range(-1)
    own = [shards(m, r) for r, m in enumerate(models)]
    g = [m.state_tensor(gs.GPT2_GRADS) for m in models]
    # reduce-scatter (average) of every bucket into its owner's shard
    for r in range(WORLD):
        for lo, hi in own[r]:
            g[r][lo:hi] = sum(gg[lo:hi] for gg in g) / WORLD
    # all-reduce (average) of region 0
    avg0 = sum(gg[r0[0]:r0[1]] for gg in g) / WORLD
    for gg in g:
        gg[r0[0]:r0[1]] = avg0
    # the norm: shard partials (region 0 once), summed across ranks
    parts = [torch.zeros(1, dtype=torch.float64, device="cuda") for _ in models]
    for r, m in enumerate(models):
        m.grad_sumsq(own[r] + ([r0] if r == 0 else []), parts[r])
    total = parts[0] + parts[1]
    norms = [m.clip_adamw_ranges(step, [r0] + own[r], total, want_norm=True) for r, m in enumerate(models)]
    # all-gather of the bf16 weights
    w = [m.state_tensor(gs.GPT2_WEIGHTS_BF16) for m in models]
    for r in range(WORLD):
        for lo, hi in own[r]:
            for q in range(WORLD):
                if q != r:
                    w[q][lo:hi] = w[r][lo:hi]
    torch.cuda.synchronize()
    return norms, own, r0


def assembled_masters(models, own, r0):
    """The fp32 masters as the ranks own them: region 0 (every rank) and each shard from its owner."""
    p = models[0].state_tensor(gs.GPT2_PARAMS).clone()
    for r, m in enumerate(models):
        pr = m.state_tensor(gs.GPT2_PARAMS)
        for lo, hi in own[r]:
            p[lo:hi] = pr[lo:hi]
    return p


@pytest.mark.parametrize("name,over", [("tiny", dict(total_steps=10)),
                                       ("tiny", dict(total_steps=10, n_head=2, seq_len=256, micro_batch=2))])
def test_sharded_step_on_two_instances_matches_one_model_and_the_oracle(name, over):
    args = workloads.model_args(name, **over)
    cfg = gs.Config.make(**args)
    ranks = [gs.GPT2(cfg, 1337) for _ in range(WORLD)]
    whole = gs.GPT2(cfg, 1337)
    ocfg = G.Config(**args)
    B, T, V = args["micro_batch"], args["seq_len"], args["vocab_real"]
    batches = [synth.uniform_next_token_batch(B, T, V, 500 + i) for i in range(4)]
    p = G.init_params(ocfg, 1337)
    om, ov = G.zeros_like_params(ocfg), G.zeros_like_params(ocfg)
    names = [t.name for t in whole.tensors()]
    for step in range(2):
        for i, (x, y) in enumerate(batches):
            ranks[i % WORLD].fwd_bwd(i32(x), i32(y))     # rank r takes micro-batches r, r + 2
            whole.fwd_bwd(i32(x), i32(y))
        norms, own, r0 = emulated_sharded_step(ranks, step)
        wnorm = whole.clip_adamw(step, want_norm=True)
        oloss, onorm = G.train_step(ocfg, p, om, ov, step, batches)
        assert norms[0] == norms[1]                              # one global norm on every rank
        # against one model: the same sums in another order (atomics, bf16 roundings of
        # slightly different fp32 activation gradients)
        assert norms[0] == pytest.approx(wnorm, rel=2e-4)
        assert abs(norms[0] - onorm) <= 3e-2 * onorm
        # every rank computes with the same weights: region 0 in fp32 and the bf16 copy
        w0, w1 = (m.state_tensor(gs.GPT2_WEIGHTS_BF16) for m in ranks)
        assert torch.equal(w0, w1)
        a0, a1 = (m.state_tensor(gs.GPT2_PARAMS)[r0[0]:r0[1]] for m in ranks)
        assert torch.equal(a0, a1)
        # the owned masters are the one-model step's and the oracle's. Against the one
        # model they differ only by the summation order of the gradients, which can
        # flip the sign decision of a first Adam step for a gradient within its
        # rounding of zero (a 2 lr move on that element): 1e-3 leaves room for those,
        # while a shard left out of the update or averaged wrongly moves half of all
        # elements by about lr (a relative error near 3e-2).
        got = assembled_masters(ranks, own, r0)
        ref = whole.state_tensor(gs.GPT2_PARAMS)
        assert rel_l2(got.double().cpu().numpy(), ref.double().cpu().numpy()) < 1e-3
        assert rel_l2(w0.float().cpu().numpy(), whole.state_tensor(gs.GPT2_WEIGHTS_BF16).float().cpu().numpy()) < 1e-3
        named = {n: whole.read(gs.GPT2_PARAMS, i) for i, n in enumerate(names)}
        oref = G.split_named(ocfg, p)
        flat_got = np.concatenate([named[n].ravel() for n in names]).astype(np.float64)
        flat_ref = np.concatenate([np.asarray(oref[n]).ravel() for n in names])
        # bf16 activations against the fp64 definition: the first-step floor (1.3e-3, pinned on the CPU)
        assert rel_l2(flat_got, flat_ref) <= 2e-3, (step, rel_l2(flat_got, flat_ref))
    # the next forward on either rank (bf16 copy + region 0) is the one model's forward
    x, y = batches[0]
    l0 = ranks[0].eval_loss(i32(x), i32(y))
    l1 = ranks[1].eval_loss(i32(x), i32(y))
    lw = whole.eval_loss(i32(x), i32(y))
    assert l0 == l1 and l0 == pytest.approx(lw, abs=1e-3)
    for m in ranks + [whole]:
        m.close()
