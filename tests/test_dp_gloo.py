"""Data parallelism, host logic on the CPU: two gloo ranks.

A fake model (fp64 torch state, a gradient that is linear in the batch, a
clipped SGD update scaled by the micro-steps since the last update) stands in
for the device model behind the same interface. Two ranks that each take half
of the micro-batches and average their gradients must end where one process
that took all of them ends, with bit-identical weights on both ranks; the
held-out loss is the mean of the ranks' losses.
"""
import math
import multiprocessing as mp
import socket

import numpy as np
import pytest
import torch

from gpt_step_b200 import dp

# flat layout of the fake: region 0 (the "1-D parameters") then three buckets
REGION0 = (0, 64)
BUCKETS = [(64, 320), (320, 448), (448, 832)]
N = 832
LR0, B1, B2, EPS, WD = 0.1, 0.9, 0.95, 1e-8, 0.1


def _feat(x, y):
    x = np.asarray(x, np.float64).ravel()
    y = np.asarray(y, np.float64).ravel()
    f = np.zeros(N)
    np.add.at(f, np.arange(x.size) % N, np.sin(x) + 0.5 * np.cos(y))
    return torch.tensor(f / x.size, dtype=torch.float64)


class FakeModel:
    """fp64 stand-in with the device model's state interface: fp32-master-like
    parameters p, the copy w the forward reads outside region 0 (the bf16 copy on
    the device), gradients accumulated over micro-steps, AdamW moments, the
    bucket layout, and the range-restricted update with an external norm."""

    def __init__(self, seed=0, dtype=torch.float64):
        g = torch.Generator().manual_seed(seed)
        self.dtype = dtype
        self.p = torch.randn(N, generator=g, dtype=torch.float64).to(dtype)
        self.w = self.p.clone()
        self.g = torch.zeros(N, dtype=dtype)
        self.m = torch.zeros(N, dtype=dtype)
        self.v = torch.zeros(N, dtype=dtype)
        self.k = 0
        self.losses = []
        self.stats = (0.0, 0.0)

    def weights(self):
        """What the forward computes with: region 0 from p, the buckets from the copy."""
        e = self.w.clone()
        e[REGION0[0]:REGION0[1]] = self.p[REGION0[0]:REGION0[1]]
        return e

    def state_tensor(self, what):
        return {dp.PARAMS: self.p, dp.GRADS: self.g, dp.ADAM_M: self.m, dp.ADAM_V: self.v,
                dp.WEIGHTS_BF16: self.w}[what]

    def num_buckets(self):
        return len(BUCKETS)

    def bucket_range(self, b):
        return REGION0 if b == -1 else BUCKETS[b]

    def fwd_bwd(self, x, y):
        f = _feat(x, y).to(self.dtype)
        self.g += 0.3 * self.weights() - f
        self.losses.append(float(f @ self.weights()))
        self.k += 1

    def grad_sumsq(self, ranges, out):
        out[0] = sum(float((self.g[a:b] ** 2).sum()) for a, b in ranges)

    def clip_adamw_ranges(self, step, ranges, sumsq):
        norm = math.sqrt(float(sumsq[0])) / self.k
        scale = min(1.0, 1.0 / norm) / self.k
        lr, t = LR0 / (step + 1), step + 1
        for a, b in ranges:
            gg = self.g[a:b] * scale
            self.m[a:b] = B1 * self.m[a:b] + (1 - B1) * gg
            self.v[a:b] = B2 * self.v[a:b] + (1 - B2) * gg * gg
            upd = (self.m[a:b] / (1 - B1 ** t)) / (torch.sqrt(self.v[a:b] / (1 - B2 ** t)) + EPS)
            lam = torch.where(torch.arange(a, b) >= REGION0[1], WD, 0.0).to(self.dtype)
            self.p[a:b] = self.p[a:b] - lr * (upd + lam * self.p[a:b])
            self.w[a:b] = self.p[a:b]
        self.stats = (float(np.mean(self.losses)), norm)
        self.g.zero_()
        self.k = 0
        self.losses = []

    def clip_adamw(self, step):
        s = torch.zeros(1, dtype=torch.float64)
        self.grad_sumsq([(0, N)], s)
        self.clip_adamw_ranges(step, [(0, N)], s)

    def last_step_stats(self):
        return self.stats

    def eval_loss(self, x, y):
        return float(_feat(x, y).to(self.dtype) @ self.weights())


def _batches(step, a, rank, world):
    """Micro-batch a of optimizer step `step` on `rank` (global index interleaved by rank)."""
    rng = np.random.default_rng(1000 * step + world * a + rank)
    return rng.integers(0, 50, (2, 8)), rng.integers(0, 50, (2, 8))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q, A, steps, mode):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        m = FakeModel()
        d = dp.DataParallel(m, mode=mode)
        norms = []
        for s in range(steps):
            xs, ys = zip(*[_batches(s, a, rank, world) for a in range(A)])
            if s == 0:
                d.step(xs, ys, s)
            else:   # the host-buffer path, with CPU tensors standing in for pinned / device buffers
                hx, hy = torch.tensor(np.stack(xs)), torch.tensor(np.stack(ys))
                _, n = d.step_host(hx, hy, torch.empty_like(hx), torch.empty_like(hy), s)
            norms.append(m.last_step_stats()[1])
        ex, ey = _batches(99, 0, rank, world)
        ev_local = m.eval_loss(ex, ey)
        ev = d.eval_loss(ex, ey)
        agree = d.replicas_agree()
        used = m.weights().tolist()
        d.gather_state()                  # the sharded masters made whole: every p equals the used weights
        whole = m.p.tolist()
        if rank == 1:
            m.p[3] += 1e-9                # region 0: read by the forward in both forms
        disagree = not d.replicas_agree()
        q.put((rank, used, norms, ev_local, ev, agree, disagree, whole))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["zero1", "allreduce"])
def test_two_ranks_average_gradients_like_one_process(mode):
    """Two ranks with half the micro-batches each end where one process with all
    of them ends: in the sharded form (reduce-scatter per bucket, norm from the
    summed shard partials, update of the own shards, gather of the copies) and
    in the all-reduce form."""
    A, steps, world = 3, 3, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, A, steps, mode)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    # one process taking every rank's micro-batches (A x world micro-steps per step)
    ref = FakeModel()
    ref_norms = []
    for s in range(steps):
        for a in range(A):
            for r in range(world):
                ref.fwd_bwd(*_batches(s, a, r, world))
        ref.clip_adamw(s)
        ref_norms.append(ref.last_step_stats()[1])

    p0, p1 = np.array(out[0][1]), np.array(out[1][1])
    assert np.array_equal(p0, p1)                      # every rank computes with the same weights
    assert np.allclose(p0, ref.p.numpy(), rtol=0, atol=1e-13)
    assert np.array_equal(np.array(out[0][7]), p0) and np.array_equal(np.array(out[1][7]), p1)
    assert np.allclose(out[0][2], ref_norms, rtol=1e-12)
    assert out[0][2] == out[1][2]                      # the same norm on every rank
    # held-out loss: the mean of the ranks' own losses
    assert out[0][4] == out[1][4]
    assert abs(out[0][4] - 0.5 * (out[0][3] + out[1][3])) < 1e-14
    assert out[0][5] and out[1][5]                     # identical weights detected
    assert out[0][6] and out[1][6]                     # a 1e-9 difference on one rank detected


def test_single_process_is_the_plain_step():
    m, ref = FakeModel(), FakeModel()
    d = dp.DataParallel(m)
    assert d.world == 1
    xs, ys = zip(*[_batches(0, a, 0, 1) for a in range(2)])
    d.step(xs, ys, 0)
    for x, y in zip(xs, ys):
        ref.fwd_bwd(x, y)
    ref.clip_adamw(0)
    assert torch.equal(m.p, ref.p)
    assert d.mean_over_ranks(2.5) == 2.5 and d.replicas_agree()


# --- data parallel with the checkpoint / eval cadence ----------------------------------------

class CkptFake(FakeModel):
    """FakeModel with the state interface a checkpoint needs (one flat tensor)."""

    class Cfg(dict):
        grad_accum = 2

    def __init__(self, seed=0):
        super().__init__(seed, dtype=torch.float32)     # fp32 state, as the checkpoint stores it
        self.cfg = CkptFake.Cfg(n_embd=N, grad_accum=2)

    def tensors(self):
        from types import SimpleNamespace
        return [SimpleNamespace(name="w", shape=(N,))]

    def read(self, what, i):
        return self.state_tensor(what).numpy().copy()

    def write(self, what, i, a):
        self.state_tensor(what)[:] = torch.tensor(a, dtype=self.dtype)
        if what == dp.PARAMS:          # as gpt2_write: the copy follows the masters
            self.w[:] = self.p


class RankSource:
    def __init__(self, rank):
        self.rank, self.next = rank, 0

    def get(self):
        rng = np.random.default_rng(7919 * self.rank + self.next)
        self.next += 1
        return rng.integers(0, 50, (2, 8)), rng.integers(0, 50, (2, 8))


def _ckpt_rank_main(rank, world, port, q, root):
    import os

    import torch.distributed as dist

    from gpt_step_b200 import checkpoint as ck
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cad = ck.Cadence(eval_every=2, ckpt_every=2)
        ex, ey = _batches(5, 0, rank, world)
        ev = lambda m: m.eval_loss(ex, ey)
        ident = lambda a: a
        a = CkptFake()
        ra = ck.run(a, RankSource(rank), 0, 4, ident, cad, os.path.join(root, "a"), ev, par=dp.DataParallel(a))
        b = CkptFake()
        ck.run(b, RankSource(rank), 0, 2, ident, cad, os.path.join(root, "b"), ev, par=dp.DataParallel(b))
        dist.barrier()                           # rank 0 has written step 2
        c = CkptFake(seed=5)
        h = ck.load(c, ck.latest(os.path.join(root, "b")))
        s = RankSource(rank)
        s.next = h["data_cursor"]
        rc = ck.run(c, s, h["step"], 4, ident, cad, None, ev, par=dp.DataParallel(c))
        strip = lambda recs: [{k: v for k, v in r.items() if k != "checkpoint"} for r in recs]
        q.put((rank, a.weights().tolist(), c.weights().tolist(), strip(ra), strip(ra[:2]) + strip(rc),
               sorted(os.listdir(os.path.join(root, "b")))))
    finally:
        dist.destroy_process_group()


def test_data_parallel_run_checkpoints_on_rank_0_and_resumes(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ckpt_rank_main, args=(r, world, port, q, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, pa, pc, ra, rresumed, files in out:
        assert pa == pc                          # stop, restore, continue = straight run, bitwise
        assert ra == rresumed                    # same logged (rank-averaged) losses and evals
        assert files == ["step_0000002.npz"]     # rank 0 alone wrote, once
    assert out[0][1] == out[1][1]                # ranks hold the same weights
    assert out[0][3] == out[1][3]                # and log the same averaged values
    assert [r["step"] for r in out[0][3] if "eval_loss" in r] == [1, 3]
