"""Data parallelism, host logic on the CPU: two gloo ranks.

A fake model (fp64 torch state, a gradient that is linear in the batch, a
clipped SGD update scaled by the micro-steps since the last update) stands in
for the device model behind the same interface. Two ranks that each take half
of the micro-batches and average their gradients must end where one process
that took all of them ends, with bit-identical weights on both ranks; the
held-out loss is the mean of the ranks' losses.
"""
import multiprocessing as mp
import socket

import numpy as np
import torch

from gpt_step_b200 import dp

N = 37


def _feat(x, y):
    x = np.asarray(x, np.float64).ravel()
    y = np.asarray(y, np.float64).ravel()
    f = np.zeros(N)
    np.add.at(f, np.arange(x.size) % N, np.sin(x) + 0.5 * np.cos(y))
    return torch.tensor(f / x.size, dtype=torch.float64)


class FakeModel:
    def __init__(self, seed=0):
        g = torch.Generator().manual_seed(seed)
        self.p = torch.randn(N, generator=g, dtype=torch.float64)
        self.g = torch.zeros(N, dtype=torch.float64)
        self.k = 0
        self.losses = []
        self.stats = (0.0, 0.0)

    def state_tensor(self, what):
        return self.g if what == dp.GRADS else self.p

    def fwd_bwd(self, x, y):
        f = _feat(x, y)
        self.g += 0.3 * self.p - f
        self.losses.append(float(f.sum()))
        self.k += 1

    def clip_adamw(self, step):
        gm = self.g / self.k
        norm = float(torch.linalg.vector_norm(gm))
        if norm > 1.0:
            gm = gm / norm
        self.p -= 0.1 / (step + 1) * gm
        self.stats = (float(np.mean(self.losses)), norm)
        self.g.zero_()
        self.k = 0
        self.losses = []

    def last_step_stats(self):
        return self.stats

    def eval_loss(self, x, y):
        return float(_feat(x, y) @ self.p)


def _batches(step, a, rank, world):
    """Micro-batch a of optimizer step `step` on `rank` (global index interleaved by rank)."""
    rng = np.random.default_rng(1000 * step + world * a + rank)
    return rng.integers(0, 50, (2, 8)), rng.integers(0, 50, (2, 8))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q, A, steps):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        m = FakeModel()
        d = dp.DataParallel(m)
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
        if rank == 1:
            m.p[3] += 1e-9
        disagree = not d.replicas_agree()
        q.put((rank, m.p.tolist(), norms, ev_local, ev, agree, disagree))
    finally:
        dist.destroy_process_group()


def test_two_ranks_average_gradients_like_one_process():
    A, steps, world = 3, 3, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, A, steps)) for r in range(world)]
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
    assert np.array_equal(p0[:3], p1[:3]) and np.array_equal(p0[4:], p1[4:])
    assert np.allclose(p0, ref.p.numpy(), rtol=0, atol=1e-13)
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
    """FakeModel in fp32 with the state interface a checkpoint needs."""

    class Cfg(dict):
        grad_accum = 2

    def __init__(self, seed=0):
        super().__init__(seed)
        self.p = self.p.float()
        self.g = self.g.float()
        self.mom = {2: torch.zeros(N), 3: torch.zeros(N)}
        self.cfg = CkptFake.Cfg(n_embd=N, grad_accum=2)

    def fwd_bwd(self, x, y):
        f = _feat(x, y).float()
        self.g += 0.3 * self.p - f
        self.losses.append(float(f.sum()))
        self.k += 1

    def eval_loss(self, x, y):
        return float(_feat(x, y).float() @ self.p)

    def tensors(self):
        from types import SimpleNamespace
        return [SimpleNamespace(name="w", shape=(N,))]

    def read(self, what, i):
        return (self.p if what == dp.PARAMS else self.mom[what]).numpy().copy()

    def write(self, what, i, a):
        t = torch.tensor(a)
        if what == dp.PARAMS:
            self.p = t
        else:
            self.mom[what] = t


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
        q.put((rank, a.p.tolist(), c.p.tolist(), strip(ra), strip(ra[:2]) + strip(rc),
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
