"""Checkpoint / resume and the eval cadence, host logic on the CPU.

A fake model (numpy state, a toy deterministic update) stands in for the
device model behind the same read/write interface, so these tests pin the file
format, the refusal rules, the cadence and the resume arithmetic exactly; the
device round trip is in test_gpu_model.py.
"""
import os
from dataclasses import dataclass

import numpy as np
import pytest

from gpt_step_b200 import checkpoint as ck


@dataclass
class Info:
    name: str
    shape: tuple


class FakeCfg(dict):
    @property
    def grad_accum(self):
        return self["grad_accum"]


class FakeModel:
    """fp32 params + two moments; fwd_bwd accumulates a gradient from the batch,
    clip_adamw applies a step-dependent update and zeroes it."""

    def __init__(self, seed, accum=2):
        rng = np.random.default_rng(seed)
        self.cfg = FakeCfg(n_layer=1, n_embd=4, grad_accum=accum, max_lr=6e-4)
        self.infos = [Info("wte", (5, 4)), Info("ln_f.b", (4,))]
        self.state = {w: [rng.standard_normal(i.shape).astype(np.float32) for i in self.infos]
                      for w in (ck.PARAMS, ck.ADAM_M, ck.ADAM_V)}
        self.grad = [np.zeros(i.shape, np.float32) for i in self.infos]
        self.stats = (0.0, 0.0)
        self.losses = []

    def tensors(self):
        return self.infos

    def read(self, what, i):
        return self.state[what][i].copy()

    def write(self, what, i, a):
        self.state[what][i] = np.array(a, np.float32)

    def fwd_bwd(self, x, y):
        s = np.float32(np.sum(x) * 1e-3 - np.sum(y) * 2e-3)
        for g, p in zip(self.grad, self.state[ck.PARAMS]):
            g += np.float32(0.5) * p + s
        self.losses.append(float(s))

    def clip_adamw(self, step):
        lr = np.float32(1e-2 / (step + 1))
        for i, g in enumerate(self.grad):
            m, v, p = (self.state[w][i] for w in (ck.ADAM_M, ck.ADAM_V, ck.PARAMS))
            m[...] = np.float32(0.9) * m + np.float32(0.1) * g
            v[...] = np.float32(0.95) * v + np.float32(0.05) * g * g
            p -= lr * m / (np.sqrt(np.abs(v)) + np.float32(1e-8))
            g[...] = 0
        self.stats = (float(np.mean(self.losses[-self.cfg.grad_accum:])), float(lr))

    def last_step_stats(self):
        return self.stats


class FakeSource:
    def __init__(self, seed):
        self.seed, self.next = seed, 0

    def get(self):
        rng = np.random.default_rng(self.seed + self.next)
        self.next += 1
        return rng.integers(0, 100, (2, 3)), rng.integers(0, 100, (2, 3))


def snapshot(m):
    return {w: [a.copy() for a in m.state[w]] for w in m.state}


def test_round_trip_is_bitwise(tmp_path):
    a, b = FakeModel(1), FakeModel(2)
    p = ck.save(a, str(tmp_path / "c.npz"), 17, data_cursor=34)
    h = ck.load(b, p)
    assert h["step"] == 17 and h["data_cursor"] == 34
    for w in a.state:
        for x, y in zip(a.state[w], b.state[w]):
            assert x.dtype == y.dtype == np.float32
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    assert [f for f in os.listdir(tmp_path)] == ["c.npz"]  # no temporary left behind


def test_refuses_other_config_and_writes_nothing(tmp_path):
    a, b = FakeModel(1), FakeModel(2)
    p = ck.save(a, str(tmp_path / "c.npz"), 3)
    b.cfg["n_embd"] = 8
    before = snapshot(b)
    with pytest.raises(ValueError, match="n_embd"):
        ck.load(b, p)
    after = snapshot(b)
    assert all(np.array_equal(x, y) for w in before for x, y in zip(before[w], after[w]))


def test_refuses_other_tensor_list(tmp_path):
    a, b = FakeModel(1), FakeModel(2)
    p = ck.save(a, str(tmp_path / "c.npz"), 3)
    b.infos = [Info("wte", (5, 4)), Info("ln_f.w", (4,))]
    with pytest.raises(ValueError, match="tensor list"):
        ck.load(b, p)


def test_cadence_matches_the_pages():
    # held-out scoring every 250 steps, checkpoints every 500 (with optimizer state)
    c = ck.Cadence()
    evals = [d for d in range(1, 1501) if c.eval_due(d)]
    ckpts = [d for d in range(1, 1501) if c.ckpt_due(d)]
    assert evals == [250, 500, 750, 1000, 1250, 1500]
    assert ckpts == [500, 1000, 1500]
    assert not c.eval_due(0) and not ck.Cadence(0, 0).ckpt_due(500)


def test_latest_picks_highest_step(tmp_path):
    assert ck.latest(str(tmp_path / "none")) is None
    m = FakeModel(1)
    for s in (500, 1500, 1000):
        ck.save(m, ck.ckpt_path(str(tmp_path), s), s)
    (tmp_path / "step_x.npz").write_bytes(b"")
    assert ck.latest(str(tmp_path)).endswith("step_0001500.npz")
    assert ck.read_header(ck.latest(str(tmp_path)))["step"] == 1500


def test_resume_continues_instead_of_repeating(tmp_path):
    """Steps 0..5 straight equal steps 0..2, a checkpoint, a fresh model and source
    restored from it, then steps 3..5: bitwise, with the same losses and evals."""
    cad = ck.Cadence(eval_every=2, ckpt_every=3)
    ev = lambda m: float(np.sum(m.state[ck.PARAMS][0]))
    ident = lambda x: x

    a, sa = FakeModel(7), FakeSource(11)
    ra = ck.run(a, sa, 0, 6, ident, cad, str(tmp_path / "a"), ev)

    b, sb = FakeModel(7), FakeSource(11)
    rb1 = ck.run(b, sb, 0, 3, ident, cad, str(tmp_path / "b"), ev)
    path = ck.latest(str(tmp_path / "b"))
    assert path.endswith("step_0000003.npz")
    c, sc = FakeModel(99), FakeSource(11)
    h = ck.load(c, path)
    sc.next = h["data_cursor"]
    rc = ck.run(c, sc, h["step"], 6, ident, cad, str(tmp_path / "c"), ev)

    strip = lambda r: {k: v for k, v in r.items() if k != "checkpoint"}
    assert [strip(r) for r in ra] == [strip(r) for r in rb1 + rc]
    assert [r["step"] for r in ra if "eval_loss" in r] == [1, 3, 5]
    assert [r["step"] for r in ra if "checkpoint" in r] == [2, 5]
    for w in a.state:
        for x, y in zip(a.state[w], c.state[w]):
            assert np.array_equal(x, y)


def test_failed_save_keeps_the_previous_checkpoint(tmp_path, monkeypatch):
    a = FakeModel(1)
    p = ck.save(a, str(tmp_path / "c.npz"), 5, data_cursor=10)
    b = FakeModel(2)

    def boom(*args, **kw):
        raise OSError("disk full")
    monkeypatch.setattr(ck.np, "savez", boom)
    with pytest.raises(OSError):
        ck.save(b, p, 6, data_cursor=12)
    monkeypatch.undo()
    assert os.listdir(tmp_path) == ["c.npz"]          # no temporary left behind
    c = FakeModel(3)
    h = ck.load(c, p)
    assert h["step"] == 5 and h["data_cursor"] == 10
    assert all(np.array_equal(x, y) for x, y in zip(a.state[ck.PARAMS], c.state[ck.PARAMS]))
