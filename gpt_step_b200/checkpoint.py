"""Checkpoint / resume and the evaluation cadence of a training run.

"Pretraining and adapting a language model on a dependency-free stack":
§4.4 scores held-out batches every 250 steps; the supervision paragraph after
§5.1 writes a checkpoint every 500 steps WITH the optimizer state, so that a
restarted run continues where it stopped instead of repeating steps.

A checkpoint is one ``.npz`` file holding, for every named tensor of the model,
the fp32 master weight and both AdamW moments, plus a JSON header with the
step counter (the number of optimizer steps already taken, which is also the
index of the next step, its learning rate and its bias correction) and the data
cursor of the token source. Nothing else is state: gradients are zero between
steps, and the bf16 weight copy the kernels read is re-derived from the fp32
masters by ``gpt2_write`` when they are loaded. The file is written to a
temporary name and renamed, so a crash during a save leaves the previous
checkpoint intact.

Host logic only: the arrays move through the model's ``read``/``write``
(the C ABI's ``gpt2_read``/``gpt2_write``), so the format and the cadence are
exercised on the CPU with any object that offers ``cfg``, ``tensors()``,
``read`` and ``write``.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass

import numpy as np

PARAMS, ADAM_M, ADAM_V = 0, 2, 3          # the C ABI's state selectors
_KINDS = (("param", PARAMS), ("m", ADAM_M), ("v", ADAM_V))
FORMAT = "gpt2-step-checkpoint/1"


def _config_dict(cfg) -> dict:
    """The model configuration as plain numbers (a ctypes struct or a mapping)."""
    if isinstance(cfg, dict):
        return dict(cfg)
    return {name: getattr(cfg, name) for name, _ in cfg._fields_}


def save(model, path: str, step: int, data_cursor: int | None = None) -> str:
    """Write the model's fp32 weights, AdamW moments, ``step`` and ``data_cursor`` to ``path``."""
    if step < 0:
        raise ValueError("step must be >= 0")
    arrays = {}
    names = []
    for i, t in enumerate(model.tensors()):
        names.append(t.name)
        for key, what in _KINDS:
            a = np.asarray(model.read(what, i), dtype=np.float32)
            if a.shape != tuple(t.shape):
                raise ValueError(f"{t.name}: read shape {a.shape} != {tuple(t.shape)}")
            arrays[f"{key}/{t.name}"] = a
    header = {"format": FORMAT, "step": int(step),
              "data_cursor": None if data_cursor is None else int(data_cursor),
              "config": _config_dict(model.cfg), "tensors": names}
    arrays["header"] = np.frombuffer(json.dumps(header).encode(), dtype=np.uint8)
    tmp = f"{path}.tmp-{os.getpid()}"
    try:
        with open(tmp, "wb") as f:
            np.savez(f, **arrays)
            f.flush()
            os.fsync(f.fileno())
        os.replace(tmp, path)
    except BaseException:
        # a failed save leaves any earlier checkpoint at `path` as it was
        if os.path.exists(tmp):
            os.remove(tmp)
        raise
    return path


def read_header(path: str) -> dict:
    with np.load(path) as z:
        return json.loads(bytes(z["header"]).decode())


def load(model, path: str) -> dict:
    """Restore weights and moments into ``model``; returns the header (``step``, ``data_cursor``).

    Refuses a checkpoint whose format, configuration or tensor list differs from
    the model's (a resumed run must be the same run), before writing anything.
    """
    with np.load(path) as z:
        header = json.loads(bytes(z["header"]).decode())
        if header.get("format") != FORMAT:
            raise ValueError(f"{path}: not a {FORMAT} file")
        want = _config_dict(model.cfg)
        got = header["config"]
        diff = sorted(k for k in want if k not in got or not np.isclose(got[k], want[k], rtol=0, atol=0))
        if diff:
            raise ValueError(f"{path}: configuration differs in {diff}")
        infos = model.tensors()
        if header["tensors"] != [t.name for t in infos]:
            raise ValueError(f"{path}: tensor list differs from the model's")
        staged = []
        for i, t in enumerate(infos):
            for key, what in _KINDS:
                a = z[f"{key}/{t.name}"]
                if a.shape != tuple(t.shape) or a.dtype != np.float32:
                    raise ValueError(f"{path}: {key}/{t.name} has {a.dtype}{a.shape}")
                staged.append((what, i, a))
    for what, i, a in staged:
        model.write(what, i, a)
    return header


@dataclass
class Cadence:
    """When to score held-out batches and when to checkpoint, counted in completed steps."""
    eval_every: int = 250
    ckpt_every: int = 500

    def eval_due(self, done: int) -> bool:
        return self.eval_every > 0 and done > 0 and done % self.eval_every == 0

    def ckpt_due(self, done: int) -> bool:
        return self.ckpt_every > 0 and done > 0 and done % self.ckpt_every == 0


def latest(directory: str, prefix: str = "step_") -> str | None:
    """The checkpoint in ``directory`` with the highest step, or None."""
    best, best_step = None, -1
    if not os.path.isdir(directory):
        return None
    for name in os.listdir(directory):
        if name.startswith(prefix) and name.endswith(".npz"):
            try:
                s = int(name[len(prefix):-4])
            except ValueError:
                continue
            if s > best_step:
                best, best_step = os.path.join(directory, name), s
    return best


def ckpt_path(directory: str, step: int, prefix: str = "step_") -> str:
    return os.path.join(directory, f"{prefix}{step:07d}.npz")


def run(model, source, first_step: int, last_step: int, put, cadence: Cadence,
        ckpt_dir: str | None = None, evaluate=None, log=None, par=None) -> list:
    """Optimizer steps ``first_step .. last_step-1`` with the eval and checkpoint cadence.

    ``source.get()`` yields host (tokens, targets) micro-batches and carries the
    data cursor in ``source.next``; ``put`` moves one host array to the device;
    ``evaluate(model) -> float`` scores the held-out batches. Each step runs
    ``grad_accum`` micro-steps, then the clip + AdamW step. Returns the log
    records (one per step: step, the mean loss over its micro-steps, the
    pre-clip gradient norm, and the eval loss where one was due).

    With ``par`` (a ``dp.DataParallel``) the run is one rank of a data-parallel
    job: gradients are averaged across ranks before each update (in the
    sharded form each rank updates its shards and the weights are gathered),
    the logged and held-out losses are averaged across ranks, and rank 0 alone
    writes the checkpoints, after the sharded state has been gathered. Every rank's data cursor advances alike (same micro-batch
    count per step), so rank 0's cursor is every rank's.
    """
    records = []
    accum = model.cfg.grad_accum
    mean = (lambda v: par.mean_over_ranks(v)) if par is not None else (lambda v: v)
    writer = par is None or par.rank == 0
    for step in range(first_step, last_step):
        for _ in range(accum):
            x, y = source.get()
            model.fwd_bwd(put(x), put(y))
        if par is not None:
            par.update(step)          # the exchange across ranks and the (sharded) update
        else:
            model.clip_adamw(step)
        loss, norm = model.last_step_stats()
        rec = {"step": step, "loss": mean(loss), "grad_norm": norm}
        done = step + 1
        if evaluate is not None and cadence.eval_due(done):
            rec["eval_loss"] = mean(evaluate(model))
        if ckpt_dir is not None and cadence.ckpt_due(done) and par is not None:
            par.gather_state()        # collective: sharded masters and moments made whole on every rank
        if ckpt_dir is not None and cadence.ckpt_due(done) and writer:
            os.makedirs(ckpt_dir, exist_ok=True)
            rec["checkpoint"] = save(model, ckpt_path(ckpt_dir, done), done, getattr(source, "next", None))
        records.append(rec)
        if log is not None:
            log(rec)
    return records
