"""Data parallelism: the multi-card arrangement of the training step.

"Pretraining and adapting a language model on a dependency-free stack" §4.4:
every card runs the same model on its own micro-batches (19 sequences x 9
accumulation steps per card, three cards); once per optimizer step the
gradients are averaged across the cards, so that each card's clip + AdamW sees
the gradient of the whole global batch and the copies stay identical; held-out
losses are averaged across cards in the same way.

The exchange is one all-reduce (average) of the flat fp32 gradient array
(``gpt2_state_device_ptr``: 124.5 M floats, 498 MB for the 124M model) between
the last micro-step's backward and the clip + AdamW, issued through
torch.distributed on the model's stream: NCCL between GPUs (NVLink / NVSwitch,
in-switch reduction where NCCL enables it), gloo for the CPU tests. At 725 GB/s
of measured all-reduce bus bandwidth that is about 1.2 ms against a ~180 ms
step. The norm and the AdamW update then run unchanged on every rank, on
identical averaged gradients, so no parameter traffic is needed.

Host logic only; the model is anything with ``state_tensor(GPT2_GRADS)``,
``fwd_bwd``, ``clip_adamw``, ``last_step_stats`` and ``eval_loss``.
"""
from __future__ import annotations

import contextlib

import torch
import torch.distributed as dist

GRADS, PARAMS = 1, 0   # the C ABI's state selectors


class DataParallel:
    def __init__(self, model, group=None):
        self.model = model
        self.group = group
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        self.backend = dist.get_backend(group) if on else None

    def _on_model_stream(self, t):
        s = getattr(self.model, "stream", None)
        if t.is_cuda and s is not None:
            return torch.cuda.stream(s)
        return contextlib.nullcontext()

    def _allreduce_mean(self, t):
        """In place: t <- mean over ranks of t."""
        if self.world == 1:
            return t
        with self._on_model_stream(t):
            if self.backend == "nccl":
                dist.all_reduce(t, op=dist.ReduceOp.AVG, group=self.group)
            else:  # gloo has no AVG
                dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
                t.mul_(1.0 / self.world)
        return t

    def sync_grads(self):
        """Average the accumulated gradients across ranks (no-op on one rank)."""
        if self.world > 1:
            self._allreduce_mean(self.model.state_tensor(GRADS))

    def step(self, tokens, targets, step: int):
        """One optimizer step: the rank's micro-batches, the gradient average, clip + AdamW."""
        for x, y in zip(tokens, targets):
            self.model.fwd_bwd(x, y)
        self.sync_grads()
        self.model.clip_adamw(step)

    def step_host(self, htok, htgt, dtok, dtgt, step: int):
        """The same from host (pinned) micro-batches [A, B, T]: copied into the device
        staging tensors dtok / dtgt on the model's stream, then the step; returns the
        mean over ranks of the step's mean loss and the (common) gradient norm."""
        with self._on_model_stream(dtok):
            dtok.copy_(htok, non_blocking=True)
            dtgt.copy_(htgt, non_blocking=True)
        self.step(dtok, dtgt, step)
        loss, norm = self.model.last_step_stats()
        return self.mean_over_ranks(loss), norm

    def mean_over_ranks(self, value: float) -> float:
        if self.world == 1:
            return float(value)
        dev = self.model.state_tensor(GRADS).device
        t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
        return float(self._allreduce_mean(t).item())

    def eval_loss(self, tokens, targets) -> float:
        """Held-out loss of this rank's batch, averaged across ranks."""
        return self.mean_over_ranks(self.model.eval_loss(tokens, targets))

    def replicas_agree(self) -> bool:
        """Whether every rank holds bit-identical fp32 weights (an fp64 checksum's
        max and min over ranks coincide)."""
        p = self.model.state_tensor(PARAMS)
        w = torch.arange(1, p.numel() + 1, device=p.device, dtype=torch.float64).remainder_(977.0)
        c = torch.stack([torch.sum(p.double() * w), torch.sum(p.double())])
        if self.world == 1:
            return True
        hi, lo = c.clone(), -c
        with self._on_model_stream(c):
            dist.all_reduce(hi, op=dist.ReduceOp.MAX, group=self.group)
            dist.all_reduce(lo, op=dist.ReduceOp.MAX, group=self.group)
        return bool(torch.equal(hi, -lo))
