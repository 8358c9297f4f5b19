"""Data parallelism: the multi-card arrangement of the training step.

"Pretraining and adapting a language model on a dependency-free stack" §4.4:
every card runs the same model on its own micro-batches (19 sequences x 9
accumulation steps per card, three cards); once per optimizer step the
gradients are averaged across the cards, so that each card's clip + AdamW sees
the gradient of the whole global batch and the copies stay identical; held-out
losses are averaged across cards in the same way.

Two forms of the exchange, both through torch.distributed (NCCL between GPUs
over NVLink / NVSwitch, gloo for the CPU tests), on views of the model's flat
state arrays (``gpt2_state_device_ptr``):

``zero1`` (default): the optimizer state is sharded. The flat layout holds the
    1-D parameters in region 0 and the 2-D weights in buckets, in the order the
    backward pass finishes their gradients (one per block from the last, then
    {wpe, wte}). The library records one CUDA event per bucket during every
    backward pass; after the last micro-step's ``fwd_bwd`` has been enqueued,
    a communication stream waits on each bucket's event and reduce-scatters
    (averages) that bucket at once, so the exchange of block l overlaps the
    backward of blocks l-1 .. 0. Region 0 (0.5 MB) is all-reduced at the end.
    Each rank then takes the sum of squares of its shards (rank 0 adds region
    0), all-reduces that scalar, updates region 0 and its own shards with the
    global norm (``gpt2_clip_adamw_ranges``), and the bf16 weights of every
    bucket are all-gathered. Per rank the update touches 1/N of the 2-D
    weights; the gradient traffic equals an all-reduce's half, the weight
    traffic is bf16.
``allreduce``: one all-reduce (average) of the whole fp32 gradient array
    between the last backward and an unchanged clip + AdamW on every rank.

Host logic only; the model is anything with the calls used below.
"""
from __future__ import annotations

import contextlib

import torch
import torch.distributed as dist

PARAMS, GRADS, ADAM_M, ADAM_V, WEIGHTS_BF16 = 0, 1, 2, 3, 4   # the C ABI's state selectors


class DataParallel:
    def __init__(self, model, group=None, mode: str = "zero1", overlap: bool = True):
        if mode not in ("zero1", "allreduce"):
            raise ValueError(mode)
        self.model = model
        self.group = group
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        self.backend = dist.get_backend(group) if on else None
        self.mode = mode
        self.overlap = overlap
        self.comm = None
        if mode == "zero1":
            self._setup_zero1()

    # -- helpers ------------------------------------------------------------------------------
    def _stream(self):
        return getattr(self.model, "stream", None)

    def _on(self, t, stream=None):
        s = stream if stream is not None else self._stream()
        if t.is_cuda and s is not None:
            return torch.cuda.stream(s)
        return contextlib.nullcontext()

    def _avg_inplace(self, t):
        if self.backend == "nccl":
            dist.all_reduce(t, op=dist.ReduceOp.AVG, group=self.group)
        else:  # gloo has no AVG
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
            t.mul_(1.0 / self.world)

    def _allreduce_mean(self, t):
        """In place, on the model's stream: t <- mean over ranks of t."""
        if self.world == 1:
            return t
        with self._on(t):
            self._avg_inplace(t)
        return t

    def _reduce_scatter_avg(self, full, shard):
        """shard (this rank's slice of `full`) <- the mean over ranks of that slice."""
        if self.backend == "nccl":
            dist.reduce_scatter_tensor(shard, full, op=dist.ReduceOp.AVG, group=self.group)
        else:
            out = torch.empty_like(shard)
            dist.reduce_scatter_tensor(out, full, op=dist.ReduceOp.SUM, group=self.group)
            shard.copy_(out.mul_(1.0 / self.world))

    def _all_gather(self, full, shard):
        if self.backend == "nccl":
            dist.all_gather_into_tensor(full, shard, group=self.group)
        else:
            dist.all_gather_into_tensor(full, shard.clone(), group=self.group)

    # -- sharded (ZeRO-1) form ------------------------------------------------------------------
    def _setup_zero1(self):
        m = self.model
        self.region0 = m.bucket_range(-1)
        self.buckets = [m.bucket_range(b) for b in range(m.num_buckets())]
        for lo, hi in self.buckets:
            if (hi - lo) % (64 * self.world):
                raise ValueError(f"world size {self.world} does not split the buckets into 64-element shards "
                                 "(it must divide 120)")
        self.shards = []
        for lo, hi in self.buckets:
            n = (hi - lo) // self.world
            self.shards.append((lo + self.rank * n, lo + (self.rank + 1) * n))
        g = m.state_tensor(GRADS)
        self.sumsq = torch.zeros(1, dtype=torch.float64, device=g.device)
        self.events = None
        if g.is_cuda and self.world > 1 and self.overlap:
            self.comm = torch.cuda.Stream(device=g.device)
            self.events = [torch.cuda.Event() for _ in self.buckets]
            m.set_bucket_events(self.events)

    def update_ranges(self):
        """Element ranges this rank updates: region 0 (every rank) and its shard of each bucket."""
        return [self.region0] + self.shards

    def _zero1_exchange_grads(self):
        g = self.model.state_tensor(GRADS)
        r0lo, r0hi = self.region0
        if self.comm is not None:
            # bucket b's reduce-scatter starts when the backward has finished bucket b
            with torch.cuda.stream(self.comm):
                for b, ((lo, hi), (slo, shi)) in enumerate(zip(self.buckets, self.shards)):
                    self.comm.wait_event(self.events[b])
                    self._reduce_scatter_avg(g[lo:hi], g[slo:shi])
                self._avg_inplace(g[r0lo:r0hi])
            self._stream().wait_stream(self.comm)
        else:
            with self._on(g):
                for (lo, hi), (slo, shi) in zip(self.buckets, self.shards):
                    self._reduce_scatter_avg(g[lo:hi], g[slo:shi])
                self._avg_inplace(g[r0lo:r0hi])

    def _zero1_update(self, step: int):
        m = self.model
        w = m.state_tensor(WEIGHTS_BF16)
        norm_ranges = list(self.shards) + ([self.region0] if self.rank == 0 else [])
        m.grad_sumsq(norm_ranges, self.sumsq)
        with self._on(self.sumsq):
            dist.all_reduce(self.sumsq, op=dist.ReduceOp.SUM, group=self.group)
        m.clip_adamw_ranges(step, self.update_ranges(), self.sumsq)
        with self._on(w):
            for (lo, hi), (slo, shi) in zip(self.buckets, self.shards):
                self._all_gather(w[lo:hi], w[slo:shi])

    # -- the step -------------------------------------------------------------------------------
    def sync_grads(self):
        """All-reduce form: average the accumulated gradients across ranks (no-op on one rank)."""
        if self.world > 1:
            self._allreduce_mean(self.model.state_tensor(GRADS))

    def update(self, step: int):
        """Everything between the last micro-step and the next forward: the exchange and the update."""
        if self.world == 1:
            self.model.clip_adamw(step)
        elif self.mode == "allreduce":
            self.sync_grads()
            self.model.clip_adamw(step)
        else:
            self._zero1_exchange_grads()
            self._zero1_update(step)

    def step(self, tokens, targets, step: int):
        """One optimizer step: the rank's micro-batches, the exchange, the update."""
        for x, y in zip(tokens, targets):
            self.model.fwd_bwd(x, y)
        self.update(step)

    def step_host(self, htok, htgt, dtok, dtgt, step: int):
        """The same from host (pinned) micro-batches [A, B, T]: copied into the device
        staging tensors dtok / dtgt on the model's stream, then the step; returns the
        mean over ranks of the step's mean loss and the (common) gradient norm."""
        with self._on(dtok):
            dtok.copy_(htok, non_blocking=True)
            dtgt.copy_(htgt, non_blocking=True)
        self.step(dtok, dtgt, step)
        loss, norm = self.model.last_step_stats()
        return self.mean_over_ranks(loss), norm

    def gather_state(self):
        """Sharded form: make every rank's fp32 masters and Adam moments whole (each
        bucket all-gathered from its owners), e.g. before rank 0 writes a
        checkpoint. Collective: every rank calls it. No-op in the all-reduce form."""
        if self.mode != "zero1" or self.world == 1:
            return
        for what in (PARAMS, ADAM_M, ADAM_V):
            t = self.model.state_tensor(what)
            with self._on(t):
                for (lo, hi), (slo, shi) in zip(self.buckets, self.shards):
                    self._all_gather(t[lo:hi], t[slo:shi])

    def mean_over_ranks(self, value: float) -> float:
        if self.world == 1:
            return float(value)
        g = self.model.state_tensor(GRADS)
        with self._on(g):       # built, reduced and read on the model's stream
            t = torch.tensor([float(value)], dtype=torch.float64, device=g.device)
            self._avg_inplace(t)
            return float(t.item())

    def eval_loss(self, tokens, targets) -> float:
        """Held-out loss of this rank's batch, averaged across ranks."""
        return self.mean_over_ranks(self.model.eval_loss(tokens, targets))

    def replicas_agree(self) -> bool:
        """Whether every rank computes with identical weights: an fp64 checksum of the
        weights the forward reads (all fp32 masters in the all-reduce form; region 0
        in fp32 and the bf16 copy in the sharded form) has equal max and min over ranks."""
        m = self.model
        with self._on(m.state_tensor(GRADS)):
            if self.mode == "zero1":
                r0lo, r0hi = self.region0
                parts = [m.state_tensor(PARAMS)[r0lo:r0hi].double(), m.state_tensor(WEIGHTS_BF16).double()]
            else:
                parts = [m.state_tensor(PARAMS).double()]
            sums = []
            for p in parts:
                w = torch.arange(1, p.numel() + 1, device=p.device, dtype=torch.float64).remainder_(977.0)
                sums += [torch.sum(p * w), torch.sum(p)]
            c = torch.stack(sums)
            if self.world == 1:
                return True
            hi, lo = c.clone(), -c
            dist.all_reduce(hi, op=dist.ReduceOp.MAX, group=self.group)
            dist.all_reduce(lo, op=dist.ReduceOp.MAX, group=self.group)
            return bool(torch.equal(hi, -lo))
