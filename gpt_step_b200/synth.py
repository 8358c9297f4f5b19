"""Seeded synthetic inputs for the GPT-2 training step.

This module is the only code shared by the CUDA path's callers (tests, bench)
and the CPU oracle's callers. It holds none of the training step's arithmetic:
it only draws token streams and arbitrary test tensors from a seed.

Token streams stand in for the corpus the pages train on (FineWeb's 10B-token
sample tokenised with GPT-2's byte-level BPE, each document preceded by an
end-of-text marker -- "Pretraining and adapting a language model on a
dependency-free stack", §4.2, Fig. 2), which is not available here:

* document lengths are Geometric(p = 1/mean) on {1, 2, ...};
* every document is preceded by the end-of-text id (``eot``);
* document tokens are iid Zipf(s) over the non-EOT ids ``{0 .. V-2}``,
  P(id = k) proportional to (k + 1) ** -s, drawn by inverse CDF;
* the stream is cut into consecutive windows of T + 1 ids; inputs are the
  first T ids of a window and targets the last T.

The tiny configuration instead uses a uniform iid stream of B*T + 1 ids whose
inputs are ``stream[:-1]`` and targets ``stream[1:]``.
"""
from __future__ import annotations

import numpy as np


def zipf_cdf(n_ids: int, s: float = 1.1) -> np.ndarray:
    """Cumulative distribution of Zipf(s) over ids 0..n_ids-1."""
    w = (np.arange(1, n_ids + 1, dtype=np.float64)) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_document_stream(n_tokens: int, vocab_real: int, eot: int,
                         mean_doc_len: float, seed: int, s: float = 1.1) -> np.ndarray:
    """Return ``n_tokens`` int32 ids: EOT-preceded documents of Zipf tokens.

    ``eot`` must be ``vocab_real - 1``; document tokens are drawn from the
    other ``vocab_real - 1`` ids.
    """
    if eot != vocab_real - 1:
        raise ValueError("the end-of-text id is the last real id")
    rng = np.random.default_rng(seed)
    out = np.empty(n_tokens, dtype=np.int32)
    cdf = zipf_cdf(vocab_real - 1, s)
    pos = 0
    p = 1.0 / float(mean_doc_len)
    while pos < n_tokens:
        # draw document lengths in bulk; each document costs length + 1 ids
        lens = rng.geometric(p, size=max(16, int((n_tokens - pos) * p) + 16))
        for L in lens:
            if pos >= n_tokens:
                break
            out[pos] = eot
            pos += 1
            take = int(min(L, n_tokens - pos))
            if take > 0:
                u = rng.random(take)
                out[pos:pos + take] = np.minimum(np.searchsorted(cdf, u, side="right"),
                                                 vocab_real - 2)
                pos += take
    return out


def windows(stream: np.ndarray, batch: int, seq_len: int, first_window: int = 0):
    """Cut consecutive windows of seq_len + 1 ids; return (inputs, targets) [B, T] int32."""
    w = seq_len + 1
    need = (first_window + batch) * w
    if stream.size < need:
        raise ValueError("stream too short for the requested windows")
    chunk = stream[first_window * w: need].reshape(batch, w)
    return (np.ascontiguousarray(chunk[:, :seq_len], dtype=np.int32),
            np.ascontiguousarray(chunk[:, 1:], dtype=np.int32))


def uniform_next_token_batch(batch: int, seq_len: int, vocab_real: int, seed: int):
    """Tiny-configuration batch: uniform iid stream of B*T+1 ids, shifted by one."""
    rng = np.random.default_rng(seed)
    s = rng.integers(0, vocab_real, size=batch * seq_len + 1, dtype=np.int64).astype(np.int32)
    return (np.ascontiguousarray(s[:-1].reshape(batch, seq_len)),
            np.ascontiguousarray(s[1:].reshape(batch, seq_len)))


class TokenSource:
    """Micro-batches for a configuration, consumed in stream order."""

    def __init__(self, batch: int, seq_len: int, vocab_real: int, seed: int,
                 mean_doc_len: float | None, n_windows: int):
        self.batch, self.seq_len = batch, seq_len
        self.vocab_real = vocab_real
        if mean_doc_len is None:
            self.stream = None
            self.seed = seed
        else:
            self.stream = zipf_document_stream(n_windows * (seq_len + 1), vocab_real,
                                               vocab_real - 1, mean_doc_len, seed)
        self.n_windows = n_windows
        self.next = 0

    def get(self):
        if self.stream is None:
            x, y = uniform_next_token_batch(self.batch, self.seq_len, self.vocab_real,
                                            self.seed + self.next)
            self.next += 1
            return x, y
        if self.next + self.batch > self.n_windows:
            self.next = 0
        x, y = windows(self.stream, self.batch, self.seq_len, self.next)
        self.next += self.batch
        return x, y


def random_tensor(shape, seed: int, scale: float = 1.0, dtype=np.float32) -> np.ndarray:
    """Arbitrary normal test values (not a model initialisation)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(dtype)
