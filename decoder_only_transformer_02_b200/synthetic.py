"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke run.

This module draws numbers only: it holds none of the model's arithmetic, and it
is the one piece of code that both the CUDA path's callers and the CPU oracle's
callers use.  It imports neither the oracle nor the CUDA binding.

The pages train on a web-text dataset that is not available here; a finite
Zipf(s) distribution over the real vocabulary stands in for natural-text unigram
statistics (id r-1 has probability proportional to r^-s, so id 0 is the most
frequent).  Batches are cut from one token stream the way a plain data loader
does it: inputs are a window of the stream and targets the same window shifted
by one token.
"""
from __future__ import annotations

import numpy as np


def zipf_stream(n: int, vocab: int, s: float = 1.1, seed: int = 0) -> np.ndarray:
    """n int32 token ids in [0, vocab) drawn i.i.d. from a finite Zipf(s)."""
    rng = np.random.default_rng(seed)
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    w = ranks ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def uniform_stream(n: int, vocab: int, seed: int = 0) -> np.ndarray:
    """n int32 token ids uniform in [0, vocab)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def micro_batches(stream: np.ndarray, B: int, T: int, n_micro: int):
    """Cut n_micro (tokens, targets) pairs of shape [B,T] out of one stream of
    at least n_micro*B*T + 1 ids: micro-step k reads stream[k*B*T : (k+1)*B*T]
    as inputs and the same window shifted by one as targets."""
    need = n_micro * B * T + 1
    assert stream.size >= need, (stream.size, need)
    out = []
    for k in range(n_micro):
        lo = k * B * T
        x = stream[lo:lo + B * T].reshape(B, T)
        y = stream[lo + 1:lo + B * T + 1].reshape(B, T)
        out.append((np.ascontiguousarray(x), np.ascontiguousarray(y)))
    return out


def token_batches(kind: str, vocab: int, B: int, T: int, n_micro: int = 1, seed: int = 0):
    """Micro-batches from a fresh stream: kind 'zipf' (s = 1.1) or 'uniform'."""
    n = n_micro * B * T + 1
    if kind == "zipf":
        stream = zipf_stream(n, vocab, 1.1, seed)
    elif kind == "uniform":
        stream = uniform_stream(n, vocab, seed)
    else:
        raise ValueError(kind)
    return micro_batches(stream, B, T, n_micro)


def normal_array(shape, seed: int = 0, dtype=np.float32) -> np.ndarray:
    """i.i.d. N(0, 1) values (e.g. attention q/k/v/dO for the standalone
    attention workload)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal(size=shape).astype(dtype)
