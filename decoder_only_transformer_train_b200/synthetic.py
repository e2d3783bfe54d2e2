"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

The training data of the pages (Tiny Shakespeare, FineWeb-Edu token shards) is not
available, so token batches are drawn from a seeded Zipf(s) law over the real
vocabulary, with the same shapes as the pages' workload: a flat run of B*T+1 ids,
inputs = run[:-1], targets = run[1:] ("Karpathy's Zero to Hero, Lecture 9: Reproduce
GPT-2 (124M) — notes", section "41:44 – 52:38 From random weights to a first batch",
the B*T+1 batching trick).

This module holds no arithmetic of the method itself: it only produces inputs.
All randomness is counter based (SplitMix64, Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014), so any element can be regenerated
from (seed, stream, index) alone.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser (variant 13 of Stafford's mixers)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(state: int, index: np.ndarray) -> np.ndarray:
    """The index-th output (0-based) of the SplitMix64 sequence started at `state`."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(state & 0xFFFFFFFFFFFFFFFF) + (idx + np.uint64(1)) * _GAMMA)


def stream_state(seed: int, stream: int) -> int:
    """Independent sub-stream `stream` of a seed: the stream-th SplitMix64 output of the seed."""
    return int(splitmix64(seed, np.array([stream], dtype=np.uint64))[0])


def uniform01(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """n doubles in [0, 1) with 53 random bits each."""
    s = stream_state(seed, stream)
    r = splitmix64(s, np.arange(offset, offset + n, dtype=np.uint64))
    return (r >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normal doubles (Box–Muller on pairs of counter-based uniforms)."""
    u = uniform01(seed, stream, 2 * n).reshape(n, 2)
    u1 = 1.0 - u[:, 0]                      # (0, 1]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u[:, 1])


def zipf_cdf(vocab: int, s: float = 1.1) -> np.ndarray:
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_tokens(seed: int, n: int, vocab: int, s: float = 1.1, stream: int = 0,
                offset: int = 0) -> np.ndarray:
    """n token ids in [0, vocab) with P(k) proportional to (k+1)^-s, int32."""
    u = uniform01(seed, stream, n, offset)
    ids = np.searchsorted(zipf_cdf(vocab, s), u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def token_batch(seed: int, B: int, T: int, vocab: int, micro_step: int = 0,
                s: float = 1.1) -> tuple[np.ndarray, np.ndarray]:
    """(inputs, targets), each int32 [B, T], from one run of B*T+1 Zipf ids.

    Micro-step k of an accumulation loop reads the k-th consecutive run, so a
    stream of grad_accum_steps micro-batches is one seeded token stream.
    """
    run = zipf_tokens(seed, B * T + 1, vocab, s, stream=0, offset=micro_step * B * T)
    return run[:-1].reshape(B, T).copy(), run[1:].reshape(B, T).copy()


def ignore_mask(seed: int, n: int, frac: float = 0.01, stream: int = 7) -> np.ndarray:
    """Boolean [n]: True where a target is replaced by the ignore index -1."""
    return uniform01(seed, stream, n) < frac


def uniform_targets(seed: int, n: int, vocab: int, stream: int = 5) -> np.ndarray:
    u = uniform01(seed, stream, n)
    return np.minimum((u * vocab).astype(np.int64), vocab - 1).astype(np.int32)
