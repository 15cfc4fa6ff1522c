"""KV concentration under asynchronous continuous refill, and decode batches shaped by it.

KV4-RL (ai.info summary), "Key Contributions" item 1 and "Methodology in Plain English"
paragraph 1: scheduling cannot change the total attention work of a set of responses, only when
it happens.  A synchronous batch of B responses occupies its B decode slots until the longest
one finishes, M_B = max of B i.i.d. lengths.  Continuous refill gives a finished slot a new
response at once.  The same responses then need E[M_B] / E[L] times fewer decode steps, so each
step reads that much more KV.  Proposition 4.1 states this concentration factor
C_KV = E[M_B] / E[L] >= 1, strictly above 1 for any non-degenerate length distribution and
nondecreasing in B.  At a random step an occupied slot holds a length-biased response
(inspection paradox), which is why the async-refill decode batches are long-tailed.

This module computes the factor exactly, for a discrete or continuous length law, and
simulates both schedules.  It also draws snapshot decode batches (current context lengths of
the B slots at a random step of continuous refill).  All of this is host-side NumPy and is not
used by the decode kernels.
"""
from __future__ import annotations

import math

import numpy as np


def expected_max_discrete(values: np.ndarray, probs: np.ndarray, B: int) -> float:
    """E[max of B i.i.d. draws] of a discrete law on `values` (any order) with `probs`:
    sum_v v (F(v)^B - F(v-)^B), F the CDF."""
    v = np.asarray(values, np.float64)
    p = np.asarray(probs, np.float64)
    o = np.argsort(v)
    v, p = v[o], p[o] / p.sum()
    F = np.cumsum(p)
    Fm = np.concatenate([[0.0], F[:-1]])
    return float(np.sum(v * (F ** B - Fm ** B)))


def concentration_factor_discrete(values: np.ndarray, probs: np.ndarray, B: int) -> float:
    """C_KV = E[M_B] / E[L] of a discrete length law."""
    v = np.asarray(values, np.float64)
    p = np.asarray(probs, np.float64) / np.sum(probs)
    return expected_max_discrete(v, p, B) / float(np.sum(v * p))


def expected_max_continuous(survival, B: int, upper: float, n: int = 200001) -> float:
    """E[max of B i.i.d. non-negative draws] = integral over [0, inf) of 1 - (1 - S(x))^B, with S
    the survival function; evaluated by the trapezoid rule on [0, upper], with upper large enough
    for the tail beyond it to vanish."""
    x = np.linspace(0.0, upper, n)
    return float(np.trapezoid(1.0 - (1.0 - survival(x)) ** B, x))


def harmonic(B: int) -> float:
    return float(sum(1.0 / k for k in range(1, B + 1)))


def simulate_schedules(sample_lengths, B: int, n_responses: int, rng: np.random.Generator) -> dict:
    """Decode steps to finish the same n_responses responses (lengths from sample_lengths(rng, n),
    each >= 1) on B slots: synchronously (batches of B, each lasting its longest response) and with
    continuous refill (a slot takes the next response the step after its current one ends).  Also
    the KV tokens read (sum over decode steps of the occupied slots' context lengths), the same
    for both schedules.  Returns steps, KV reads and KV per step for both."""
    L = np.maximum(1, np.asarray(sample_lengths(rng, n_responses), np.int64))
    n = (L.size // B) * B
    L = L[:n]
    sync_steps = int(L.reshape(-1, B).max(axis=1).sum())
    # continuous refill: slot end times by repeatedly giving the next response to the slot that
    # frees first (a min-heap over slot free times)
    import heapq
    heap = [0] * B
    for x in L:
        t = heapq.heappop(heap)
        heapq.heappush(heap, t + int(x))
    async_steps = int(max(heap))
    work = int(np.sum(L * (L + 1) // 2))  # sum over responses of context lengths 1..L
    return {"sync_steps": sync_steps, "async_steps": async_steps, "kv_reads": work,
            "sync_kv_per_step": work / sync_steps, "async_kv_per_step": work / async_steps,
            "step_ratio": sync_steps / async_steps}


def async_snapshot(sample_lengths, B: int, rng: np.random.Generator, cap: int | None = None) -> np.ndarray:
    """Context lengths of the B slots at one decode step of steady-state continuous refill.  Each
    slot's current response is length-biased and its position is uniform within it.

    The refill is simulated (a finished slot takes the next response at once) until every slot
    has started at least two responses.  The simulation then runs on to a step t drawn uniformly
    from the next mean-length steps, refilling as it goes.  The result is, per slot, how many
    tokens of its current response exist at step t: between 1 and that response's length, at
    most cap."""
    pool = [np.maximum(1, np.asarray(sample_lengths(rng, 4 * B), np.int64))]
    k = 0

    def nxt() -> int:
        nonlocal k
        if k >= pool[-1].size:
            pool.append(np.maximum(1, np.asarray(sample_lengths(rng, 4 * B), np.int64)))
            k = 0
        v = int(pool[-1][k])
        k += 1
        return v

    free = np.zeros(B, np.int64)   # step at which each slot's current response ends
    start = np.zeros(B, np.int64)  # step at which it began
    count = np.zeros(B, np.int64)
    while count.min() < 2:
        s = int(np.argmin(free))
        start[s] = free[s]
        free[s] += nxt()
        count[s] += 1
    mean = float(np.mean(np.concatenate(pool)))
    t = int(free.min()) + int(rng.integers(0, max(1, int(mean))))
    while free.min() <= t:
        s = int(np.argmin(free))
        start[s] = free[s]
        free[s] += nxt()
    ctx = t - start + 1
    if cap is not None:
        ctx = np.minimum(ctx, cap)
    return ctx.astype(np.int64)


def exponential_lengths(mean: float, cap: int | None = None):
    """Sampler of ceil(Exp(mean)) lengths, optionally clipped to cap."""
    def f(rng: np.random.Generator, n: int) -> np.ndarray:
        x = np.ceil(rng.exponential(mean, size=n)).astype(np.int64)
        return np.minimum(x, cap) if cap is not None else x
    return f


def lognormal_lengths(median: float, sigma: float, cap: int | None = None):
    """Sampler of rint(lognormal(log median, sigma)) lengths (at least 1), optionally clipped."""
    def f(rng: np.random.Generator, n: int) -> np.ndarray:
        x = np.maximum(1, np.rint(rng.lognormal(math.log(median), sigma, size=n))).astype(np.int64)
        return np.minimum(x, cap) if cap is not None else x
    return f
