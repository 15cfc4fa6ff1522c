"""KV concentration (KV4-RL, "Key Contributions" item 1, Proposition 4.1): C_KV = E[M_B] / E[L],
pinned to what the mathematics fixes.

- For exponential lengths of mean mu, E[max of B] = mu * H_B (the harmonic number): the textbook
  identity (the k-th spacing of B exponentials is exponential with rate (B - k + 1) / mu).
- Brute force over every outcome of a small discrete law.
- The proposition's own claims: C_KV >= 1, = 1 for a degenerate law, > 1 otherwise,
  nondecreasing in B.
- The schedule simulation's step ratio converges to C_KV.
- Snapshot context lengths of continuous refill with exponential lengths are again exponential
  with the same mean (memorylessness).
"""
import itertools

import numpy as np
import pytest

from int4_kv_cache_append_b200 import concentration as C


@pytest.mark.parametrize("B", [1, 2, 8, 64, 256])
def test_exponential_max_is_harmonic(B):
    mu = 6144.0
    em = C.expected_max_continuous(lambda x: np.exp(-x / mu), B, upper=60 * mu, n=600001)
    assert em / mu == pytest.approx(C.harmonic(B), rel=1e-6)


def test_discrete_expected_max_brute_force():
    values, probs = np.array([3.0, 10.0, 1.0]), np.array([0.5, 0.2, 0.3])
    for B in (1, 2, 3, 4):
        exact = 0.0
        for combo in itertools.product(range(3), repeat=B):
            exact += np.prod(probs[list(combo)]) * values[list(combo)].max()
        assert C.expected_max_discrete(values, probs, B) == pytest.approx(exact, rel=1e-12)


def test_proposition_properties():
    assert C.concentration_factor_discrete([7.0], [1.0], 64) == pytest.approx(1.0, abs=1e-12)
    rng = np.random.default_rng(3)
    for _ in range(20):
        n = int(rng.integers(2, 8))
        v = rng.integers(1, 1000, size=n).astype(float)
        if np.unique(v).size < 2:
            continue
        p = rng.random(n) + 0.01
        prev = 1.0
        for B in (1, 2, 3, 8, 32, 256):
            c = C.concentration_factor_discrete(v, p, B)
            assert c >= prev - 1e-12
            prev = c
        assert C.concentration_factor_discrete(v, p, 1) == pytest.approx(1.0, abs=1e-12)
        assert C.concentration_factor_discrete(v, p, 2) > 1.0


def test_simulated_step_ratio_converges_to_the_factor():
    values = np.array([200, 1000, 6000])
    probs = np.array([0.5, 0.3, 0.2])

    def sample(rng, n):
        return rng.choice(values, size=n, p=probs)

    B = 16
    r = C.simulate_schedules(sample, B, B * 4000, np.random.default_rng(7))
    assert r["step_ratio"] == pytest.approx(C.concentration_factor_discrete(values, probs, B), rel=0.03)
    # the same KV reads land in fewer steps: KV per step scales by the same ratio
    assert r["async_kv_per_step"] / r["sync_kv_per_step"] == pytest.approx(r["step_ratio"], rel=1e-12)


def test_snapshot_of_exponential_lengths_is_exponential():
    mu = 500.0
    rng = np.random.default_rng(11)
    snaps = np.concatenate([C.async_snapshot(C.exponential_lengths(mu), 64, rng) for _ in range(60)])
    assert snaps.min() >= 1
    assert snaps.mean() == pytest.approx(mu, rel=0.06)
    # exponential: median = mu ln 2
    assert np.median(snaps) == pytest.approx(mu * np.log(2.0), rel=0.08)
