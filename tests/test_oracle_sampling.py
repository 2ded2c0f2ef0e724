"""Pins of oracle.sampling (temperature / top-p sampling with a given draw)."""
import math

import numpy as np
import pytest

from oracle import sampling as sp


def test_hand_computed_nucleus():
    # p = [0.1, 0.2, 0.3, 0.4]; largest first: 3 (0.4), 2 (0.3), 1, 0.
    # top_p 0.65: 0.4 < 0.65 <= 0.7, so the nucleus is {3, 2}, renormalized
    # to 4/7 and 3/7.
    z = np.log([1.0, 2.0, 3.0, 4.0])
    toks, pk = sp.nucleus(sp.probabilities(z, 1.0), 0.65)
    assert list(toks) == [3, 2]
    assert np.allclose(pk, [0.4, 0.3])
    assert sp.sample(z, 1.0, 0.65, 0.0) == 3
    assert sp.sample(z, 1.0, 0.65, 0.5) == 3          # 0.5 < 4/7
    assert sp.sample(z, 1.0, 0.65, 4.0 / 7.0 + 1e-9) == 2
    assert sp.sample(z, 1.0, 0.65, 0.999) == 2
    # the boundary is inclusive: a prefix whose mass equals top_p is enough
    assert list(sp.nucleus(sp.probabilities(z, 1.0), 0.7)[0]) == [3, 2]


def test_ties_go_to_the_lower_index():
    z = np.zeros(4)
    toks, pk = sp.nucleus(sp.probabilities(z, 1.0), 0.5)
    assert list(toks) == [0, 1] and np.allclose(pk, [0.25, 0.25])
    assert sp.sample(z, 1.0, 0.5, 0.49) == 0
    assert sp.sample(z, 1.0, 0.5, 0.5) == 1


def _brute(z, T, top_p, u):
    """Enumeration with plain loops: exp, sort by (-p, index), prefix, walk."""
    m = max(z)
    w = [math.exp((v - m) / T) for v in z]
    s = sum(w)
    p = [x / s for x in w]
    ranked = sorted(range(len(p)), key=lambda i: (-p[i], i))
    kept, mass = [], 0.0
    for i in ranked:
        kept.append(i)
        mass += p[i]
        if mass >= top_p:
            break
    acc = 0.0
    for i in kept:
        acc += p[i] / mass
        if acc > u:
            return i
    return kept[-1]


@pytest.mark.parametrize("seed", range(20))
def test_matches_enumeration_on_tiny_rows(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 9))
    z = rng.normal(0.0, 2.0, n)
    if seed % 4 == 0:
        z[rng.integers(0, n)] = z[0]  # a tie
    T = float(rng.choice([0.6, 1.0, 1.7]))
    top_p = float(rng.choice([0.3, 0.95, 1.0]))
    for u in np.linspace(0.0, 0.999, 37):
        assert sp.sample(z, T, top_p, float(u)) == _brute(list(z), T, top_p, float(u))


def test_greedy_limits():
    rng = np.random.default_rng(7)
    z = rng.normal(0.0, 1.0, 1000)
    best = int(np.argmax(z))
    for u in (0.0, 0.3, 0.999):
        assert sp.sample(z, 1e-6, 0.95, u) == best     # temperature -> 0
        assert sp.sample(z, 1.0, 1e-12, u) == best     # nucleus of one token


def test_shift_and_temperature_invariance():
    rng = np.random.default_rng(11)
    z = rng.normal(0.0, 3.0, 500)
    for u in np.linspace(0.0, 0.999, 23):
        a = sp.sample(z, 0.6, 0.95, float(u))
        assert sp.sample(z + 123.0, 0.6, 0.95, float(u)) == a
        assert sp.sample(z / 0.6, 1.0, 0.95, float(u)) == a


def test_draw_frequencies_are_the_nucleus_distribution():
    """Over an even grid of draws each nucleus token is drawn exactly in
    proportion to its renormalized probability (to the grid's resolution)."""
    rng = np.random.default_rng(3)
    z = rng.normal(0.0, 1.5, 50)
    toks, pk = sp.nucleus(sp.probabilities(z, 0.6), 0.95)
    assert pk.sum() >= 0.95 and pk[:-1].sum() < 0.95
    N = 20000
    counts = {}
    for i in range(N):
        t = sp.sample(z, 0.6, 0.95, (i + 0.5) / N)
        counts[t] = counts.get(t, 0) + 1
    assert set(counts) <= set(int(t) for t in toks)
    for t, q in zip(toks, pk / pk.sum()):
        assert abs(counts.get(int(t), 0) / N - q) <= 1.0 / N + 1e-12


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        sp.sample([0.0, 1.0], 0.0, 0.9, 0.5)
    with pytest.raises(ValueError):
        sp.sample([0.0, 1.0], 1.0, 0.0, 0.5)
    with pytest.raises(ValueError):
        sp.sample([0.0, 1.0], 1.0, 0.9, 1.0)
