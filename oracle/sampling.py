"""Temperature / top-p (nucleus) sampling of one token from a row of logits.

TEST INFRASTRUCTURE ONLY (see the package header).

The sampling the model card's benchmark harness and prompting guide use
(ATLAS-OLMo-3-32B-Think-v4, "Benchmarks" and "Prompting guide for Think
models": temperature 0.6, top-p 0.95), written as nucleus sampling
(Holtzman et al., "The Curious Case of Neural Text Degeneration", 2019) with
the random draw passed in, so that a device implementation can be compared
token for token:

* p = softmax(z / T) over the vocabulary, in float64;
* the tokens are ordered by logit z, largest first (the order of p), equal
  logits by the lower index;
* the nucleus is the shortest prefix of that order whose mass reaches top_p
  (at least one token);
* with u uniform in [0, 1), the token is the first of the nucleus whose
  cumulative mass, divided by the nucleus mass, exceeds u.

Parity: pinned by tests/test_oracle_sampling.py (hand-computed cases,
brute-force enumeration of tiny rows, the greedy limits, shift and
temperature invariances, exact draw frequencies) and, for the nucleus and its
renormalised probabilities, by the ``transformers`` package's own temperature
and top-p logits processors (tests/test_oracle_library_sampling.py).
"""
from __future__ import annotations

import numpy as np


def probabilities(logits, temperature: float) -> np.ndarray:
    """softmax(logits / temperature) in float64."""
    if temperature <= 0:
        raise ValueError("temperature must be positive")
    z = np.asarray(logits, dtype=np.float64) / float(temperature)
    z = z - np.max(z)
    e = np.exp(z)
    return e / np.sum(e)


def order(keys) -> np.ndarray:
    """Token indices by key (logit or probability), largest first; equal keys
    by index."""
    k = np.asarray(keys, dtype=np.float64)
    # lexsort sorts by the last key first: -key descending, then index ascending
    return np.lexsort((np.arange(k.size), -k))


def nucleus(probs, top_p: float, keys=None):
    """(tokens of the nucleus in sampling order, their probabilities); the
    order follows `keys` (the logits) when given, else the probabilities."""
    if not (0.0 < top_p <= 1.0):
        raise ValueError("top_p must be in (0, 1]")
    p = np.asarray(probs, dtype=np.float64)
    idx = order(p if keys is None else keys)
    cum = np.cumsum(p[idx])
    # shortest prefix whose mass reaches top_p; float round-off may leave the
    # full sum a hair below 1, so the whole vocabulary is the fallback
    k = int(np.searchsorted(cum, top_p, side="left")) + 1
    k = min(max(k, 1), p.size)
    return idx[:k], p[idx[:k]]


def sample(logits, temperature: float, top_p: float, u: float) -> int:
    """The token drawn with u in [0, 1)."""
    if not (0.0 <= u < 1.0):
        raise ValueError("u must be in [0, 1)")
    toks, pk = nucleus(probabilities(logits, temperature), top_p, keys=logits)
    cum = np.cumsum(pk) / np.sum(pk)
    j = int(np.searchsorted(cum, u, side="right"))  # first cumulative mass > u
    return int(toks[min(j, toks.size - 1)])
