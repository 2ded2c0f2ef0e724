"""The sampling oracle's nucleus against an independent library (CPU).

The model card ("Benchmarks", "Prompting guide for Think models") samples with
temperature 0.6 and top-p 0.95 through the usual generate call and defines
neither further; the oracle reads them as published nucleus sampling.  The
``transformers`` package's own temperature and top-p logits processors, run in
float64, keep a set of tokens and a renormalised distribution that must be the
oracle's nucleus and its probabilities: this fixes the temperature placement
(dividing the logits before the softmax) and the nucleus boundary (the
shortest most-probable prefix whose mass reaches top-p, the token that crosses
it included).
"""
import numpy as np
import pytest
import torch

from oracle import sampling

transformers = pytest.importorskip("transformers")
from transformers.generation.logits_process import TemperatureLogitsWarper, TopPLogitsWarper  # noqa: E402


def _library_nucleus(logits, temperature, top_p):
    scores = torch.from_numpy(np.asarray(logits, np.float64))[None]
    ids = torch.zeros((1, 1), dtype=torch.long)
    scores = TemperatureLogitsWarper(temperature)(ids, scores)
    scores = TopPLogitsWarper(top_p)(ids, scores)[0]
    kept = torch.nonzero(torch.isfinite(scores)).flatten().numpy()
    return kept, torch.softmax(scores, -1).numpy()


@pytest.mark.parametrize("vocab,scale", [(1000, 1.0), (1000, 4.0), (100278, 3.0)])
@pytest.mark.parametrize("temperature,top_p", [(0.6, 0.95), (1.0, 0.95), (0.6, 0.5), (1.3, 0.9)])
def test_nucleus_matches_library(vocab, scale, temperature, top_p):
    r = np.random.default_rng(vocab + int(10 * scale) + int(100 * top_p))
    for _ in range(4):
        logits = r.standard_normal(vocab) * scale
        toks, pk = sampling.nucleus(sampling.probabilities(logits, temperature), top_p, keys=logits)
        kept, lib_p = _library_nucleus(logits, temperature, top_p)
        assert np.array_equal(np.sort(toks), kept)
        assert np.allclose(pk / pk.sum(), lib_p[toks], rtol=1e-12, atol=1e-300)
        assert lib_p[np.setdiff1d(np.arange(vocab), toks)].max(initial=0.0) == 0.0


def test_single_dominant_token_is_kept_alone():
    logits = np.zeros(50)
    logits[17] = 40.0
    toks, _ = sampling.nucleus(sampling.probabilities(logits, 0.6), 0.95, keys=logits)
    kept, _ = _library_nucleus(logits, 0.6, 0.95)
    assert list(toks) == [17] and list(kept) == [17]
