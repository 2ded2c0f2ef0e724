"""Device temperature / top-p sampling (w4a_sample) against the oracle, token
for token, on the same seeded logits and draws.  Where the oracle's decision
sits within 1e-9 of a boundary (the nucleus mass against top_p, or the
cumulative mass against the draw) either neighbour is accepted: the two sides
sum the same float64 masses in different orders."""
import numpy as np
import pytest
import torch

from oracle import sampling as sp
from w4_weight_only_b200 import synth

pytestmark = pytest.mark.gpu


def _margins(z, T, top_p, u):
    p = sp.probabilities(z, T)
    idx = sp.order(z)
    cum = np.cumsum(p[idx])
    k = min(int(np.searchsorted(cum, top_p, side="left")) + 1, p.size)
    m1 = min(abs(cum[k - 1] - top_p), abs(cum[k - 2] - top_p) if k >= 2 else 1.0)
    c = np.cumsum(p[idx[:k]]) / cum[k - 1]
    j = min(int(np.searchsorted(c, u, side="right")), k - 1)
    m2 = min(abs(c[j] - u), abs(c[j - 1] - u) if j >= 1 else 1.0)
    return min(m1, m2)


def _check(logits, T, top_p, u):
    from w4_weight_only_b200 import api
    got = api.sample(logits.cuda(), T, top_p, u.cuda()).cpu().numpy()
    z = logits.double().numpy()
    uu = u.double().numpy()
    for b in range(z.shape[0]):
        ref = sp.sample(z[b], T, top_p, float(uu[b]))
        if int(got[b]) != ref:
            assert _margins(z[b], T, top_p, float(uu[b])) < 1e-9, (b, int(got[b]), ref)


@pytest.mark.parametrize("T,top_p", [(0.6, 0.95), (1.0, 1.0), (0.3, 0.5), (2.0, 0.999)])
def test_full_vocab_rows(built_lib, cuda, T, top_p):
    B, V = 8, 100278
    logits = synth.logits_rows(17, B, V)
    u = synth.uniforms(18, B)
    _check(logits, T, top_p, u)


def test_many_draws_small_vocab(built_lib, cuda):
    B, V = 64, 37
    logits = synth.logits_rows(21, B, V, scale=1.0)
    u = synth.uniforms(22, B)
    for T, top_p in ((0.6, 0.95), (1.0, 0.3), (1.0, 1.0)):
        _check(logits, T, top_p, u)


def test_ties_signed_zero_and_single_token(built_lib, cuda):
    # equal logits go by the lower index; -0 and +0 are one logit
    row = torch.tensor([[1.0, 3.0, 3.0, 0.0, 3.0, -0.0, 0.0]], dtype=torch.float32)
    for top_p in (0.2, 0.5, 0.9, 1.0):
        for uv in (0.0, 0.2, 0.45, 0.7, 0.99):
            _check(row, 1.0, top_p, torch.tensor([uv], dtype=torch.float32))
    _check(torch.tensor([[0.5]], dtype=torch.float32), 0.6, 0.95, torch.tensor([0.7], dtype=torch.float32))


def test_greedy_limit_and_determinism(built_lib, cuda):
    from w4_weight_only_b200 import api
    logits = synth.logits_rows(31, 4, 100278).cuda()
    u = synth.uniforms(32, 4).cuda()
    a = api.sample(logits, 1.0, 1e-7, u)
    assert torch.equal(a.long().cpu(), logits.argmax(dim=1).cpu())
    b1 = api.sample(logits, 0.6, 0.95, u)
    b2 = api.sample(logits, 0.6, 0.95, u)
    assert torch.equal(b1, b2)


def test_rejects_bad_arguments(built_lib, cuda):
    from w4_weight_only_b200 import api, _abi
    logits = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    u = torch.zeros((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(_abi.W4AError):
        api.sample(logits, 0.0, 0.9, u)
    with pytest.raises(_abi.W4AError):
        api.sample(logits, 1.0, 1.5, u)
