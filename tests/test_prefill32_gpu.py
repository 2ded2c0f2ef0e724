"""w4a_prefill at the full OLMo-3-32B shape against the oracle's prefill.

The model: two layers of the 32B shape (a sliding-window layer and a full
YaRN layer), the full vocabulary (seed 5).  Prompts of 1,200 uniform token ids
(ATLAS-OLMo-3-32B-Think-v4 model card, "Performance & footprint": TTFT at
~1.2K context):

* from position 0 (the time-to-first-token case);
* continuing at position 3,500 after a pre-filled N(0, 1) history, so that
  the 4,096-slot ring of the sliding-window layer wraps during the prompt.

Checks: the last token's logits, and its greedy token when the oracle's
top-2 gap exceeds 2 x the logit bound, and the K and V rows the prefill wrote
for sampled positions of both layers, within 2e-2 of the RMS of the oracle's
rows (they are bf16 roundings of values derived from the layer inputs).  The
oracle runs its layer-at-a-time prefill, pinned against sequential decode.

The logit bound: every prompt token, the last one included, runs through the
dense path, whose tensor-core products take q and the attention
probabilities rounded once to bf16 (relative 2^-9 each, uniform), where the
decode step carries both as hi + lo bf16 pairs.  The logits' error is then
roughly normal with an RMS near 7e-3 (the final hidden state's ~0.5 %
relative error times the lm_head's gain, 0.02 sqrt(d) ~ 1.4), so its maximum
over 100,278 logits sits near 4.4 RMS ~ 3e-2: the test bounds the RMS at
1e-2 and the maximum at 4.5e-2.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import Pair

pytestmark = pytest.mark.gpu

LOGIT_TOL = 4.5e-2
LOGIT_RMS = 1e-2
KV_TOL = 2e-2
T = 1200


@pytest.fixture(scope="module")
def pair(built_lib, cuda):
    c = wc.olmo3_32b(2)
    c.full_layers = [False, True]
    return Pair(c, seed=5, gen_device="cuda", oracle_cache=True, oracle_fast=True)


def _history(P, kv, okv, n):
    cfg = P.cfg
    for l in range(cfg.n_layers):
        k, v = synth.kv_rows(P.seed + 100, l, 0, cfg.n_kv_heads, n, cfg.head_dim, "cuda")
        kv.fill_history(l, 0, k, v)
        okv.fill(l, 0, 0, k.cpu().double().numpy(), v.cpu().double().numpy())


@pytest.mark.parametrize("start", [0, 3500])
def test_prefill_1200_tokens_full_shape(pair, start):
    from w4_weight_only_b200 import api
    P = pair
    cfg = P.cfg
    cap = (start + T + 15) // 16 * 16
    kv = api.KVCache(cfg, 1, cap)
    okv = om.OracleKV(P.ocfg, 1, cap)
    if start:
        _history(P, kv, okv, start)
    toks = synth.token_ids(P.seed, T, cfg.vocab, "cpu", "prefill", start)
    last = P.gpu.prefill(kv, toks.to("cuda"), seq=0, start_pos=start)
    P.gpu.check()
    ref, _ = om.prefill_layers(P.oracle, okv, toks.numpy(), b=0, start_pos=start)
    got = last.cpu().numpy().astype(np.float64)
    err = float(np.max(np.abs(got - ref)))
    rms = float(np.sqrt(np.mean((got - ref) ** 2)))
    assert err <= LOGIT_TOL and rms <= LOGIT_RMS, (err, rms)
    top2 = np.sort(ref)[-2:]
    if top2[1] - top2[0] >= 2 * LOGIT_TOL:
        assert int(np.argmax(got)) == int(np.argmax(ref))
    positions = sorted({start, start + 1, start + T // 2, start + T - 2, start + T - 1,
                        min(start + T - 1, max(start, 4095)), min(start + T - 1, 4096)})
    for l in range(cfg.n_layers):
        sl = kv.slots(l)
        for pos in positions:
            k, v = kv.read(l, 0, pos % sl, 1)
            for name, g, r in (("K", k, okv.K[l][0, :, pos]), ("V", v, okv.V[l][0, :, pos])):
                g = g[:, 0].float().cpu().numpy().astype(np.float64)
                e = float(np.max(np.abs(g - r))) / float(np.sqrt(np.mean(r * r)))
                assert e <= KV_TOL, (name, l, pos, e)
