"""Device-side failures are reported through the workspace's error word.

* A bounded wait that runs out: the environment variable
  W4A_BARRIER_WAIT_CYCLES bounds the waits of a CTA for the other CTAs (grid
  barrier, attention segment merge).  Set to a few dozen cycles, the first
  grid barrier of a decode step cannot complete in time; the launch records
  the timeout, unwinds (every CTA leaves at its next wait, copies in flight
  land first) and w4a_check returns W4A_ERR_TIMEOUT.  With the bound back to
  its default and the workspace zeroed, the next step gives the same bits as
  before.  No wait is left unbounded and nothing traps.
* A token id outside the vocabulary and a position outside the cache: the
  kernel clamps the token before it reads the embedding and attends no keys
  for the bad position (no cache row is written), and reports
  W4A_ERR_KERNEL.
"""
import os

import pytest
import torch

from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import Pair

pytestmark = pytest.mark.gpu


def _abi():
    from w4_weight_only_b200 import _abi
    return _abi


@pytest.fixture(scope="module")
def pair(built_lib, cuda):
    return Pair(wc.tiny(), seed=0, gen_device="cpu")


def _prefilled(P):
    from w4_weight_only_b200 import api
    kv = api.KVCache(P.cfg, 1, 64)
    P.gpu.prefill(kv, synth.token_ids(11, 20, P.cfg.vocab, "cpu").to("cuda"), want_logits=False)
    P.gpu.check()
    return kv


def _step(P, kv, tok, pos):
    return P.gpu.decode_step(kv, torch.tensor([tok], dtype=torch.int32, device="cuda"),
                             torch.tensor([pos], dtype=torch.int32, device="cuda"))


def test_barrier_timeout_reported_then_recovers(pair):
    abi = _abi()
    P = pair
    kv = _prefilled(P)
    snap = kv.mem.clone()
    good, _ = _step(P, kv, 9, 20)
    good = good.clone()
    P.gpu.check()
    kv.mem.copy_(snap)
    os.environ["W4A_BARRIER_WAIT_CYCLES"] = "32"
    try:
        _step(P, kv, 9, 20)
        with pytest.raises(abi.W4AError) as e:
            P.gpu.check()
    finally:
        del os.environ["W4A_BARRIER_WAIT_CYCLES"]
    assert e.value.code == abi.ERR_TIMEOUT
    # the context still works: zero the workspace, restore the cache, step again
    P.gpu.workspace(1).zero_()
    kv.mem.copy_(snap)
    again, _ = _step(P, kv, 9, 20)
    P.gpu.check()
    assert torch.equal(again, good)


def test_bad_token_and_position_reported(pair):
    abi = _abi()
    P = pair
    cfg = P.cfg
    kv = _prefilled(P)
    for tok, pos in ((cfg.vocab, 20), (-1, 20), (3, kv.max_ctx), (3, -5)):
        P.gpu.workspace(1).zero_()
        _step(P, kv, tok, pos)
        with pytest.raises(abi.W4AError) as e:
            P.gpu.check()
        assert e.value.code == abi.ERR_KERNEL, (tok, pos)
    P.gpu.workspace(1).zero_()
    _step(P, kv, 3, 21)
    P.gpu.check()
