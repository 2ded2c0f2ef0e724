"""KVCache.fill_history: a sequence's positions land where the engine reads
them (a layer with room for every position: slot = position; a
sliding-window ring: the last `slots` positions at slot = position % slots).
Host logic only: the device write is replaced by a recorder."""
import pytest
import torch

from w4_weight_only_b200.api import KVCache


class _Recorder:
    def __init__(self, slots):
        self.n_slots, self.rows = slots, {}

    def slots(self, layer):
        return self.n_slots

    def write(self, layer, b, slot0, k, v):
        assert 0 <= slot0 and slot0 + k.shape[1] <= self.n_slots
        assert k.is_contiguous() and v.is_contiguous()
        for i in range(k.shape[1]):
            assert int(k[0, i, 0]) == int(v[0, i, 0])
            assert slot0 + i not in self.rows  # every slot written once
            self.rows[slot0 + i] = int(k[0, i, 0])


@pytest.mark.parametrize("n,slots", [(16384, 4096), (5000, 4096), (4096, 4096), (4097, 4096), (100, 4096),
                                     (9000, 64), (130, 64), (1, 64), (64, 64)])
def test_fill_history_slots(n, slots):
    rec = _Recorder(slots)
    pos = torch.arange(n, dtype=torch.int64).view(1, n, 1)
    KVCache.fill_history(rec, 0, 0, pos, pos.clone())
    held = range(max(0, n - slots), n)
    assert len(rec.rows) == len(held)
    for p in held:
        assert rec.rows[p % slots if n > slots else p] == p
