"""The fp16 range guard of the int4 GEMVs, and fp16 overflow reporting.

The GEMVs take their activations as fp16 (11-bit significand) after an exact
power-of-two scaling of every row whose max |x| reaches 2^15; the partial sums
are scaled back when they leave the warp.  Inputs of N(0, 1) never reach the
guard, so these cases drive it on purpose and compare with the oracle:

* a standalone GEMV with rows whose largest entry is 2^15, 2^20 (beyond the
  fp16 range: without the guard the staged value is infinite) and 3e4 (just
  below the guard), next to ordinary rows;
* a decode of the small decoder whose embedding is scaled by 2^20, so that the
  residual entering the QKV and gate/up GEMVs reaches ~8e4 (the gate/up
  weights are scaled by 2^-10 so that the SwiGLU output stays inside fp16).

The SwiGLU output h and the attention output are carried between phases in
fp16; a value beyond its range is reported as W4A_ERR_KERNEL, never passed on.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import fast
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import Pair, max_rel_to_rms, np64

pytestmark = pytest.mark.gpu

TOL = 2e-3        # GEMV: max error / RMS of the reference row
HID_TOL = 2e-2
LOGIT_TOL = 3e-2
EMBED_SCALE = 2.0 ** 20
GATE_UP_SCALE = 2.0 ** -10


def _api():
    from w4_weight_only_b200 import api, _abi
    return api, _abi


def _guard_rows(k: int, batch: int) -> torch.Tensor:
    """bf16 [batch, k]: row 0 holds one entry 2^15, row 1 is N(0, 1) * 2^18
    (max ~ 2^20), row 2 holds one entry 3e4 (below the guard), the others are
    N(0, 1)."""
    x = synth.normal((batch, k), "cpu", 1.0, 0.0, 40, "guard_x", k, batch)
    x[0, 7] = 2.0 ** 15
    x[1] *= 2.0 ** 18
    x[2, k - 3] = -3.0e4
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("n,k,batch", [(768, 512, 4), (1024, 1536, 5), (7168, 5120, 3), (5120, 27648, 4)])
def test_gemv_guard_rows(built_lib, cuda, n, k, batch):
    api, _ = _api()
    W = synth.normal((n, k), "cpu", 0.02, 0.0, 41, "guard_w", n, k)
    x = _guard_rows(k, batch)
    assert float(x[1].float().abs().max()) >= 2.0 ** 19
    lin = api.quantize_linear(W.to(cuda))
    ws = api.gemv_workspace(lin, batch)
    y = api.gemv(lin, x.to(cuda), ws=ws).cpu().numpy()
    api.check(ws)
    rows = np.arange(n) if n <= 1024 else np.concatenate([np.arange(32), np.arange(n - 32, n),
                                                          np.arange(100, n, 97)])
    ref = np64(x) @ fast.dense_matrix(W[rows]).T
    assert np.all(np.isfinite(y))
    for b in range(batch):  # the rows differ in scale by 2^18: compare each to its own RMS
        assert max_rel_to_rms(y[b, rows], ref[b]) <= TOL, b


@pytest.fixture(scope="module")
def big_pair(built_lib, cuda):
    return Pair(wc.tiny(), seed=0, gen_device="cpu", embed_scale=EMBED_SCALE,
                weight_scale={"gate_up": GATE_UP_SCALE})


def test_decode_guard_residual(big_pair):
    """Prefill 9 tokens, then one decode step; the residual (max ~8e4, past
    the fp16 range) enters the QKV and gate/up GEMVs of every layer."""
    from w4_weight_only_b200 import api
    P = big_pair
    cfg = P.cfg
    toks = synth.token_ids(7, 10, cfg.vocab, "cpu")
    kv = api.KVCache(cfg, 1, 32)
    okv = om.OracleKV(P.ocfg, 1, 32)
    P.gpu.prefill(kv, toks[:9].to("cuda"), want_logits=False)
    om.prefill(P.oracle, okv, toks[:9].numpy())
    dump = torch.zeros((cfg.n_layers + 1, 1, cfg.d_model), dtype=torch.float32, device="cuda")
    lg, _ = P.gpu.decode_step(kv, toks[9:].to("cuda"), torch.tensor([9], dtype=torch.int32, device="cuda"),
                              hidden_dump=dump)
    P.gpu.check()
    ref_lg, ref_hid = om.decode_step(P.oracle, okv, [int(toks[9])], [9])
    # the GEMV inputs are past the guard (and past fp16's 65504)
    assert float(np.abs(ref_hid[:cfg.n_layers, 0]).max()) >= 65536.0
    got = dump[:, 0].cpu().numpy()
    for l in range(cfg.n_layers + 1):
        assert max_rel_to_rms(got[l], ref_hid[l, 0]) <= HID_TOL, l
    assert float(np.max(np.abs(lg[0].cpu().numpy() - ref_lg[0]))) <= LOGIT_TOL


def test_decode_fp16_overflow_reported(built_lib, cuda):
    """The same embedding with ordinary gate/up weights: silu(gate) * up is
    ~1e9, beyond fp16, and the step reports W4A_ERR_KERNEL."""
    api, abi = _api()
    P = Pair(wc.tiny(), seed=0, gen_device="cpu", embed_scale=EMBED_SCALE)
    cfg = P.cfg
    kv = api.KVCache(cfg, 1, 32)
    P.gpu.decode_step(kv, torch.tensor([5], dtype=torch.int32, device="cuda"),
                      torch.tensor([0], dtype=torch.int32, device="cuda"))
    with pytest.raises(abi.W4AError) as e:
        P.gpu.check()
    assert e.value.code == abi.ERR_KERNEL
    assert "overflow" in str(e.value)
