"""The benchmark's model against the oracle: all 64 layers of the
OLMo-3-32B-shaped int4 decoder (seed 3), KV cache pre-filled to 4,096
positions, one decode step at position 4,096 in the benchmark's launch
configuration (ATLAS-OLMo-3-32B-Think-v4 model card, "Architecture
deep-dive": the [SWA, SWA, SWA, full] x 16 stack).

Two checks per layer, both within 2e-2 * RMS of the oracle's residual:

* chained: the GPU's residual after layer l (the step's hidden dump) against
  the oracle's, both having run layers 0 .. l themselves, so the error of a
  layer includes the drift the earlier layers passed on;
* isolated: the oracle's input to layer l (rounded to bf16, the embedding
  format) fed to a one-layer GPU model made of the same device weights, so
  that no drift is charged to the layer.

Then all 100,278 logits within 3e-2 and the greedy token when the oracle's
top-2 gap exceeds 2 x 3e-2.  The oracle quantizes and dequantizes each layer
itself (``oracle.fast``, pinned to ``oracle.quant``) one layer at a time.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fast
from oracle import model as om
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import max_rel_to_rms, oracle_config

pytestmark = pytest.mark.gpu

SEED = 3          # the benchmark's model
CTX = 4096
TOKEN = 1         # the benchmark's first token
HID_TOL = 2e-2
LOGIT_TOL = 3e-2


def _one_layer_cfg(full: bool, vocab: int) -> wc.Config:
    c = wc.olmo3_32b(1)
    c.full_layers = [full]
    c.vocab = vocab
    return c


def _fill(kv, layer, k, v):
    kv.fill_history(layer, 0, k, v)


def test_decode_64_layers_against_oracle(built_lib, cuda):
    from w4_weight_only_b200 import api
    cfg = wc.olmo3_32b(64)
    emb, head, fin = synth.embed_head(cfg, SEED, "cuda")
    model = api.Model.from_float(cfg, emb, head, fin, lambda l: synth.layer_float(cfg, SEED, l, "cuda"))
    cap = CTX + 16
    kv = api.KVCache(cfg, 1, cap)
    for l in range(cfg.n_layers):
        k, v = synth.kv_rows(SEED, l, 0, cfg.n_kv_heads, CTX, cfg.head_dim, "cuda")
        _fill(kv, l, k, v)
    dump = torch.zeros((cfg.n_layers + 1, 1, cfg.d_model), dtype=torch.float32, device="cuda")
    logits, nxt = model.decode_step(kv, torch.tensor([TOKEN], dtype=torch.int32, device="cuda"),
                                    torch.tensor([CTX], dtype=torch.int32, device="cuda"), hidden_dump=dump)
    model.check()
    got = dump[:, 0].cpu().numpy().astype(np.float64)
    logits = logits[0].cpu().numpy().astype(np.float64)
    nxt = int(nxt[0])

    # one-layer GPU models over the same device weights, for the isolated check
    small_vocab = 16
    small_head = api.tile_bf16(torch.zeros((small_vocab, cfg.d_model), dtype=torch.bfloat16, device="cuda"))
    ones = torch.ones(cfg.d_model, dtype=torch.float32, device="cuda")

    x = emb[TOKEN].to("cpu").double().numpy()
    assert max_rel_to_rms(got[0], x) == 0.0          # the embedding row itself
    worst_chain, worst_iso = (0.0, -1), (0.0, -1)
    for l in range(cfg.n_layers):
        full = bool(cfg.full_layers[l])
        c1 = _one_layer_cfg(full, small_vocab)
        oc1 = oracle_config(c1)
        raw = {n: t.cpu() for n, t in synth.layer_float(cfg, SEED, l, "cuda").items()}
        L = fast.dense_layer(raw)
        del raw
        k, v = synth.kv_rows(SEED, l, 0, cfg.n_kv_heads, CTX, cfg.head_dim, "cuda")
        kk, vv = k.cpu().double().numpy(), v.cpu().double().numpy()
        okv = om.OracleKV(oc1, 1, cap)
        okv.fill(0, 0, 0, kk, vv)
        # isolated: the oracle's input to this layer as bf16
        x16 = torch.from_numpy(x).to(torch.bfloat16)
        okv_i = om.OracleKV(oc1, 1, cap)
        okv_i.fill(0, 0, 0, kk, vv)
        ref_iso = om.layer_forward(oc1, L, 0, x16.double().numpy(), okv_i, 0, CTX)
        table = torch.zeros((small_vocab, cfg.d_model), dtype=torch.bfloat16, device="cuda")
        table[0] = x16.to("cuda")
        m1 = api.Model(c1, table, small_head, ones, [model.layers[l]])
        kv1 = api.KVCache(c1, 1, cap)
        _fill(kv1, 0, k, v)
        d1 = torch.zeros((2, 1, cfg.d_model), dtype=torch.float32, device="cuda")
        m1.decode_step(kv1, torch.tensor([0], dtype=torch.int32, device="cuda"),
                       torch.tensor([CTX], dtype=torch.int32, device="cuda"), hidden_dump=d1)
        m1.check()
        e_iso = max_rel_to_rms(d1[1, 0].cpu().numpy(), ref_iso)
        del m1, kv1, k, v
        # chained
        x = om.layer_forward(oc1, L, 0, x, okv, 0, CTX)
        e_chain = max_rel_to_rms(got[l + 1], x)
        del L, okv, okv_i
        worst_chain = max(worst_chain, (e_chain, l))
        worst_iso = max(worst_iso, (e_iso, l))
        assert e_iso <= HID_TOL, ("isolated", l, e_iso)
        assert e_chain <= HID_TOL, ("chained", l, e_chain)
    print(f"\n64-layer decode: worst chained residual error {worst_chain[0]:.3e} RMS (layer {worst_chain[1]}), "
          f"worst isolated {worst_iso[0]:.3e} RMS (layer {worst_iso[1]})")

    # final norm + lm_head (the oracle's head, over row blocks of the bf16 matrix)
    xn = om.rmsnorm(x, fin.cpu().double().numpy(), cfg.eps)
    ref = np.empty(cfg.vocab)
    hc = head.cpu()
    for r0 in range(0, cfg.vocab, 8192):
        ref[r0:r0 + 8192] = hc[r0:r0 + 8192].double().numpy() @ xn
    err = float(np.max(np.abs(logits - ref)))
    print(f"64-layer decode: max logit error {err:.3e}")
    assert err <= LOGIT_TOL
    top2 = np.sort(ref)[-2:]
    if top2[1] - top2[0] >= 2 * LOGIT_TOL:
        assert nxt == int(np.argmax(ref))
