"""The oracle's decoder against an independent library implementation (CPU).

The pages define the OLMo 3 32B layer in prose (post-norm residuals, RMSNorm
over the whole Q and K projections, GQA, RoPE with YaRN on the full-attention
layers, a final norm before the lm_head, a [SWA, SWA, SWA, full] stack) and
print no worked example of a whole layer.  The ``transformers`` package ships
its own OLMo 3 model (``Olmo3ForCausalLM``), written without reference to this
oracle, and its YaRN frequency routine.  Run in float64 on the oracle's
dequantized weights, it fixes the readings that the invariant tests leave
open:

* the YaRN ramp between the correction dimensions and the attention factor
  (ATLAS-OLMo-3-32B-Think-v4 model card, "Architecture deep-dive": YaRN x8 from
  8,192 positions, attention_factor ~1.208; archdb "Olmo-3-1125-32B": YaRN on
  the full-attention layers only);
* where RMSNorm adds its eps (inside the square root, next to the mean square);
* the final RMSNorm with gains between the last layer and the lm_head;
* the rotate-half pairing, the query-head -> KV-head map, the 1/sqrt(head_dim)
  scale, the sliding window counting the current token, the layer pattern
  (every fourth layer full, the library's own default) and the post-norm
  residual order.

The library computes its norms, rotary tables and softmax in float32 inside a
float64 model, so agreement is to ~1e-6 of the values' scale; the last test
plants the other readings in the oracle and checks that each one moves the
results far beyond the tolerance.
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import model

transformers = pytest.importorskip("transformers")
from transformers import Olmo3Config, Olmo3ForCausalLM  # noqa: E402
from transformers.models.olmo3.modeling_olmo3 import Olmo3RotaryEmbedding  # noqa: E402
from transformers.modeling_rope_utils import ROPE_INIT_FUNCTIONS  # noqa: E402

YARN = {"rope_type": "yarn", "rope_theta": 500000.0, "factor": 8.0,
        "original_max_position_embeddings": 8192, "beta_fast": 32.0, "beta_slow": 1.0}
PLAIN = {"rope_type": "default", "rope_theta": 500000.0}


def _hf_config(cfg: model.OracleConfig, rope: dict) -> Olmo3Config:
    c = Olmo3Config(vocab_size=cfg.vocab, hidden_size=cfg.d_model, intermediate_size=cfg.ffn,
                    num_hidden_layers=cfg.n_layers, num_attention_heads=cfg.n_heads,
                    num_key_value_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                    max_position_embeddings=65536, rms_norm_eps=cfg.eps, sliding_window=cfg.window,
                    tie_word_embeddings=False, attention_bias=False, rope_parameters=dict(rope))
    c._attn_implementation = "eager"
    return c


# ---------------------------------------------------------------------------
# the rotary tables and RMSNorm
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("head_dim", [64, 128])
def test_yarn_frequencies_and_factor_match_library(head_dim):
    cfg = replace(model.tiny_config(), head_dim=head_dim, d_model=8 * head_dim)
    inv, att = ROPE_INIT_FUNCTIONS["yarn"](_hf_config(cfg, YARN), "cpu")
    ours = model.yarn_inv_freq(head_dim, 5e5, 8.0, 8192, 32.0, 1.0)
    lib = inv.double().numpy()
    # the library forms the table in float32
    assert np.allclose(ours, lib, rtol=2e-6, atol=0), np.max(np.abs(ours / lib - 1))
    assert att == pytest.approx(model.yarn_attention_factor(8.0), abs=1e-15)
    plain, one = Olmo3RotaryEmbedding.compute_default_rope_parameters(_hf_config(cfg, PLAIN), "cpu")
    assert one == 1.0
    assert np.allclose(model.plain_inv_freq(head_dim, 5e5), plain.double().numpy(), rtol=2e-6, atol=0)


def test_rmsnorm_matches_library_where_eps_matters():
    """Mean squares from 1e-9 to 1e2 against torch's float64 rms_norm (eps
    1e-6): eps added to the mean square inside the square root."""
    r = np.random.default_rng(3)
    g = 1.0 + 0.1 * r.standard_normal(256)
    for scale in (10 ** -4.5, 1e-3, 1e-2, 1.0, 10.0):
        x = r.standard_normal((4, 256)) * scale
        lib = torch.nn.functional.rms_norm(torch.from_numpy(x), (256,), torch.from_numpy(g), eps=1e-6).numpy()
        assert np.allclose(model.rmsnorm(x, g, 1e-6), lib, rtol=1e-13, atol=0), scale


# ---------------------------------------------------------------------------
# the whole decoder
# ---------------------------------------------------------------------------
def _oracle_tiny(seed: int, cfg: model.OracleConfig) -> model.OracleModel:
    """The tiny decoder's shapes and value distributions (weights N(0, 0.02)
    quantized to int4 g128, gains 1 + N(0, 0.1), embedding and lm_head
    N(0, 0.02))."""
    r = np.random.default_rng(seed)
    d = cfg.d_model

    def w(n, k):
        return (0.02 * r.standard_normal((n, k))).astype(np.float32)

    layers = []
    for _ in range(cfg.n_layers):
        raw = {"qkv": w(cfg.qkv_dim, d), "o": w(d, cfg.q_dim), "gate_up": w(2 * cfg.ffn, d),
               "down": w(d, cfg.ffn),
               "q_norm": 1 + 0.1 * r.standard_normal(cfg.q_dim), "k_norm": 1 + 0.1 * r.standard_normal(cfg.kv_dim),
               "post_attn_norm": 1 + 0.1 * r.standard_normal(d), "post_ffn_norm": 1 + 0.1 * r.standard_normal(d)}
        layers.append(model.OracleLayer.from_float(raw, cfg.group))
    emb = 0.02 * r.standard_normal((cfg.vocab, d))
    head = 0.02 * r.standard_normal((cfg.vocab, d))
    return model.OracleModel(cfg, emb, head, 1 + 0.1 * r.standard_normal(d), layers)


def _library_model(om: model.OracleModel):
    """Olmo3ForCausalLM in float64 holding the oracle's dequantized weights;
    the full-attention layers take the YaRN table, the others plain RoPE."""
    cfg = om.cfg
    hf = Olmo3ForCausalLM(_hf_config(cfg, PLAIN)).to(torch.float64).eval()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))  # noqa: E731
    with torch.no_grad():
        hf.model.embed_tokens.weight.copy_(t(om.embed))
        hf.lm_head.weight.copy_(t(om.lm_head))
        hf.model.norm.weight.copy_(t(om.final_norm))
        q, kv = cfg.q_dim, cfg.kv_dim
        for l, layer in enumerate(hf.model.layers):
            L = om.layer(l)
            a = layer.self_attn
            a.q_proj.weight.copy_(t(L.Wqkv[:q]))
            a.k_proj.weight.copy_(t(L.Wqkv[q:q + kv]))
            a.v_proj.weight.copy_(t(L.Wqkv[q + kv:]))
            a.o_proj.weight.copy_(t(L.Wo))
            a.q_norm.weight.copy_(t(L.q_norm))
            a.k_norm.weight.copy_(t(L.k_norm))
            layer.mlp.gate_proj.weight.copy_(t(L.Wgu[:cfg.ffn]))
            layer.mlp.up_proj.weight.copy_(t(L.Wgu[cfg.ffn:]))
            layer.mlp.down_proj.weight.copy_(t(L.Wd))
            layer.post_attention_layernorm.weight.copy_(t(L.post_attn_norm))
            layer.post_feedforward_layernorm.weight.copy_(t(L.post_ffn_norm))
    yarn = Olmo3RotaryEmbedding(_hf_config(cfg, YARN)).to(torch.float64)

    def use_yarn(module, args, kwargs):
        kwargs["position_embeddings"] = yarn(args[0], kwargs["position_ids"])
        return args, kwargs

    outs = {}
    for l, layer in enumerate(hf.model.layers):
        if hf.config.layer_types[l] == "full_attention":
            layer.register_forward_pre_hook(use_yarn, with_kwargs=True)
        layer.register_forward_hook(lambda m, a, o, l=l: outs.__setitem__(l, o[0] if isinstance(o, tuple) else o))
    return hf, outs


def _rel(got, ref) -> float:
    ref = np.asarray(ref)
    return float(np.max(np.abs(np.asarray(got) - ref)) / np.sqrt(np.mean(ref * ref)))


TOL = 2e-5          # of the reference's RMS: float32 norms / rotary / softmax inside the library


def test_library_layer_pattern_is_the_oracles():
    cfg = model.tiny_config()
    types = _hf_config(cfg, PLAIN).layer_types
    assert [t == "full_attention" for t in types] == list(cfg.full_layers)
    types64 = _hf_config(replace(cfg, n_layers=64, full_layers=model.layer_pattern(64)), PLAIN).layer_types
    assert [t == "full_attention" for t in types64] == model.layer_pattern(64)


@pytest.fixture(scope="module")
def tiny_pair():
    cfg = model.tiny_config()
    om = _oracle_tiny(21, cfg)
    hf, outs = _library_model(om)
    return cfg, om, hf, outs


def test_prompt_matches_library_every_layer_and_cache(tiny_pair):
    """A 100-token prompt (the SWA layers' window of 64 slides past its start):
    every layer's residual, every rotated key and value, the last logits."""
    cfg, om, hf, outs = tiny_pair
    toks = np.random.default_rng(22).integers(0, cfg.vocab, 100)
    kv = model.OracleKV(cfg, 1, 128)
    logits, hidden = model.prefill_layers(om, kv, toks, keep_hidden=True)
    with torch.no_grad():
        res = hf(torch.from_numpy(toks).long()[None], use_cache=True)
    for l in range(cfg.n_layers):
        err = _rel(outs[l][0].numpy(), hidden[l + 1])
        assert err < TOL, (l, err)
        # the library's cache keeps every position of a full layer and the
        # last window - 1 of a sliding-window layer (all the next token needs)
        cache = res.past_key_values.layers[l]
        n = cache.keys.shape[2]
        assert n == (100 if cfg.full_layers[l] else cfg.window - 1), (l, n)
        assert _rel(cache.keys[0].numpy(), kv.K[l][0, :, 100 - n:100]) < TOL, l
        assert _rel(cache.values[0].numpy(), kv.V[l][0, :, 100 - n:100]) < TOL, l
    assert _rel(res.logits[0, -1].numpy(), logits) < TOL
    # the sequential definition gives the same last logits
    kv2 = model.OracleKV(cfg, 1, 128)
    assert np.allclose(model.prefill(om, kv2, toks), logits, rtol=1e-10, atol=1e-12)


def test_decode_step_matches_library(tiny_pair):
    """Prompt of 70 tokens, then three decode steps through the library's cache
    against oracle.decode_step_one at positions 70, 71, 72."""
    cfg, om, hf, outs = tiny_pair
    toks = np.random.default_rng(23).integers(0, cfg.vocab, 73)
    kv = model.OracleKV(cfg, 1, 128)
    model.prefill(om, kv, toks[:70])
    with torch.no_grad():
        res = hf(torch.from_numpy(toks[:70]).long()[None], use_cache=True)
        past = res.past_key_values
        for p in range(70, 73):
            lg, hid = model.decode_step_one(om, kv, int(toks[p]), 0, p)
            res = hf(torch.tensor([[int(toks[p])]]), past_key_values=past, use_cache=True,
                     position_ids=torch.tensor([[p]]))
            past = res.past_key_values
            assert _rel(res.logits[0, -1].numpy(), lg) < TOL, p
            for l in range(cfg.n_layers):
                assert _rel(outs[l][0, -1].numpy(), hid[l + 1]) < TOL, (p, l)


def test_planted_readings_are_caught(tiny_pair, monkeypatch):
    """Each alternative reading, planted in the oracle, leaves the library's
    results by far more than the tolerance: eps outside the square root, no
    final norm, a YaRN ramp shifted by one dimension, YaRN on every layer, a
    sliding window one key longer (measured: 1.2, 7.7, 0.024, 2.3 and 0.48 of
    the logits' RMS, against agreement to ~2e-6)."""
    cfg, om, hf, outs = tiny_pair
    toks = np.random.default_rng(24).integers(0, cfg.vocab, 90)
    with torch.no_grad():
        ref = hf(torch.from_numpy(toks).long()[None]).logits[0, -1].numpy()

    def last_logits(m=om):
        return model.prefill_layers(m, model.OracleKV(m.cfg, 1, 128), toks)[0]

    assert _rel(last_logits(), ref) < TOL
    errs = {}
    with monkeypatch.context() as mp:
        mp.setattr(model, "rmsnorm", lambda x, g, eps: np.asarray(x, np.float64) * np.asarray(g) /
                   (np.sqrt(np.mean(np.asarray(x, np.float64) ** 2, axis=-1, keepdims=True)) + eps))
        errs["eps outside the root"] = _rel(last_logits(), ref)
    nofinal = model.OracleModel(cfg, om.embed, om.lm_head, None, lambda l: om.layer(l))
    errs["no final norm"] = _rel(last_logits(nofinal), ref)
    with monkeypatch.context() as mp:
        rng = model.yarn_correction_range
        mp.setattr(model, "yarn_correction_range", lambda *a: tuple(v + 1 for v in rng(*a)))
        errs["ramp shifted"] = _rel(last_logits(), ref)
    with monkeypatch.context() as mp:
        lr = model.layer_rope
        mp.setattr(model, "layer_rope", lambda c, full: lr(c, True))
        errs["YaRN everywhere"] = _rel(last_logits(), ref)
    with monkeypatch.context() as mp:
        vis = model.visible_positions
        mp.setattr(model, "visible_positions", lambda pos, full, w: vis(pos, full, w + 1))
        errs["window one key longer"] = _rel(last_logits(), ref)
    for name, e in errs.items():
        assert e > 50 * TOL, (name, e)
