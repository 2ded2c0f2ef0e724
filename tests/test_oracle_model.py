"""Pins for the oracle's decoder definition (CPU only).

Invariants and closed forms from the pages (RMSNorm, softmax, rotation norms
and relative-position dependence, YaRN's band structure, the attention factor
1.208, SWA == full attention inside the window, GQA reducing to MHA), plus a
loop-by-loop restatement of a whole layer on tiny shapes.
"""
import json
import math
from dataclasses import replace
from pathlib import Path

import numpy as np
import pytest

from oracle import brute, model, quant

GOLD = json.loads((Path(__file__).parent / "golden" / "pages_numbers.json").read_text())


def test_rmsnorm_unit_gain_has_unit_rms():
    x = np.random.default_rng(0).standard_normal((3, 512)) * 7.0
    y = model.rmsnorm(x, np.ones(512), 1e-6)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-6)


def test_softmax_rows_sum_to_one():
    s = np.random.default_rng(1).standard_normal((5, 777)) * 30
    p = model.softmax(s)
    assert np.all(np.abs(p.sum(-1) - 1.0) < 1e-12) and np.all(p >= 0)


def test_attention_factor_closed_form():
    m = model.yarn_attention_factor(8.0)
    assert m == pytest.approx(0.1 * math.log(8.0) + 1.0, abs=0)
    assert abs(m - GOLD["attention_factor"]["value"]) <= GOLD["attention_factor"]["tolerance_abs"]


def test_yarn_correction_range_values():
    # d = 128, theta 5e5, L0 8192: dims 18 .. 35; d = 64: 9 .. 18
    assert model.yarn_correction_range(128, 5e5, 8192, 32, 1) == (18, 35)
    assert model.yarn_correction_range(64, 5e5, 8192, 32, 1) == (9, 18)


def test_yarn_band_structure():
    f = model.plain_inv_freq(128, 5e5)
    fy = model.yarn_inv_freq(128, 5e5, 8.0, 8192, 32, 1)
    lo, hi = 18, 35
    assert np.array_equal(fy[:lo + 1], f[:lo + 1])           # high-frequency dims unchanged
    assert np.allclose(fy[hi:], f[hi:] / 8.0, rtol=1e-15)    # low-frequency dims interpolated by 8
    mid = fy[lo + 1:hi]
    assert np.all(mid < f[lo + 1:hi]) and np.all(mid > f[lo + 1:hi] / 8.0)
    # factor 1 reduces YaRN to plain RoPE
    assert np.allclose(model.yarn_inv_freq(128, 5e5, 1.0, 8192, 32, 1), f, rtol=0)
    assert model.yarn_attention_factor(1.0) == 1.0


def test_rope_preserves_norms_and_is_relative():
    r = np.random.default_rng(2)
    q = r.standard_normal((3, 128))
    k = r.standard_normal((3, 128))
    f = model.yarn_inv_freq(128, 5e5, 8.0, 8192, 32, 1)
    m = 1.2
    for pos in (0, 1, 4095, 65535):
        rq = model.rope(q, pos, f, m)
        assert np.allclose(np.linalg.norm(rq, axis=-1), m * np.linalg.norm(q, axis=-1), rtol=1e-12)
    a = np.sum(model.rope(q, 700, f) * model.rope(k, 300, f), axis=-1)
    b = np.sum(model.rope(q, 1400, f) * model.rope(k, 1000, f), axis=-1)
    assert np.allclose(a, b, rtol=1e-9, atol=1e-9)
    assert np.allclose(model.rope(q, 0, f), q)
    # pairing: dimension i rotates with i + 64
    e = np.zeros(128)
    e[5] = 1.0
    out = model.rope(e, 3, f)
    assert np.count_nonzero(np.abs(out) > 1e-15) == 2 and abs(out[69]) > 0


def _textbook_mha(q, K, V):
    """Per-head softmax(q k^T / sqrt(d)) V written out head by head."""
    hq, d = q.shape
    out = np.zeros_like(q)
    for h in range(hq):
        s = np.array([np.dot(q[h], K[h, j]) for j in range(K.shape[1])]) / math.sqrt(d)
        p = np.exp(s - s.max())
        p /= p.sum()
        out[h] = sum(p[j] * V[h, j] for j in range(K.shape[1]))
    return out


def test_gqa_with_equal_heads_is_mha():
    r = np.random.default_rng(3)
    cfg = replace(model.tiny_config(), n_heads=4, n_kv_heads=4, head_dim=16, window=1000)
    q = r.standard_normal((4, 16))
    K = r.standard_normal((4, 9, 16))
    V = r.standard_normal((4, 9, 16))
    o = model.gqa_decode(cfg, q, K, V, pos=8, full=True)
    assert np.allclose(o, _textbook_mha(q, K, V), rtol=1e-12, atol=1e-12)


def test_gqa_group_mapping():
    """Query head h reads KV head h // (heads / kv_heads)."""
    r = np.random.default_rng(4)
    cfg = replace(model.tiny_config(), n_heads=6, n_kv_heads=2, head_dim=8, window=1000)
    q = r.standard_normal((6, 8))
    K = r.standard_normal((2, 5, 8))
    V = r.standard_normal((2, 5, 8))
    o = model.gqa_decode(cfg, q, K, V, pos=4, full=True)
    Kx = K[[0, 0, 0, 1, 1, 1]]
    Vx = V[[0, 0, 0, 1, 1, 1]]
    assert np.allclose(o, _textbook_mha(q, Kx, Vx), rtol=1e-12, atol=1e-12)


def test_visible_positions_window():
    assert list(model.visible_positions(3, False, 4)) == [0, 1, 2, 3]
    assert list(model.visible_positions(4, False, 4)) == [1, 2, 3, 4]       # window counts the token
    assert list(model.visible_positions(9, True, 4)) == list(range(10))


# ---------------------------------------------------------------------------
# small random models
# ---------------------------------------------------------------------------
def micro_config(**kw):
    base = dict(d_model=32, n_layers=4, n_heads=4, n_kv_heads=2, head_dim=8, ffn=64, vocab=50, window=4,
                full_layers=model.layer_pattern(4), group=32)
    base.update(kw)
    return model.OracleConfig(**base)


def micro_model(cfg, seed=0):
    r = np.random.default_rng(seed)
    d = cfg.d_model
    layers = []
    for _ in range(cfg.n_layers):
        raw = {"qkv": r.standard_normal((cfg.qkv_dim, d)) * 0.2, "o": r.standard_normal((d, cfg.q_dim)) * 0.2,
               "gate_up": r.standard_normal((2 * cfg.ffn, d)) * 0.2, "down": r.standard_normal((d, cfg.ffn)) * 0.2,
               "q_norm": 1 + 0.1 * r.standard_normal(cfg.q_dim), "k_norm": 1 + 0.1 * r.standard_normal(cfg.kv_dim),
               "post_attn_norm": 1 + 0.1 * r.standard_normal(d), "post_ffn_norm": 1 + 0.1 * r.standard_normal(d)}
        layers.append(model.OracleLayer.from_float(raw, cfg.group))
    emb = r.standard_normal((cfg.vocab, d)) * 0.5
    head = r.standard_normal((cfg.vocab, d)) * 0.5
    return model.OracleModel(cfg, emb, head, 1 + 0.1 * r.standard_normal(d), layers)


@pytest.mark.parametrize("full", [False, True])
def test_layer_matches_loop_by_loop_restatement(full):
    cfg = micro_config(full_layers=[full] * 4)
    m = micro_model(cfg, seed=11)
    L = m.layer(0)
    r = np.random.default_rng(12)
    kv = model.OracleKV(cfg, 1, 16)
    Kh, Vh = {}, {}
    x = r.standard_normal(cfg.d_model)
    for pos in range(9):     # beyond the window of 4 on the SWA variant
        xv = model.layer_forward(cfg, L, 0, x, kv, 0, pos)
        xb = brute.layer(cfg, L.Wqkv.tolist(), L.Wo.tolist(), L.Wgu.tolist(), L.Wd.tolist(), L.q_norm, L.k_norm,
                         L.post_attn_norm, L.post_ffn_norm, list(x), Kh, Vh, pos, full)
        assert np.allclose(xv, xb, rtol=1e-11, atol=1e-11), pos
        x = xv + 0.1 * r.standard_normal(cfg.d_model)


def test_swa_equals_full_inside_window():
    """With no YaRN, a sliding-window layer and a full layer agree while the
    context fits the window, and differ once it does not."""
    cfg_swa = micro_config(window=6, yarn_factor=1.0, full_layers=[False] * 4)
    cfg_full = replace(cfg_swa, full_layers=[True] * 4)
    toks = [3, 17, 42, 5, 9, 11, 30, 2]
    outs = {}
    for name, cfg in (("swa", cfg_swa), ("full", cfg_full)):
        m = micro_model(cfg, seed=5)
        kv = model.OracleKV(cfg, 1, 16)
        outs[name] = [model.decode_step_one(m, kv, t, 0, p)[0] for p, t in enumerate(toks)]
    for p in range(6):
        assert np.allclose(outs["swa"][p], outs["full"][p], rtol=1e-12, atol=1e-12)
    assert not np.allclose(outs["swa"][7], outs["full"][7])


def test_batched_decode_equals_single_and_prefill_is_sequential():
    cfg = micro_config()
    m = micro_model(cfg, seed=7)
    toks = [[1, 2, 3, 4, 5, 6], [7, 8, 9, 10, 11, 12]]
    kv1 = model.OracleKV(cfg, 2, 8)
    kv2 = model.OracleKV(cfg, 2, 8)
    for p in range(6):
        lg, hid = model.decode_step(m, kv1, [toks[0][p], toks[1][p]], [p, p])
        for b in range(2):
            l1, h1 = model.decode_step_one(m, kv2, toks[b][p], b, p)
            assert np.allclose(lg[b], l1, rtol=1e-13, atol=1e-13)
            assert np.allclose(hid[:, b], h1, rtol=1e-13, atol=1e-13)
    kv3 = model.OracleKV(cfg, 2, 8)
    last = model.prefill(m, kv3, toks[1], b=1)
    assert np.allclose(last, lg[1], rtol=1e-13, atol=1e-13)


def test_argmax_ties_to_lowest_index():
    assert model.argmax(np.array([[1.0, 3.0, 3.0, 2.0]]))[0] == 1


@pytest.mark.parametrize("start", [0, 5])
def test_layer_at_a_time_prefill_equals_sequential(start):
    """prefill_layers (all tokens' projections as one matrix product per
    layer, then attention per position) gives what sequential decode gives:
    the last logits, every K/V it wrote, and the residual after each layer of
    every token; the window of 4 wraps within the 11 tokens, and start > 0
    continues from a pre-filled history."""
    cfg = micro_config()
    m = micro_model(cfg, seed=21)
    r = np.random.default_rng(22)
    toks = list(r.integers(0, cfg.vocab, size=11))
    cap = start + len(toks) + 1
    kv_a = model.OracleKV(cfg, 2, cap)
    kv_b = model.OracleKV(cfg, 2, cap)
    for l in range(cfg.n_layers):
        hk = r.standard_normal((cfg.n_kv_heads, start, cfg.head_dim))
        hv = r.standard_normal((cfg.n_kv_heads, start, cfg.head_dim))
        kv_a.fill(l, 1, 0, hk, hv)
        kv_b.fill(l, 1, 0, hk, hv)
    seq_hidden = []
    for i, t in enumerate(toks):
        lg_seq, h = model.decode_step_one(m, kv_a, int(t), 1, start + i)
        seq_hidden.append(h)
    lg_lay, hid = model.prefill_layers(m, kv_b, toks, b=1, start_pos=start, keep_hidden=True)
    assert np.allclose(lg_lay, lg_seq, rtol=1e-12, atol=1e-12)
    assert np.allclose(hid, np.stack(seq_hidden, axis=1), rtol=1e-12, atol=1e-12)
    for l in range(cfg.n_layers):
        assert np.allclose(kv_a.K[l], kv_b.K[l], rtol=1e-12, atol=1e-12)
        assert np.allclose(kv_a.V[l], kv_b.V[l], rtol=1e-12, atol=1e-12)
    # early stop: the first two layers' residuals only
    kv_c = model.OracleKV(cfg, 2, cap)
    for l in range(cfg.n_layers):
        kv_c.K[l][:], kv_c.V[l][:] = kv_b.K[l], kv_b.V[l]
    none, hid2 = model.prefill_layers(m, kv_c, toks, b=1, start_pos=start, n_layers=2, keep_hidden=True)
    assert none is None and np.allclose(hid2, hid[:3], rtol=1e-12, atol=1e-12)
