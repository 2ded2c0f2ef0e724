"""Pins for the oracle's KV-size, FLOP and parameter counters against the
numbers the pages print (tests/golden/pages_numbers.json, each with its page
and section)."""
import json
from pathlib import Path

import pytest

from oracle import counts, model

GOLD = json.loads((Path(__file__).parent / "golden" / "pages_numbers.json").read_text())
CFG = model.olmo3_32b_config()


def g(name):
    return GOLD[name]["value"]


def test_layer_mix():
    assert [CFG.n_layers - counts.n_full_layers(CFG), counts.n_full_layers(CFG)] == g("layers_swa_full")
    assert CFG.full_layers[-1] and CFG.window == g("sliding_window")


def test_kv_per_token():
    assert counts.kv_bytes_per_token(CFG, 2, full_only=True) == g("kv_bytes_per_token_full_layers_bf16")
    assert counts.kv_bytes_per_token(CFG, 2) == g("kv_bytes_per_token_all_layers_bf16")
    assert counts.kv_bytes_per_token(CFG, 4) == g("kv_bytes_per_token_all_layers_f32")


def test_kv_at_context():
    assert counts.kv_bytes_at_context(CFG, 65536, 2) == g("kv_bytes_64k_bf16_swa_aware")
    assert counts.kv_bytes_at_context(CFG, 65536, 2) / 2 ** 30 == pytest.approx(4.75, abs=1e-12)
    assert counts.kv_bytes_at_context(CFG, 131072, 2) == g("kv_bytes_131072_bf16")
    assert counts.kv_bytes_at_context(CFG, 131072, 2) // 131072 == g("kv_bytes_per_token_avg_131072")
    assert counts.kv_bytes_at_context(CFG, 16384, 4) == g("kv_bytes_16k_f32_swa_aware")
    assert counts.kv_bytes_at_context(CFG, 16384, 4, swa_aware=False) == g("kv_bytes_16k_f32_naive")


def test_decode_flops_4k():
    f = counts.decode_flops(CFG, 4096)
    assert f == 68_806_799_360
    assert abs(f / 1e9 - g("decode_gflop_4k")) <= GOLD["decode_gflop_4k"]["tolerance_rel"] * g("decode_gflop_4k")


def test_prefill_flops_4k():
    f = counts.prefill_flops(CFG, 4096)
    assert abs(f / 1e12 - g("prefill_tflop_4k")) <= GOLD["prefill_tflop_4k"]["tolerance_rel"] * g("prefill_tflop_4k")


def test_parameter_counts():
    assert counts.linear_params_per_layer(CFG) == 487_587_840
    assert counts.params_per_layer(CFG) == 487_604_224
    assert abs(counts.params_per_layer(CFG) / 1e6 - g("params_per_layer_millions")) <= 0.05
    assert abs(counts.backbone_params(CFG) / 1e9 - g("params_backbone_billions")) <= 0.005
    assert counts.embed_head_params(CFG) == 1_026_846_720
    assert abs(counts.embed_head_params(CFG) / 1e9 - g("params_embed_head_billions")) <= 0.0005
    assert abs(counts.total_params(CFG) / 1e9 - g("params_total_billions")) <= 0.005
    assert abs(CFG.vocab * CFG.d_model * 2 / 1e9 - g("lm_head_gb")) <= 0.05


def test_stream_bytes_4k():
    # every W4 matrix (codes + fp16 scales + int4 zeros), bf16 lm_head, K and V of 4,096 keys per layer
    b = counts.decode_stream_bytes(CFG, [4096] * CFG.n_layers)
    assert b == 16_212_295_680 + 1_026_846_720 + 64 * 4096 * 4096
