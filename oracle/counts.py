"""Oracle: KV-cache sizes, FLOP and parameter counts, streamed bytes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Sources:
* ATLAS-OLMo-3-32B-Think-v4 model card, "Why the 3:1 SWA layout matters for
  serving": f32 KV of all 64 layers costs 512 KiB per token (8 GB at 16K); an
  SWA-aware cache (16 full layers x ctx + 48 SWA layers x 4,096) needs about
  3.75 GB in f32 at 16K and about 5.1 GB in bf16 at 64K.
* Olmo 3 32B, "Modelled costs": KV per token 64 KiB (layers that grow with
  context, bf16); KV + state at 64K 4.75 GiB; decode 68.8 GFLOP per token at
  4K context; prefill 267 TFLOP for a 4K prompt; 32.2B parameters, 31.2B
  without embeddings and head.
* OLMo 3 (32B) summary card: KV cache 256 KiB per token in bf16 (all layers).
* archdb "Olmo-3-1125-32B": 487.6M parameters per layer, 31.21B backbone,
  1.027B embedding + head, 32.23B total; retained KV 9,395,240,960 bytes at
  131,072 tokens, 71,680 bytes per token averaged, 65,536 bytes global KV per
  token.

Counting conventions (stated, then pinned against the numbers above):
* A linear layer of n x k weights costs 2 n k FLOPs per token; attention costs
  4 * n_heads * head_dim FLOPs per visible key (q.k and p.v).
* The decode cost model counts every layer against the same number of keys.
* Prefill is causal: token t sees t + 1 keys on a full layer and
  min(t + 1, window) on an SWA layer; the lm_head runs for the last token only.

Parity status: pinned (every function reproduces a printed number).
"""
from __future__ import annotations

from .model import OracleConfig


def n_full_layers(cfg: OracleConfig) -> int:
    return sum(1 for f in cfg.full_layers if f)


def kv_bytes_per_token(cfg: OracleConfig, elem_bytes: int = 2, full_only: bool = False) -> int:
    """K and V of one token over the full layers only, or over all layers."""
    layers = n_full_layers(cfg) if full_only else cfg.n_layers
    return layers * 2 * cfg.kv_dim * elem_bytes


def kv_bytes_at_context(cfg: OracleConfig, ctx: int, elem_bytes: int = 2, swa_aware: bool = True) -> int:
    """Retained cache for one sequence of ``ctx`` tokens.

    SWA-aware: full layers keep ctx tokens, SWA layers keep min(ctx, window).
    Naive: every layer keeps ctx tokens.
    """
    per = 2 * cfg.kv_dim * elem_bytes
    total = 0
    for full in cfg.full_layers:
        keep = ctx if (full or not swa_aware) else min(ctx, cfg.window)
        total += keep * per
    return total


def linear_params_per_layer(cfg: OracleConfig) -> int:
    d = cfg.d_model
    return cfg.qkv_dim * d + d * cfg.q_dim + 2 * cfg.ffn * d + d * cfg.ffn


def norm_params_per_layer(cfg: OracleConfig) -> int:
    return cfg.q_dim + cfg.kv_dim + 2 * cfg.d_model


def params_per_layer(cfg: OracleConfig) -> int:
    return linear_params_per_layer(cfg) + norm_params_per_layer(cfg)


def embed_head_params(cfg: OracleConfig) -> int:
    return 2 * cfg.vocab * cfg.d_model


def backbone_params(cfg: OracleConfig) -> int:
    return cfg.n_layers * params_per_layer(cfg) + (cfg.d_model if cfg.final_norm else 0)


def total_params(cfg: OracleConfig) -> int:
    return backbone_params(cfg) + embed_head_params(cfg)


def decode_flops(cfg: OracleConfig, keys: int) -> int:
    """FLOPs of one decode token when every layer sees ``keys`` keys."""
    lin = 2 * (cfg.n_layers * linear_params_per_layer(cfg) + cfg.vocab * cfg.d_model)
    att = cfg.n_layers * 4 * cfg.n_heads * cfg.head_dim * keys
    return lin + att


def prefill_flops(cfg: OracleConfig, T: int) -> int:
    """FLOPs of a causal prefill of T tokens (lm_head on the last token)."""
    lin = 2 * T * cfg.n_layers * linear_params_per_layer(cfg) + 2 * cfg.vocab * cfg.d_model
    att = 0
    for full in cfg.full_layers:
        if full:
            keys = T * (T + 1) // 2
        else:
            W = cfg.window
            keys = sum(min(t + 1, W) for t in range(T)) if T > W else T * (T + 1) // 2
        att += 4 * cfg.n_heads * cfg.head_dim * keys
    return lin + att


def w4_bytes(n: int, k: int, group: int = 128) -> int:
    """Stored bytes of one int4 matrix: codes, fp16 scales, int4 zeros."""
    return n * k // 2 + (k // group) * n * 2 + (k // group) * n // 2


def decode_stream_bytes(cfg: OracleConfig, keys_per_layer) -> int:
    """HBM bytes one batch-1 decode token must read: every W4 matrix, the bf16
    lm_head, and K and V of the visible keys of each layer (bf16)."""
    d = cfg.d_model
    per_layer = (w4_bytes(cfg.qkv_dim, d, cfg.group) + w4_bytes(d, cfg.q_dim, cfg.group)
                 + w4_bytes(2 * cfg.ffn, d, cfg.group) + w4_bytes(d, cfg.ffn, cfg.group))
    kv = sum(2 * cfg.kv_dim * 2 * int(n) for n in keys_per_layer)
    return cfg.n_layers * per_layer + cfg.vocab * d * 2 + kv
