"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

Holds none of the method's arithmetic: it only draws random numbers, so that
the CUDA path and the oracle receive identical inputs.  Every tensor is drawn
from its own ``torch.Generator`` seeded from (seed, name, index...) through
SHA-256, so any single layer can be regenerated alone, on the CPU or on the GPU
(the two devices give different streams; a test uses one device for both
sides).

Recipes (the pages' shapes with random-init values; no checkpoint is used):
* linear weights  N(0, 0.02) fp32, quantized by the consumer;
* norm gains      1 + N(0, 0.1) fp32;
* embedding, lm_head N(0, 0.02) rounded to bf16;
* prompts         uniform token ids in [0, vocab);
* a pre-filled KV cache N(0, 1) bf16 (already-rotated keys);
* GEMV activations N(0, 1) bf16; raw attention projections N(0, 1) fp32;
* checkpoints in the model card's symmetric group-32 format: uniform random
  packed nibbles and bf16 scales 0.004 * |1 + 0.25 N(0, 1)| (+ 0.0002).
"""
from __future__ import annotations

import hashlib

import torch


def seed_of(*keys) -> int:
    h = hashlib.sha256(repr(keys).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *keys) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*keys))
    return g


def normal(shape, device, std: float, mean: float, *keys) -> torch.Tensor:
    t = torch.randn(shape, generator=_gen(device, *keys), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def layer_float(cfg, seed: int, l: int, device="cpu") -> dict:
    """fp32 weights of layer l: qkv [q+2kv, d] ([Q; K; V] rows), o [d, q],
    gate_up [2 ffn, d] ([gate; up] rows), down [d, ffn] and the four gains."""
    d, qd, kvd, f = cfg.d_model, cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.ffn
    return {
        "qkv": normal((qd + 2 * kvd, d), device, 0.02, 0.0, seed, "qkv", l),
        "o": normal((d, qd), device, 0.02, 0.0, seed, "o", l),
        "gate_up": normal((2 * f, d), device, 0.02, 0.0, seed, "gate_up", l),
        "down": normal((d, f), device, 0.02, 0.0, seed, "down", l),
        "q_norm": normal((qd,), device, 0.1, 1.0, seed, "q_norm", l),
        "k_norm": normal((kvd,), device, 0.1, 1.0, seed, "k_norm", l),
        "post_attn_norm": normal((d,), device, 0.1, 1.0, seed, "post_attn_norm", l),
        "post_ffn_norm": normal((d,), device, 0.1, 1.0, seed, "post_ffn_norm", l),
    }


def embed_head(cfg, seed: int, device="cpu"):
    """(embedding bf16 [V, d], lm_head bf16 [V, d], final norm gains fp32 [d])."""
    e = normal((cfg.vocab, cfg.d_model), device, 0.02, 0.0, seed, "embed").to(torch.bfloat16)
    h = normal((cfg.vocab, cfg.d_model), device, 0.02, 0.0, seed, "lm_head").to(torch.bfloat16)
    g = normal((cfg.d_model,), device, 0.1, 1.0, seed, "final_norm")
    return e, h, g


def token_ids(seed: int, n: int, vocab: int, device="cpu", *keys) -> torch.Tensor:
    return torch.randint(0, vocab, (n,), generator=_gen(device, seed, "tokens", *keys), device=device,
                         dtype=torch.int64).to(torch.int32)


def kv_rows(seed: int, l: int, b: int, n_kv: int, n: int, hd: int, device="cpu"):
    """(K, V) bf16 [n_kv, n, hd] N(0, 1): pre-filled cache rows of sequence b, layer l."""
    k = normal((n_kv, n, hd), device, 1.0, 0.0, seed, "kv_k", l, b).to(torch.bfloat16)
    v = normal((n_kv, n, hd), device, 1.0, 0.0, seed, "kv_v", l, b).to(torch.bfloat16)
    return k, v


def gemv_case(seed: int, n: int, k: int, batch: int, device="cpu"):
    """(W fp32 [n, k] N(0, 0.02), x bf16 [batch, k] N(0, 1))."""
    W = normal((n, k), device, 0.02, 0.0, seed, "gemv_w", n, k)
    x = normal((batch, k), device, 1.0, 0.0, seed, "gemv_x", n, k, batch).to(torch.bfloat16)
    return W, x


def weight_rows(seed: int, n: int, k: int, rows, device="cpu"):
    """Selected rows of the gemv_case weight (same values, drawn in full on
    ``device``; used when only a sample of rows is checked)."""
    return gemv_case(seed, n, k, 1, device)[0][rows]


def logits_rows(seed: int, batch: int, vocab: int, scale: float = 3.0, device="cpu") -> torch.Tensor:
    """fp32 [batch, vocab] N(0, scale^2): rows of logits for the sampler."""
    return normal((batch, vocab), device, scale, 0.0, seed, "logits")


def uniforms(seed: int, n: int, device="cpu") -> torch.Tensor:
    """fp32 [n] uniform in [0, 1): the draws of the sampler."""
    g = _gen(device, seed, "uniform")
    return torch.rand((n,), generator=g, device=device, dtype=torch.float32)


def sym32_matrix(seed: int, n: int, k: int, device="cpu", *keys):
    """A checkpoint matrix in the symmetric group-32 format: (qweight int32
    [n, k/8] of uniform random bits, i.e. eight uniform 4-bit nibbles per
    word; scales bf16 [n, k/32] drawn as 0.004 * (1 + 0.25 N(0, 1)), kept
    positive)."""
    g = _gen(device, seed, "sym32_q", n, k, *keys)
    qw = torch.randint(-(2 ** 31), 2 ** 31, (n, k // 8), generator=g, device=device, dtype=torch.int64)
    s = normal((n, k // 32), device, 0.25, 1.0, seed, "sym32_s", n, k, *keys).abs_().add_(0.05).mul_(0.004)
    return qw.to(torch.int32), s.to(torch.bfloat16)


def g128_storage(seed: int, n: int, k: int, *keys):
    """Storage of an int4 group-128 matrix with random contents, for timing
    only: (qweight int32 [n, k/8] and qzeros int32 [k/128, n/8] of uniform
    random bits, scales as fp16 bits [k/128, n] of 0.003 * (1 + 0.25 N(0, 1)),
    kept positive), the size and layout of a quantized N(0, 0.02) matrix."""
    g = _gen("cpu", seed, "g128_q", n, k, *keys)
    qw = torch.randint(-(2 ** 31), 2 ** 31, (n, k // 8), generator=g, dtype=torch.int64).to(torch.int32)
    qz = torch.randint(-(2 ** 31), 2 ** 31, (k // 128, n // 8), generator=g, dtype=torch.int64).to(torch.int32)
    s = normal((k // 128, n), "cpu", 0.25, 1.0, seed, "g128_s", n, k, *keys).abs_().add_(0.05).mul_(0.003)
    return qw, s.to(torch.float16).view(torch.int16), qz


def sym32_layer(cfg, seed: int, l: int, device="cpu") -> dict:
    """Layer l in the symmetric group-32 format: checkpoint pairs for qkv
    [q+2kv, d] ([Q; K; V]), o, gate_up [2 ffn, d] ([gate; up]) and down,
    and the four gains (1 + N(0, 0.1))."""
    d, qd, kvd, f = cfg.d_model, cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.ffn
    return {
        "qkv": sym32_matrix(seed, qd + 2 * kvd, d, device, "qkv", l),
        "o": sym32_matrix(seed, d, qd, device, "o", l),
        "gate_up": sym32_matrix(seed, 2 * f, d, device, "gate_up", l),
        "down": sym32_matrix(seed, d, f, device, "down", l),
        "q_norm": normal((qd,), device, 0.1, 1.0, seed, "q_norm", l),
        "k_norm": normal((kvd,), device, 0.1, 1.0, seed, "k_norm", l),
        "post_attn_norm": normal((d,), device, 0.1, 1.0, seed, "post_attn_norm", l),
        "post_ffn_norm": normal((d,), device, 0.1, 1.0, seed, "post_ffn_norm", l),
    }
