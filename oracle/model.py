"""Oracle: float64 definition of the OLMo-3-32B-shaped decoder step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What it computes, and where each step comes from:

* Layer stack: 64 layers in a repeating [SWA, SWA, SWA, full] pattern, the last
  layer full; sliding window 4,096 (ATLAS-OLMo-3-32B-Think-v4 model card,
  "Architecture deep-dive"; Olmo 3 32B, "Every architecture field", layout;
  archdb "Olmo-3-1125-32B", "3 SWA : 1 global (last layer global)").
* Attention: GQA, 40 query heads over 8 KV heads, head_dim 128 (model card
  "Architecture deep-dive"; LLM Architecture KB "OLMo 3 32B", item 2).  Query
  head h reads KV head h // (heads / kv_heads) (reading D11).  Scores are scaled
  by 1/sqrt(head_dim) (D12).
* QK-norm: RMSNorm over the whole Q projection and over the whole K projection,
  not per head (model card, "What ATLAS implements for the W4 path":
  "full-projection QK-norm"; D17).
* RoPE theta 500,000 on every layer; YaRN x8 (8,192 -> 65,536) only on the
  full-attention layers with attention_factor ~ 1.208 (model card
  "Architecture deep-dive"; LLM Architecture KB "Techniques used", item 4;
  archdb context-extension field: "YaRN on full-attention layers only").
  Rotation pairs dimension i with i + head_dim/2 (D5); YaRN follows the
  published method of Peng et al. with beta_fast = 32, beta_slow = 1 (D6); the
  attention factor 0.1 ln(8) + 1 multiplies both cos and sin, so it scales the
  rotated q and the rotated k (D7).
* Post-norm residuals: x <- x + RMSNorm(attn(x)), x <- x + RMSNorm(ffn(x)), no
  pre-norm (Olmo 3 32B, "Norm placement: post"; LLM Architecture KB
  "Techniques used", item 1).  RMSNorm eps 1e-6 (archdb field list).
* FFN: SwiGLU, down(silu(gate x) * up x), d_ff 27,648 (model card; archdb).
  No biases anywhere (archdb field list).
* Head: RMSNorm with gains (reading D9), then an untied bf16 lm_head over the
  vocabulary (model card "Performance & footprint": "BF16 lm_head"); greedy
  argmax, ties to the lowest index (D15).
* Fused row order: QKV rows [Q; K; V], gate/up rows [gate; up] (D13).

All arithmetic is float64 on the exactly dequantized weights; the inputs that
are bf16 by definition (embedding, lm_head, a pre-filled KV cache) enter as the
float64 values of those bf16 numbers.

Parity status: rmsnorm, rope (plain and YaRN), softmax, GQA attention, the
sliding window and one full layer are pinned by tests (invariants, closed
forms, a loop-by-loop implementation in ``brute``).  The pages print no worked
example of a layer, so the conventions they give only in prose (the rotation
pairing, the YaRN ramp and attention factor, eps inside the square root, the
final norm, a window that counts the current token, the layer pattern) are
pinned against an independent implementation: the ``transformers`` package's
OLMo 3 model in float64 on the same weights agrees on every layer's residual,
the cache and the logits to ~3e-6 of their RMS, and each alternative reading
planted here moves the logits by 2e-2 to 8 of their RMS.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence

import numpy as np

from . import quant


# --------------------------------------------------------------------------
# configuration
# --------------------------------------------------------------------------
@dataclass
class OracleConfig:
    d_model: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    window: int
    full_layers: Sequence[bool]
    rope_theta: float = 500000.0
    yarn_factor: float = 8.0
    yarn_orig_ctx: int = 8192
    beta_fast: float = 32.0
    beta_slow: float = 1.0
    eps: float = 1e-6
    group: int = 128
    final_norm: bool = True

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_dim(self) -> int:
        return self.q_dim + 2 * self.kv_dim


def layer_pattern(n_layers: int) -> List[bool]:
    """[SWA, SWA, SWA, full] repeated: layer l is full iff l % 4 == 3."""
    return [(l % 4) == 3 for l in range(n_layers)]


def olmo3_32b_config(n_layers: int = 64) -> OracleConfig:
    return OracleConfig(d_model=5120, n_layers=n_layers, n_heads=40, n_kv_heads=8,
                        head_dim=128, ffn=27648, vocab=100278, window=4096,
                        full_layers=layer_pattern(n_layers))


def tiny_config() -> OracleConfig:
    return OracleConfig(d_model=512, n_layers=4, n_heads=8, n_kv_heads=2, head_dim=64,
                        ffn=1536, vocab=4096, window=64, full_layers=layer_pattern(4))


# --------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------
def rmsnorm(x, gain, eps: float):
    """x / sqrt(mean(x^2) + eps) * gain over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(gain, dtype=np.float64)


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def softmax(s):
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - np.max(s, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def plain_inv_freq(head_dim: int, theta: float):
    """f_i = theta^(-2i/head_dim), i = 0 .. head_dim/2 - 1."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / head_dim)


def yarn_correction_range(head_dim: int, theta: float, orig_ctx: int,
                          beta_fast: float, beta_slow: float):
    """Dimension index range [lo, hi] over which YaRN blends the frequencies.

    For b rotations over the original context L0, the dimension index is
    d * ln(L0 / (2 pi b)) / (2 ln theta); lo uses beta_fast (floored), hi uses
    beta_slow (ceiled), clamped to [0, head_dim - 1].
    """
    def dim_for(b):
        return head_dim * math.log(orig_ctx / (b * 2.0 * math.pi)) / (2.0 * math.log(theta))
    lo = max(math.floor(dim_for(beta_fast)), 0)
    hi = min(math.ceil(dim_for(beta_slow)), head_dim - 1)
    return lo, hi


def yarn_inv_freq(head_dim: int, theta: float, factor: float, orig_ctx: int,
                  beta_fast: float, beta_slow: float):
    """YaRN frequencies: f'_i = (f_i / factor) * r_i + f_i * (1 - r_i),
    r_i = clamp((i - lo) / (hi - lo), 0, 1)."""
    f = plain_inv_freq(head_dim, theta)
    lo, hi = yarn_correction_range(head_dim, theta, orig_ctx, beta_fast, beta_slow)
    span = (hi - lo) if hi != lo else 0.001
    i = np.arange(head_dim // 2, dtype=np.float64)
    r = np.clip((i - lo) / span, 0.0, 1.0)
    return (f / factor) * r + f * (1.0 - r)


def yarn_attention_factor(factor: float) -> float:
    """0.1 * ln(factor) + 1 (1.0 when factor <= 1)."""
    return 1.0 if factor <= 1.0 else 0.1 * math.log(factor) + 1.0


def layer_rope(cfg: OracleConfig, full: bool):
    """(inv_freq [head_dim/2], mscale) for a full (YaRN) or SWA (plain) layer."""
    if full:
        return (yarn_inv_freq(cfg.head_dim, cfg.rope_theta, cfg.yarn_factor, cfg.yarn_orig_ctx,
                              cfg.beta_fast, cfg.beta_slow),
                yarn_attention_factor(cfg.yarn_factor))
    return plain_inv_freq(cfg.head_dim, cfg.rope_theta), 1.0


def rope(x, pos: int, inv_freq, mscale: float = 1.0):
    """Rotate every head of x [..., head_dim] at position pos.

    Pair (i, i + head_dim/2) rotates by pos * f_i; cos and sin carry mscale.
    """
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    ang = float(pos) * np.asarray(inv_freq, dtype=np.float64)
    c = np.cos(ang) * mscale
    s = np.sin(ang) * mscale
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attend(q, K, V, scale: float):
    """Decode attention for one KV group.

    q [hq, hd] (the query heads sharing this KV head), K, V [n, hd] (the keys
    and values the token may see).  Returns o [hq, hd] =
    softmax(q K^T * scale) V.
    """
    s = (np.asarray(q, np.float64) @ np.asarray(K, np.float64).T) * scale
    return softmax(s) @ np.asarray(V, np.float64)


def visible_positions(pos: int, full: bool, window: int):
    """Positions a token at ``pos`` attends to: [0, pos] on a full layer,
    (pos - window, pos] on a sliding-window layer (the window counts the token
    itself, reading D10)."""
    lo = 0 if full else max(0, pos - window + 1)
    return np.arange(lo, pos + 1)


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------
class W4Matrix:
    """One quantized linear layer in canonical storage."""

    def __init__(self, qweight, scales_bits, qzeros, n: int, k: int, group: int = 128):
        self.qweight, self.scales_bits, self.qzeros = qweight, scales_bits, qzeros
        self.n, self.k, self.group = n, k, group

    @classmethod
    def from_float(cls, W, group: int = 128):
        W = np.asarray(W, dtype=np.float32)
        qw, sb, qz = quant.quantize_pack(W, group)
        return cls(qw, sb, qz, W.shape[0], W.shape[1], group)

    def dequantized(self):
        return quant.dequantize(self.qweight, self.scales_bits, self.qzeros,
                                self.n, self.k, self.group)

    def matvec(self, x):
        """W~ x for x [..., k] (float64)."""
        return np.asarray(x, np.float64) @ self.dequantized().T


@dataclass
class OracleLayer:
    qkv: W4Matrix
    o: W4Matrix
    gate_up: W4Matrix
    down: W4Matrix
    q_norm: np.ndarray
    k_norm: np.ndarray
    post_attn_norm: np.ndarray
    post_ffn_norm: np.ndarray

    @classmethod
    def from_float(cls, raw: dict, group: int = 128):
        """raw: fp32 matrices 'qkv' [qkv_dim, d], 'o' [d, q_dim], 'gate_up'
        [2 ffn, d], 'down' [d, ffn] and fp32 gains."""
        return cls(qkv=W4Matrix.from_float(raw["qkv"], group),
                   o=W4Matrix.from_float(raw["o"], group),
                   gate_up=W4Matrix.from_float(raw["gate_up"], group),
                   down=W4Matrix.from_float(raw["down"], group),
                   q_norm=np.asarray(raw["q_norm"], np.float64),
                   k_norm=np.asarray(raw["k_norm"], np.float64),
                   post_attn_norm=np.asarray(raw["post_attn_norm"], np.float64),
                   post_ffn_norm=np.asarray(raw["post_ffn_norm"], np.float64))


class DenseLayer:
    """An OracleLayer with its four matrices dequantized once (small models)."""

    def __init__(self, layer: OracleLayer):
        self.src = layer
        self.Wqkv = layer.qkv.dequantized()
        self.Wo = layer.o.dequantized()
        self.Wgu = layer.gate_up.dequantized()
        self.Wd = layer.down.dequantized()
        self.q_norm, self.k_norm = layer.q_norm, layer.k_norm
        self.post_attn_norm, self.post_ffn_norm = layer.post_attn_norm, layer.post_ffn_norm


class OracleModel:
    """Embedding, lm_head, final norm gains and a layer provider.

    ``layers`` is either a list of OracleLayer or a callable l -> OracleLayer
    (built on demand, so a 64-layer model never sits dequantized in memory);
    a provider may also return the layer already dequantized (the
    attributes of DenseLayer, as ``fast.dense_layer`` builds them).
    """

    def __init__(self, cfg: OracleConfig, embed, lm_head, final_norm, layers,
                 cache_dense: bool = True):
        self.cfg = cfg
        self.embed = np.asarray(embed, np.float64)
        self.lm_head = np.asarray(lm_head, np.float64)
        self.final_norm = None if final_norm is None else np.asarray(final_norm, np.float64)
        self._layers = layers
        self._dense = {} if cache_dense else None

    def layer(self, l: int) -> DenseLayer:
        if self._dense is not None and l in self._dense:
            return self._dense[l]
        src = self._layers(l) if callable(self._layers) else self._layers[l]
        d = src if hasattr(src, "Wqkv") else DenseLayer(src)   # already dense (oracle.fast)
        if self._dense is not None:
            self._dense[l] = d
        return d


class OracleKV:
    """Logical KV history: K, V [L][B, kv_heads, capacity, head_dim] float64.

    Position p of sequence b lives at index p (no ring: the window is applied
    when attending)."""

    def __init__(self, cfg: OracleConfig, batch: int, capacity: int):
        shape = (batch, cfg.n_kv_heads, capacity, cfg.head_dim)
        self.K = [np.zeros(shape) for _ in range(cfg.n_layers)]
        self.V = [np.zeros(shape) for _ in range(cfg.n_layers)]

    def fill(self, l: int, b: int, start: int, k, v):
        """Store already-rotated keys k and values v [kv_heads, n, head_dim]."""
        n = np.asarray(k).shape[1]
        self.K[l][b, :, start:start + n] = k
        self.V[l][b, :, start:start + n] = v


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------
def qk_prep(cfg: OracleConfig, q_raw, k_raw, q_gain, k_gain, pos: int, full: bool):
    """QK-norm over the full projections, then rotation.

    q_raw [q_dim], k_raw [kv_dim] -> q [n_heads, hd], k [n_kv_heads, hd].
    """
    q = rmsnorm(q_raw, q_gain, cfg.eps).reshape(cfg.n_heads, cfg.head_dim)
    k = rmsnorm(k_raw, k_gain, cfg.eps).reshape(cfg.n_kv_heads, cfg.head_dim)
    inv_freq, m = layer_rope(cfg, full)
    return rope(q, pos, inv_freq, m), rope(k, pos, inv_freq, m)


def gqa_decode(cfg: OracleConfig, q, Kh, Vh, pos: int, full: bool):
    """o [n_heads, hd] for a token at ``pos`` given rotated q [n_heads, hd] and
    the KV history Kh, Vh [kv_heads, capacity, hd] that already holds ``pos``."""
    vis = visible_positions(pos, full, cfg.window)
    rep = cfg.n_heads // cfg.n_kv_heads
    scale = 1.0 / math.sqrt(cfg.head_dim)
    o = np.zeros((cfg.n_heads, cfg.head_dim))
    for g in range(cfg.n_kv_heads):
        heads = slice(g * rep, (g + 1) * rep)
        o[heads] = attend(q[heads], Kh[g, vis], Vh[g, vis], scale)
    return o


def layer_forward(cfg: OracleConfig, L: DenseLayer, l: int, x, kv: OracleKV, b: int, pos: int):
    """One post-norm decoder layer for sequence b at position pos; appends the
    token's k, v to ``kv`` and returns the new residual stream."""
    full = bool(cfg.full_layers[l])
    y = L.Wqkv @ x
    q_raw, k_raw, v = y[:cfg.q_dim], y[cfg.q_dim:cfg.q_dim + cfg.kv_dim], y[cfg.q_dim + cfg.kv_dim:]
    q, k = qk_prep(cfg, q_raw, k_raw, L.q_norm, L.k_norm, pos, full)
    kv.K[l][b, :, pos] = k
    kv.V[l][b, :, pos] = v.reshape(cfg.n_kv_heads, cfg.head_dim)
    o = gqa_decode(cfg, q, kv.K[l][b], kv.V[l][b], pos, full).reshape(-1)
    a = L.Wo @ o
    x = x + rmsnorm(a, L.post_attn_norm, cfg.eps)
    gu = L.Wgu @ x
    h = silu(gu[:cfg.ffn]) * gu[cfg.ffn:]
    f = L.Wd @ h
    return x + rmsnorm(f, L.post_ffn_norm, cfg.eps)


def head(model: OracleModel, x):
    """Final norm (reading D9) and lm_head: logits [V]."""
    cfg = model.cfg
    if model.final_norm is not None:
        x = rmsnorm(x, model.final_norm, cfg.eps)
    return model.lm_head @ x


def decode_step(model: OracleModel, kv: OracleKV, tokens, pos, n_layers: Optional[int] = None):
    """One decode step for every sequence b: token tokens[b] at position pos[b].

    Returns (logits [B, V] or None when n_layers < cfg.n_layers,
             hidden [n+1, B, d]: the embedding and the residual after each layer).
    ``n_layers`` stops early (layer-by-layer checks on the large model).
    """
    cfg = model.cfg
    n = cfg.n_layers if n_layers is None else n_layers
    B = len(tokens)
    hidden = np.zeros((n + 1, B, cfg.d_model))
    logits = np.zeros((B, cfg.vocab)) if n == cfg.n_layers else None
    xs = [model.embed[int(t)].copy() for t in tokens]
    for b in range(B):
        hidden[0, b] = xs[b]
    for l in range(n):
        L = model.layer(l)
        for b in range(B):
            xs[b] = layer_forward(cfg, L, l, xs[b], kv, b, int(pos[b]))
            hidden[l + 1, b] = xs[b]
    if logits is not None:
        for b in range(B):
            logits[b] = head(model, xs[b])
    return logits, hidden


def prefill(model: OracleModel, kv: OracleKV, tokens, b: int = 0, start_pos: int = 0):
    """Sequential decode over tokens[i] at positions start_pos + i for
    sequence b (prefill is defined as that); returns the last token's logits."""
    logits = None
    for i, t in enumerate(tokens):
        lg, _ = decode_step_one(model, kv, int(t), b, start_pos + i)
        logits = lg
    return logits


def prefill_layers(model: OracleModel, kv: OracleKV, tokens, b: int = 0, start_pos: int = 0,
                   n_layers: Optional[int] = None, keep_hidden: bool = False):
    """Prefill computed one layer at a time for all T tokens.

    The same numbers as ``prefill`` (sequential decode over positions
    start_pos + i): token i's key and value at layer l depend only on its own
    input to layer l, and its attention reads keys of positions <= its own,
    so every token's projection at layer l can be formed first (one matrix
    product over the tokens), then each position attends.  Rounding differs
    from ``prefill`` only by the order of float64 sums.

    Returns (last token's logits, or None when stopping early; the residual
    after each layer [n + 1, T, d] when keep_hidden, else None)."""
    cfg = model.cfg
    n = cfg.n_layers if n_layers is None else n_layers
    tokens = [int(t) for t in tokens]
    T = len(tokens)
    X = model.embed[tokens].copy()                       # [T, d]
    hidden = np.zeros((n + 1, T, cfg.d_model)) if keep_hidden else None
    if keep_hidden:
        hidden[0] = X
    for l in range(n):
        L = model.layer(l)
        full = bool(cfg.full_layers[l])
        Y = X @ L.Wqkv.T                                 # [T, qkv_dim]
        Q = np.zeros((T, cfg.n_heads, cfg.head_dim))
        for i in range(T):
            pos = start_pos + i
            q, k = qk_prep(cfg, Y[i, :cfg.q_dim], Y[i, cfg.q_dim:cfg.q_dim + cfg.kv_dim], L.q_norm, L.k_norm,
                           pos, full)
            Q[i] = q
            kv.K[l][b, :, pos] = k
            kv.V[l][b, :, pos] = Y[i, cfg.q_dim + cfg.kv_dim:].reshape(cfg.n_kv_heads, cfg.head_dim)
        O = np.zeros((T, cfg.q_dim))
        for i in range(T):
            O[i] = gqa_decode(cfg, Q[i], kv.K[l][b], kv.V[l][b], start_pos + i, full).reshape(-1)
        X = X + rmsnorm(O @ L.Wo.T, L.post_attn_norm, cfg.eps)
        GU = X @ L.Wgu.T
        H = silu(GU[:, :cfg.ffn]) * GU[:, cfg.ffn:]
        X = X + rmsnorm(H @ L.Wd.T, L.post_ffn_norm, cfg.eps)
        if keep_hidden:
            hidden[l + 1] = X
    logits = head(model, X[-1]) if n == cfg.n_layers else None
    return logits, hidden


def decode_step_one(model: OracleModel, kv: OracleKV, token: int, b: int, pos: int):
    """decode_step for a single sequence b of a batched cache."""
    cfg = model.cfg
    x = model.embed[token].copy()
    hidden = [x.copy()]
    for l in range(cfg.n_layers):
        x = layer_forward(cfg, model.layer(l), l, x, kv, b, pos)
        hidden.append(x.copy())
    return head(model, x), np.stack(hidden)


def argmax(logits):
    """Greedy choice, ties to the lowest index."""
    return np.argmax(np.asarray(logits), axis=-1)
