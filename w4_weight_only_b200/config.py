"""Model shape (mirror of W4AConfig in include/w4a.h) and the two presets.

Sources: ATLAS-OLMo-3-32B-Think-v4 model card, "Architecture deep-dive" (the
32B shape); archdb "Olmo-3-1125-32B" (eps, YaRN on full layers only).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

from . import _abi


def swa_full_pattern(n_layers: int) -> List[bool]:
    """[SWA, SWA, SWA, full] repeated; layer l is full iff l % 4 == 3."""
    return [(l % 4) == 3 for l in range(n_layers)]


@dataclass
class Config:
    d_model: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    window: int
    full_layers: List[bool] = field(default_factory=list)
    rope_theta: float = 500000.0
    yarn_factor: float = 8.0
    yarn_orig_ctx: int = 8192
    yarn_beta_fast: float = 32.0
    yarn_beta_slow: float = 1.0
    eps: float = 1e-6
    group: int = 128
    final_norm: bool = True

    def __post_init__(self):
        if not self.full_layers:
            self.full_layers = swa_full_pattern(self.n_layers)

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_dim(self) -> int:
        return self.q_dim + 2 * self.kv_dim

    def to_c(self) -> _abi.W4AConfig:
        c = _abi.W4AConfig()
        c.d_model, c.n_layers, c.n_heads, c.n_kv_heads = self.d_model, self.n_layers, self.n_heads, self.n_kv_heads
        c.head_dim, c.ffn, c.vocab, c.window = self.head_dim, self.ffn, self.vocab, self.window
        for l, f in enumerate(self.full_layers):
            c.full_layers[l] = 1 if f else 0
        c.rope_theta, c.yarn_factor, c.yarn_orig_ctx = self.rope_theta, self.yarn_factor, self.yarn_orig_ctx
        c.group, c.yarn_beta_fast, c.yarn_beta_slow = self.group, self.yarn_beta_fast, self.yarn_beta_slow
        c.eps, c.final_norm = self.eps, 1 if self.final_norm else 0
        return c


def olmo3_32b(n_layers: int = 64) -> Config:
    """OLMo-3-32B shape: d 5120, 64 layers, 40 q / 8 kv heads of 128, SwiGLU
    27,648, vocab 100,278, window 4,096."""
    return Config(d_model=5120, n_layers=n_layers, n_heads=40, n_kv_heads=8, head_dim=128, ffn=27648,
                  vocab=100278, window=4096)


def tiny() -> Config:
    """The small decoder used for end-to-end parity: 4 layers [SWA, SWA, SWA,
    full], d 512, 8 q / 2 kv heads of 64, SwiGLU 1536, vocab 4096, window 64."""
    return Config(d_model=512, n_layers=4, n_heads=8, n_kv_heads=2, head_dim=64, ffn=1536, vocab=4096,
                  window=64)
