"""Oracle: the int4 quantizer and the dense layer on many CPU threads.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The 64-layer OLMo-3-32B-shaped model holds 31 G int4 weights.  ``quant``
decides them with numpy on one thread (about a minute per layer); this module
states the same steps with PyTorch CPU operations, which run on every host
core, so that a whole-model oracle pass takes minutes.  It computes exactly
what ``quant.quantize`` and ``quant.dequantize`` compute (ATLAS-OLMo-3-32B-
Think-v4 model card, "Quantization recipe"; readings D1, D3, D4):

    per (row n, group g) of ``group`` consecutive columns, in IEEE binary32
    with each operation rounded to nearest-even:
        s = fp16(fl32(fl32(max - min) / 15)), 0 -> 2**-24, overflow -> 65504
        z = clamp(rint(fl32(-min / s)), 0, 15)
        q = clamp(rint(fl32(w / s)) + z, 0, 15)
    dequantized weight (q - z) * s, exact in float64.

``torch.round`` rounds halves to even like ``numpy.rint``, and CPU float32
division is IEEE-correct, so the codes agree bit for bit; the pin is
``tests/test_oracle_fast.py`` (random matrices, ties, constant and huge-range
groups, and the z = 8 case).

``dense_layer`` returns an object with the attributes ``model.layer_forward``
reads (the four dequantized float64 matrices and the gains), built from a
layer's float32 weights.

Parity status: pinned to ``quant`` (which is pinned to the pages).
"""
from __future__ import annotations

from types import SimpleNamespace

import numpy as np
import torch

_FP16_MAX = 65504.0
_FP16_MIN_SUBNORMAL = 2.0 ** -24


def quantize(W: torch.Tensor, group: int = 128):
    """W float32 [N, K] (CPU) -> (codes uint8 [N, K], scales float16 [K/g, N],
    zeros uint8 [K/g, N]), the same triple as ``quant.quantize``."""
    W = W.to(torch.float32).contiguous()
    N, K = W.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = W.view(N, K // group, group)
    mn = G.amin(dim=2)
    mx = G.amax(dim=2)
    s32 = (mx - mn) / 15.0                      # two binary32 operations
    s16 = s32.to(torch.float16)                 # nearest-even; beyond 65504 -> inf
    s16 = torch.where(torch.isinf(s16), torch.full_like(s16, _FP16_MAX), s16)
    s16 = torch.where(s16 == 0, torch.full_like(s16, _FP16_MIN_SUBNORMAL), s16)
    s = s16.to(torch.float32)
    z = torch.round(-mn / s).clamp_(0, 15)
    q = torch.round(G / s.unsqueeze(2)).add_(z.unsqueeze(2)).clamp_(0, 15)
    codes = q.to(torch.uint8).view(N, K)
    return codes, s16.t().contiguous(), z.to(torch.uint8).t().contiguous()


def dequantize(codes: torch.Tensor, s16: torch.Tensor, z: torch.Tensor, group: int = 128) -> torch.Tensor:
    """(q - z) * s as float64 [N, K] from the triple of ``quantize``."""
    N, K = codes.shape
    d = codes.view(N, K // group, group).to(torch.int16) - z.t().to(torch.int16).unsqueeze(2)
    w = d.to(torch.float64)
    w.mul_(s16.t().to(torch.float64).unsqueeze(2))
    return w.view(N, K)


def dense_matrix(W, group: int = 128) -> np.ndarray:
    """The exactly dequantized float64 form of float32 weights W [N, K]."""
    t = W if isinstance(W, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32))
    return dequantize(*quantize(t.cpu(), group), group).numpy()


def dense_layer(raw: dict, group: int = 128):
    """raw: float32 'qkv', 'o', 'gate_up', 'down' and the four gains (torch or
    numpy).  Returns the layer as ``model.layer_forward`` uses it."""
    def g(name):
        v = raw[name]
        return (v.detach().cpu().double().numpy() if isinstance(v, torch.Tensor)
                else np.asarray(v, dtype=np.float64))
    return SimpleNamespace(Wqkv=dense_matrix(raw["qkv"], group), Wo=dense_matrix(raw["o"], group),
                           Wgu=dense_matrix(raw["gate_up"], group), Wd=dense_matrix(raw["down"], group),
                           q_norm=g("q_norm"), k_norm=g("k_norm"), post_attn_norm=g("post_attn_norm"),
                           post_ffn_norm=g("post_ffn_norm"))
