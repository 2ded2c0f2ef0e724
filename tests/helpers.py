"""Builders that give the CUDA path and the oracle the same seeded inputs.

Inputs come only from ``w4_weight_only_b200.synth``; the GPU side quantizes
with the library's own kernels and the oracle with its own code.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import model as om
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth


def oracle_config(cfg: wc.Config) -> om.OracleConfig:
    return om.OracleConfig(d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                           n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                           window=cfg.window, full_layers=list(cfg.full_layers), rope_theta=cfg.rope_theta,
                           yarn_factor=cfg.yarn_factor, yarn_orig_ctx=cfg.yarn_orig_ctx,
                           beta_fast=cfg.yarn_beta_fast, beta_slow=cfg.yarn_beta_slow, eps=cfg.eps,
                           group=cfg.group, final_norm=cfg.final_norm)


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float32).numpy()


class Pair:
    """The GPU model and the oracle model built from the same seed.

    gen_device: where synth draws the float weights ('cpu' for small models,
    'cuda' for the 32B shape).  The oracle receives host copies.
    """

    def __init__(self, cfg: wc.Config, seed: int, gen_device: str = "cpu", oracle_cache: bool = True,
                 embed_scale: float = 1.0, weight_scale: dict = None, oracle_fast: bool = False):
        """embed_scale, weight_scale {name: factor}: powers of two that scale
        the embedding and the named float matrices exactly (range tests).
        oracle_fast: the oracle quantizes with oracle.fast (all host cores)."""
        from w4_weight_only_b200 import api
        self.cfg, self.seed, self.gen_device = cfg, seed, gen_device
        emb, head, fin = synth.embed_head(cfg, seed, gen_device)
        if embed_scale != 1.0:
            emb = (emb.float() * embed_scale).to(torch.bfloat16)
        self.emb, self.head, self.fin = emb, head, fin
        wscale = dict(weight_scale or {})

        def layer_float(l):
            raw = synth.layer_float(cfg, seed, l, gen_device)
            for name, f in wscale.items():
                raw[name] = raw[name] * f
            return raw

        def layer_gpu(l):
            return {k: v.to("cuda") for k, v in layer_float(l).items()}

        self.gpu = api.Model.from_float(cfg, emb.to("cuda"), head.to("cuda"),
                                        fin.to("cuda") if cfg.final_norm else None, layer_gpu)
        torch.cuda.synchronize()
        self.ocfg = oracle_config(cfg)

        def layer_oracle(l):
            if oracle_fast:
                from oracle import fast
                return fast.dense_layer({k: v.cpu() for k, v in layer_float(l).items()}, cfg.group)
            return om.OracleLayer.from_float({k: np32(v) for k, v in layer_float(l).items()}, cfg.group)

        self.oracle = om.OracleModel(self.ocfg, np64(emb), np64(head), np64(fin) if cfg.final_norm else None,
                                     layer_oracle, cache_dense=oracle_cache)


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(math.sqrt(np.mean(a * a)))


def max_rel_to_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / max(rms(ref), 1e-30))


class Sym32Pair:
    """The GPU model and the oracle built from the same seeded checkpoint in
    the model card's symmetric group-32 format (cfg.group = 32): the GPU
    tiles the stored nibbles and bf16 scales, the oracle dequantizes them
    with its own reading of the format."""

    def __init__(self, cfg: wc.Config, seed: int, gen_device: str = "cpu"):
        from types import SimpleNamespace
        from oracle import quant
        from w4_weight_only_b200 import api
        assert cfg.group == 32
        self.cfg, self.seed = cfg, seed
        emb, head, fin = synth.embed_head(cfg, seed, gen_device)
        self.emb, self.head, self.fin = emb, head, fin

        def layer_gpu(l):
            raw = synth.sym32_layer(cfg, seed, l, gen_device)
            return {k: (tuple(t.to("cuda") for t in v) if isinstance(v, tuple) else v.to("cuda"))
                    for k, v in raw.items()}

        self.gpu = api.Model.from_sym32(cfg, emb.to("cuda"), head.to("cuda"),
                                        fin.to("cuda") if cfg.final_norm else None, layer_gpu)
        torch.cuda.synchronize()
        self.ocfg = oracle_config(cfg)

        def dense(pair):
            qw, sc = pair
            n, k = qw.shape[0], qw.shape[1] * 8
            return quant.dequantize_sym32(qw.cpu().numpy().view(np.uint32), sc.cpu().view(torch.int16).numpy()
                                          .view(np.uint16), n, k)

        def layer_oracle(l):
            raw = synth.sym32_layer(cfg, seed, l, gen_device)
            return SimpleNamespace(Wqkv=dense(raw["qkv"]), Wo=dense(raw["o"]), Wgu=dense(raw["gate_up"]),
                                   Wd=dense(raw["down"]), q_norm=np64(raw["q_norm"]), k_norm=np64(raw["k_norm"]),
                                   post_attn_norm=np64(raw["post_attn_norm"]),
                                   post_ffn_norm=np64(raw["post_ffn_norm"]))

        self.oracle = om.OracleModel(self.ocfg, np64(emb), np64(head), np64(fin) if cfg.final_norm else None,
                                     layer_oracle, cache_dense=True)
