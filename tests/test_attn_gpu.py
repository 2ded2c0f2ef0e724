"""GPU parity of QK-norm + rotation + KV append (w4a_qk_prep) and GQA decode
attention (w4a_attn_decode) against the oracle.

Tolerance.  The cache holds k and v in bf16 (at most 2^-8 relative error
per element) and the standalone q input is bf16; q and the softmax weights
enter the tensor cores as hi + lo bf16 pairs and o is rounded to bf16 once.
Each bf16 rounding is an independent <= 0.4% relative perturbation, so the
max error over a head stays near 1-2% of RMS(o).  Bound: 3e-2 * RMS(o_ref).
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import max_rel_to_rms, np64, oracle_config

pytestmark = pytest.mark.gpu
TOL = 3e-2


def _api():
    from w4_weight_only_b200 import api
    return api


def _run_case(cuda, cfg, batch, ctx_list, full, sample, seed=30):
    """Sequence b holds positions [0, ctx_b) (N(0,1) rows; a ring of `window`
    slots on SWA) and decodes the token at position ctx_b."""
    api = _api()
    nkv, hd, nq = cfg.n_kv_heads, cfg.head_dim, cfg.n_heads
    W = cfg.window
    max_ctx = max(ctx_list)
    slots = ((max_ctx + 1 + 15) // 16) * 16 if full else W
    kc = torch.zeros((batch, nkv, slots, hd), dtype=torch.bfloat16, device=cuda)
    vc = torch.zeros_like(kc)
    hist = {}
    for b, ctx in enumerate(ctx_list):
        k, v = synth.kv_rows(seed, 0, b, nkv, ctx, hd, "cuda")
        hist[b] = (k, v)
        if full:
            api.kv_write_region(kc, vc, batch, nkv, hd, slots, b, 0, k, v)
        else:
            lo = max(0, ctx - (W - 1))          # the ring keeps the last W-1 old positions
            # positions [lo, ctx) land in slots p % W: at most two contiguous runs
            p = lo
            while p < ctx:
                s0 = p % W
                n = min(ctx - p, W - s0)
                api.kv_write_region(kc, vc, batch, nkv, hd, slots, b, s0, k[:, p:p + n].contiguous(),
                                    v[:, p:p + n].contiguous())
                p += n
    g = torch.Generator(device="cuda").manual_seed(seed)
    q_raw = torch.randn((batch, nq * hd), generator=g, device="cuda")
    k_raw = torch.randn((batch, nkv * hd), generator=g, device="cuda")
    v_raw = torch.randn((batch, nkv * hd), generator=g, device="cuda")
    q_gain = 1 + 0.1 * torch.randn((nq * hd,), generator=g, device="cuda")
    k_gain = 1 + 0.1 * torch.randn((nkv * hd,), generator=g, device="cuda")
    pos = torch.tensor(ctx_list, dtype=torch.int32, device="cuda")
    q = api.qk_prep(cfg, full, q_raw, k_raw, v_raw, q_gain, k_gain, pos, kc, vc, slots)
    out = api.attn_decode(q, kc, vc, nkv, slots, pos, window=0 if full else W)
    torch.cuda.synchronize()
    ocfg = oracle_config(cfg)
    GQ = nq // nkv
    worst = 0.0
    for (b, grp) in sample:
        ctx = ctx_list[b]
        qo, ko = om.qk_prep(ocfg, np64(q_raw[b]), np64(k_raw[b]), np64(q_gain), np64(k_gain), ctx, full)
        vis = om.visible_positions(ctx, full, W)
        k, v = hist[b]
        old = vis[vis < ctx]
        K = np.concatenate([np64(k[grp, old]), ko[grp][None]], 0)
        V = np.concatenate([np64(v[grp, old]), np64(v_raw[b, grp * hd:(grp + 1) * hd])[None]], 0)
        ref = om.attend(qo[grp * GQ:(grp + 1) * GQ], K, V, 1.0 / np.sqrt(hd))
        got = np64(out[b, grp * GQ:(grp + 1) * GQ])
        e = max_rel_to_rms(got, ref)
        worst = max(worst, e)
        assert e <= TOL, (b, grp, e)
    return worst


CFG32 = wc.olmo3_32b(4)


@pytest.mark.parametrize("batch", [1, 8])
@pytest.mark.parametrize("ctx,full", [(4096, True), (16384, True), (65536, True), (16384, False), (65536, False)])
def test_attention_config_shapes(built_lib, cuda, batch, ctx, full):
    sample = [(0, 0), (0, 7), (batch - 1, 3)]
    _run_case(cuda, CFG32, batch, [ctx] * batch, full, sample)


@pytest.mark.parametrize("ctx", [0, 1, 6, 7, 8, 126, 127, 128, 200, 4094, 4095, 4096, 4097, 8191])
@pytest.mark.parametrize("full", [True, False])
def test_attention_edges(built_lib, cuda, ctx, full):
    """Empty history, ragged tails of the 8-key and 128-key tiles, ctx around the
    window (ring not yet full, exactly full, wrapped)."""
    _run_case(cuda, CFG32, 1, [ctx], full, [(0, g) for g in range(8)])


def test_attention_ragged_batch(built_lib, cuda):
    ctxs = [5, 130, 4095, 4100, 700, 64, 1, 9000]
    _run_case(cuda, CFG32, 8, ctxs, True, [(b, b % 8) for b in range(8)])
    _run_case(cuda, CFG32, 8, ctxs, False, [(b, (b + 3) % 8) for b in range(8)])


def test_attention_tiny_head_dim(built_lib, cuda):
    cfg = wc.tiny()
    for ctx in (3, 63, 64, 65, 300):
        for full in (True, False):
            _run_case(cuda, cfg, 2, [ctx, ctx // 2 + 1], full, [(0, 0), (0, 1), (1, 1)])


def test_qk_prep_append_matches_oracle(built_lib, cuda):
    """The appended k (rotated, bf16) and v in the cache slot of pos."""
    api = _api()
    cfg = CFG32
    nkv, hd = cfg.n_kv_heads, cfg.head_dim
    slots, pos_v = 4096, 5000
    kc = torch.zeros((1, nkv, slots, hd), dtype=torch.bfloat16, device=cuda)
    vc = torch.zeros_like(kc)
    g = torch.Generator(device="cuda").manual_seed(3)
    q_raw = torch.randn((1, cfg.q_dim), generator=g, device="cuda")
    k_raw = torch.randn((1, cfg.kv_dim), generator=g, device="cuda")
    v_raw = torch.randn((1, cfg.kv_dim), generator=g, device="cuda")
    qg = 1 + 0.1 * torch.randn((cfg.q_dim,), generator=g, device="cuda")
    kg = 1 + 0.1 * torch.randn((cfg.kv_dim,), generator=g, device="cuda")
    pos = torch.tensor([pos_v], dtype=torch.int32, device="cuda")
    for full in (False, True):
        q = api.qk_prep(cfg, full, q_raw, k_raw, v_raw, qg, kg, pos, kc, vc, slots)
        k_rows = torch.empty((nkv, 1, hd), dtype=torch.bfloat16, device="cuda")
        v_rows = torch.empty_like(k_rows)
        from w4_weight_only_b200 import _abi
        _abi.call("w4a_kv_read", api._p(kc), api._p(vc), 1, nkv, hd, slots, 0, pos_v % slots, 1, api._p(k_rows),
                  api._p(v_rows), api._stream())
        qo, ko = om.qk_prep(oracle_config(cfg), np64(q_raw[0]), np64(k_raw[0]), np64(qg), np64(kg), pos_v, full)
        # bf16 outputs: round-to-nearest error is at most 2^-8 of the value
        for got, ref in ((np64(q[0]), qo), (np64(k_rows[:, 0]), ko)):
            slack = 1e-5 * np.sqrt(np.mean(ref * ref))
            assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + slack)
        assert np.array_equal(np64(v_rows[:, 0]).reshape(-1), np64(v_raw[0].to(torch.bfloat16)))
