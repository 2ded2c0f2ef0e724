"""Oracle: a loop-by-loop restatement of one decoder layer (tiny shapes only).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Pure-Python scalar loops over the same definition ``model`` implements with
array operations (same pages, same readings D5-D13).  It shares no helper with
``model``: norms, rotation, frequencies, softmax and the matrix products are
written out element by element, so that a transposed operand, a dropped term or
a wrong index in the vectorised oracle shows up as a mismatch.  Use it only on
shapes of a few dozen elements.
"""
from __future__ import annotations

import math


def _matvec(W, x):
    n = len(W)
    return [sum(W[i][j] * x[j] for j in range(len(x))) for i in range(n)]


def _rms(v, g, eps):
    ms = sum(t * t for t in v) / len(v)
    r = 1.0 / math.sqrt(ms + eps)
    return [v[i] * r * g[i] for i in range(len(v))]


def _freq(i, hd, theta, full, factor, orig, bf, bs):
    f = 1.0 / (theta ** ((2.0 * i) / hd))
    if not full:
        return f
    lo = math.floor(hd * math.log(orig / (bf * 2.0 * math.pi)) / (2.0 * math.log(theta)))
    hi = math.ceil(hd * math.log(orig / (bs * 2.0 * math.pi)) / (2.0 * math.log(theta)))
    lo = max(lo, 0)
    hi = min(hi, hd - 1)
    if i <= lo:
        r = 0.0
    elif i >= hi:
        r = 1.0
    else:
        r = (i - lo) / (hi - lo)
    return f * (1.0 - r) + (f / factor) * r


def _rotate(vec, pos, hd, theta, full, factor, orig, bf, bs):
    m = (0.1 * math.log(factor) + 1.0) if (full and factor > 1.0) else 1.0
    half = hd // 2
    out = [0.0] * hd
    for i in range(half):
        a = pos * _freq(i, hd, theta, full, factor, orig, bf, bs)
        c, s = math.cos(a) * m, math.sin(a) * m
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def layer(cfg, Wqkv, Wo, Wgu, Wd, q_norm, k_norm, g_attn, g_ffn, x, Khist, Vhist, pos, full):
    """One post-norm layer for a token at ``pos``.

    W* are lists of rows (already dequantized).  Khist/Vhist: dict
    (kv_head, position) -> vector for the earlier positions; the token's own
    k, v are added to them.  Returns the new residual.
    """
    hq, hk, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    kw = (cfg.rope_theta, full, cfg.yarn_factor, cfg.yarn_orig_ctx, cfg.beta_fast, cfg.beta_slow)
    y = _matvec(Wqkv, x)
    qd, kd = hq * hd, hk * hd
    q = _rms(y[:qd], q_norm, cfg.eps)
    k = _rms(y[qd:qd + kd], k_norm, cfg.eps)
    v = y[qd + kd:]
    for g in range(hk):
        Khist[(g, pos)] = _rotate(k[g * hd:(g + 1) * hd], pos, hd, *kw)
        Vhist[(g, pos)] = v[g * hd:(g + 1) * hd]
    lo = 0 if full else max(0, pos - cfg.window + 1)
    o = []
    for h in range(hq):
        g = h // (hq // hk)
        qh = _rotate(q[h * hd:(h + 1) * hd], pos, hd, *kw)
        scores = []
        for j in range(lo, pos + 1):
            kj = Khist[(g, j)]
            scores.append(sum(qh[d] * kj[d] for d in range(hd)) / math.sqrt(hd))
        mx = max(scores)
        e = [math.exp(s - mx) for s in scores]
        tot = sum(e)
        for d in range(hd):
            o.append(sum(e[i] / tot * Vhist[(g, lo + i)][d] for i in range(len(e))))
    a = _matvec(Wo, o)
    an = _rms(a, g_attn, cfg.eps)
    x = [x[i] + an[i] for i in range(len(x))]
    gu = _matvec(Wgu, x)
    F = cfg.ffn
    hvec = [gu[i] / (1.0 + math.exp(-gu[i])) * gu[F + i] for i in range(F)]
    f = _matvec(Wd, hvec)
    fn = _rms(f, g_ffn, cfg.eps)
    return [x[i] + fn[i] for i in range(len(x))]
