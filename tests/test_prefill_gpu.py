"""GPU parity of the prefill's building blocks against the oracle.

w4a_gemm (the prompt-time int4 projection on the tcgen05 tensor cores):
out = x . W~^T for fp16 x [M, k].  The kernel multiplies weights expanded to
fp16, (q - z) * s rounded to nearest (relative error <= 2^-11 per weight),
with fp32 accumulation; over k products of random sign that is ~2^-11 / sqrt(3)
of RMS(y) per output, so the bound on the max error is 3e-3 * RMS(y_ref).
M covers partial 128-row tiles (9, 77, 200, 300, 1200), both tile widths
and, at the O shape with 1,200 rows, K cut in two halves whose sums are
added into the output.  SwiGLU outputs are fp16: element-wise, the GEMM
bound carried through silu(g) * u to first order plus fp16 rounding
(2^-11 |ref|).

w4a_attn_prefill (causal GQA attention of a prompt over the cache, the
sliding window as a ring): compared with the oracle's per-query attention
(softmax(q K^T / sqrt(d)) V over the visible positions), element-wise: the
probabilities enter the P.V product rounded to bf16 (relative 2^-9), so
|err| <= 2^-9 max|v| over the visible values (bound doubled), plus the fp16
rounding of the output.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fast
from oracle import model as om
from w4_weight_only_b200 import synth
from helpers import np64

pytestmark = pytest.mark.gpu

GEMM_TOL = 3e-3


def _api():
    from w4_weight_only_b200 import api, _abi
    return api, _abi


@pytest.mark.parametrize("n,k,M,scaled", [(768, 512, 9, False), (768, 512, 200, True), (512, 1536, 77, False),
                                          (7168, 5120, 1200, True), (5120, 27648, 300, False),
                                          (5120, 5120, 130, False), (5120, 5120, 1200, True)])
def test_gemm_against_oracle(built_lib, cuda, n, k, M, scaled):
    api, _ = _api()
    dev = "cuda" if n * k > 4_000_000 else "cpu"
    W = synth.normal((n, k), dev, 0.02, 0.0, 50, "gemm_w", n, k)
    x = synth.normal((M, k), "cpu", 1.0, 0.0, 50, "gemm_x", M, k).to(torch.float16)
    rs = None
    if scaled:  # powers of two, as the range guard produces them
        rs = torch.tensor([2.0 ** ((i % 5) - 2) for i in range(M)], dtype=torch.float32)
    lin = api.quantize_linear(W.to(cuda))
    ws = api.gemm_workspace(lin)
    y = api.gemm(lin, x.to(cuda), row_scale=None if rs is None else rs.to(cuda), ws=ws).cpu().numpy()
    api.check(ws)
    ref = np64(x) @ fast.dense_matrix(W.cpu()).T
    if rs is not None:
        ref *= rs.double().numpy()[:, None]
    err = np.abs(y - ref) / np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    assert float(err.max()) <= GEMM_TOL, float(err.max())


@pytest.mark.parametrize("ffn,k,M", [(1536, 512, 130), (27648, 5120, 257)])
def test_gemm_silu_epilogue(built_lib, cuda, ffn, k, M):
    api, abi = _api()
    dev = "cuda" if ffn > 4096 else "cpu"
    W = synth.normal((2 * ffn, k), dev, 0.02, 0.0, 51, "gemm_gu", ffn, k)
    x = synth.normal((M, k), "cpu", 1.0, 0.0, 51, "gemm_gu_x", M, k).to(torch.float16)
    lin = api.quantize_linear(W.to(cuda), row_interleave=True)
    ws = api.gemm_workspace(lin)
    h = api.gemm(lin, x.to(cuda), epilogue=abi.EPI_SILU_MUL, ws=ws).float().cpu().numpy()
    api.check(ws)
    Wd = fast.dense_matrix(W.cpu())
    gu = np64(x) @ Wd.T
    g_, u_ = gu[:, :ffn], gu[:, ffn:]
    sig = 1.0 / (1.0 + np.exp(-g_))
    ref = g_ * sig * u_
    # first-order propagation of the GEMM bound e on gate and up through
    # silu(g) * u, plus the fp16 rounding of h
    e = GEMM_TOL * np.sqrt(np.mean(gu * gu))
    dsilu = sig * (1.0 + g_ * (1.0 - sig))
    bound = e * (np.abs(dsilu * u_) + np.abs(g_ * sig)) + 2.0 ** -11 * np.abs(ref) + 1e-6
    assert np.all(np.abs(h - ref) <= bound)


def _region(batch, nkv, slots, hd):
    return torch.zeros((batch, nkv, slots, hd), dtype=torch.bfloat16, device="cuda")


def _write_history(api, kreg, vreg, batch, nkv, hd, slots, seq, window, K, V, start):
    """Positions [0, start) as the cache holds them: at their own slots, or the
    last `window` of them at position % window."""
    lo = max(0, start - window) if window else 0
    p = lo
    while p < start:
        s0 = p % window if window else p
        n = min(start - p, (window - s0) if window else start - p)
        api.kv_write_region(kreg, vreg, batch, nkv, hd, slots, seq, s0, K[:, p:p + n].contiguous(),
                            V[:, p:p + n].contiguous())
        p += n


@pytest.mark.parametrize("nq,nkv,hd,T,start,window,sample", [
    (8, 2, 64, 200, 0, 0, None),        # the small decoder's shape, full attention
    (8, 2, 64, 300, 100, 64, None),     # sliding window 64 over a pre-filled history
    (8, 2, 64, 77, 37, 0, None),        # full attention after a history, ragged ends
    (40, 8, 128, 1200, 0, 0, 256),      # the 32B shape, a 1,200-token prompt
    (40, 8, 128, 1200, 3500, 4096, 256),  # window 4,096 after 3,500 positions
    (40, 8, 128, 8192, 0, 4096, 128),   # an 8,192-token prompt through a 4,096-key window
])
def test_attn_prefill_against_oracle(built_lib, cuda, nq, nkv, hd, T, start, window, sample):
    api, _ = _api()
    batch, seq = 2, 1
    end = start + T
    slots = window if window else (end + 15) // 16 * 16
    kreg, vreg = _region(batch, nkv, slots, hd), _region(batch, nkv, slots, hd)
    K, V = synth.kv_rows(60, T, start, nkv, end, hd, "cuda")
    _write_history(api, kreg, vreg, batch, nkv, hd, slots, seq, window, K, V, start)
    q = synth.normal((T, nq, hd), "cuda", 1.0, 0.0, 61, "attn_q", T, start).to(torch.bfloat16)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    snap = kreg.clone()
    out = api.attn_prefill(q, kreg, vreg, K[:, start:].contiguous(), V[:, start:].contiguous(), batch, seq, slots,
                           window, start, ws=ws).float().cpu().numpy()
    api.check(ws)
    assert torch.equal(kreg, snap)  # the cache is only read
    Kn, Vn, qn = np64(K), np64(V), np64(q)
    rep = nq // nkv
    if sample is None:
        rows = np.arange(T)
    else:
        g = torch.Generator().manual_seed(T + start)
        rows = np.unique(np.concatenate([np.arange(64), np.arange(T - 64, T),
                                         torch.randint(0, T, (sample,), generator=g).numpy()]))
    scale = 1.0 / math.sqrt(hd)
    for t in rows:
        pos = start + t
        vis = om.visible_positions(pos, window == 0, window)
        for g0 in range(nkv):
            ref = om.attend(qn[t, g0 * rep:(g0 + 1) * rep], Kn[g0, vis], Vn[g0, vis], scale)
            vmax = float(np.abs(Vn[g0, vis]).max())
            got = out[t, g0 * rep:(g0 + 1) * rep]
            # the weights enter P.V rounded to bf16 (relative 2^-9 each, the
            # normaliser unrounded): |err| <= 2^-9 max|v|; doubled for the fp32
            # sums, plus the fp16 rounding of the output
            bound = 2.0 ** -8 * vmax + 2.0 ** -10 * np.abs(ref) + 1e-6
            assert np.all(np.abs(got - ref) <= bound), (t, g0, float(np.abs(got - ref).max()))
