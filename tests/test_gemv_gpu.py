"""GPU parity of w4a_gemv (int4 dequant fused into the GEMV) against the oracle.

Tolerance.  x is bf16 and identical on both sides, the weights are the exact
dequantized values, so the only differences are fp32 accumulation-order
effects: per 128-group the tensor core sums products of size <= 143 |x| and the
zero point is removed as (128 + z) * sum(x), cancelling about 7 bits; summed
over K/128 groups this stays below 1e-4 relative to RMS(y).  The bound used,
2e-3 * RMS(y_ref) on the max error, leaves a 20x margin.  SiLU*mul outputs are
rounded to bf16, so that epilogue is checked element-wise: |err| <= 2^-8 |ref|
plus 1e-3 * RMS(ref) for the GEMV error.
"""
import numpy as np
import pytest
import torch

from oracle import fast, quant
from w4_weight_only_b200 import synth
from helpers import max_rel_to_rms, np64

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _api():
    from w4_weight_only_b200 import api, _abi
    return api, _abi


def _ref_rows(W, x, rows=None):
    """oracle: exact dequantized rows @ x (float64)."""
    Wn = W.numpy() if rows is None else W[rows].numpy()
    n, k = Wn.shape
    Wt = quant.dequantize(*quant.quantize_pack(Wn), n, k)
    return np64(x) @ Wt.T


@pytest.mark.parametrize("n,k", [(16, 512), (48, 1536), (768, 512), (512, 1536), (3072, 512), (1024, 2048)])
@pytest.mark.parametrize("batch", [1, 3, 8, 9, 16])
def test_gemv_small_shapes(built_lib, cuda, n, k, batch):
    api, _ = _api()
    W, x = synth.gemv_case(20, n, k, batch, "cpu")
    lin = api.quantize_linear(W.to(cuda))
    y = api.gemv(lin, x.to(cuda)).cpu().numpy()
    ref = _ref_rows(W, x)
    assert max_rel_to_rms(y, ref) <= TOL


# the four per-layer GEMVs of the 32B shape (gate/up fused)
FULL = [("qkv", 7168, 5120), ("o", 5120, 5120), ("gate_up", 55296, 5120), ("down", 5120, 27648)]


@pytest.mark.parametrize("name,n,k", FULL)
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_gemv_full_size_sampled(built_lib, cuda, name, n, k, batch):
    """Full-size launch (the benchmark's configuration): every output row
    against the oracle's vectorised dequantization (``oracle.fast``, equal
    bit for bit to ``oracle.quant``), and 96 sampled rows, the first and last
    row blocks included, through ``oracle.quant`` itself."""
    api, _ = _api()
    W, x = synth.gemv_case(21, n, k, batch, "cuda")
    lin = api.quantize_linear(W)
    y = api.gemv(lin, x).cpu().numpy()
    Wc, xc = W.cpu(), x.cpu()
    ref_all = np64(xc) @ fast.dense_matrix(Wc).T
    assert max_rel_to_rms(y, ref_all) <= TOL
    g = torch.Generator().manual_seed(n + k)
    rows = torch.cat([torch.arange(16), torch.arange(n - 16, n), torch.randint(0, n, (64,), generator=g)])
    ref = _ref_rows(Wc, xc, rows.numpy())
    assert max_rel_to_rms(y[:, rows.numpy()], ref) <= TOL


def test_gemv_sumsq_epilogue(built_lib, cuda):
    api, abi = _api()
    n, k, B = 1024, 1536, 3
    W, x = synth.gemv_case(22, n, k, B, "cpu")
    lin = api.quantize_linear(W.to(cuda))
    y, aux = api.gemv(lin, x.to(cuda), epilogue=abi.EPI_SUMSQ)
    ref = _ref_rows(W, x)
    assert max_rel_to_rms(y.cpu().numpy(), ref) <= TOL
    ss_ref = (ref.reshape(B, n // 16, 16) ** 2).sum(-1).T       # [n/16, B]
    assert np.allclose(aux.cpu().numpy(), ss_ref, rtol=5e-3, atol=0)


@pytest.mark.parametrize("ffn,k,batch", [(1536, 512, 1), (1536, 512, 5), (27648, 5120, 1), (27648, 5120, 16)])
def test_gemv_silu_mul_epilogue(built_lib, cuda, ffn, k, batch):
    """gate/up rows tiled interleaved; out = silu(gate x) * (up x) in bf16."""
    api, abi = _api()
    W, x = synth.gemv_case(23, 2 * ffn, k, batch, "cuda" if ffn > 4096 else "cpu")
    lin = api.quantize_linear(W.to(cuda), row_interleave=True)
    h = api.gemv(lin, x.to(cuda), epilogue=abi.EPI_SILU_MUL).float().cpu().numpy()
    g = torch.Generator().manual_seed(5)
    js = torch.cat([torch.arange(8), torch.randint(0, ffn, (56,), generator=g)]).numpy()
    gate = _ref_rows(W.cpu(), x.cpu(), js)
    up = _ref_rows(W.cpu(), x.cpu(), js + ffn)
    ref = gate / (1.0 + np.exp(-gate)) * up
    # bf16 output: round-to-nearest error <= 2^-8 of the value, plus the GEMV's own error
    slack = 1e-3 * np.sqrt(np.mean(ref * ref))
    assert np.all(np.abs(h[:, js] - ref) <= 2.0 ** -8 * np.abs(ref) + slack)


def test_gemv_deterministic(built_lib, cuda):
    api, _ = _api()
    W, x = synth.gemv_case(24, 5120, 27648, 4, "cuda")
    lin = api.quantize_linear(W)
    ws = api.gemv_workspace(lin, 4)
    y1 = api.gemv(lin, x, ws=ws).clone()
    y2 = api.gemv(lin, x, ws=ws)
    assert torch.equal(y1, y2)
    api.check(ws)
