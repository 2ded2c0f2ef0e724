"""Pins for ``oracle.fast`` (the multithreaded restatement of the quantizer):
it must give exactly the codes, scales and zeros of ``oracle.quant`` (itself
pinned to the model card's format and to brute force) and the same exact
dequantized weights.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import fast, quant


def _same(W: np.ndarray, group: int = 128):
    c_np, s_np, z_np = quant.quantize(W, group)
    c_t, s_t, z_t = fast.quantize(torch.from_numpy(W), group)
    assert np.array_equal(c_np, c_t.numpy())
    assert np.array_equal(s_np.view(np.uint16), s_t.numpy().view(np.uint16))
    assert np.array_equal(z_np, z_t.numpy())
    n, k = W.shape
    ref = quant.dequantize(*quant.pack(c_np, s_np, z_np), n, k, group)
    assert np.array_equal(ref, fast.dequantize(c_t, s_t, z_t, group).numpy())


@pytest.mark.parametrize("seed,n,k,std", [(0, 64, 512, 0.02), (1, 48, 1536, 1.0), (2, 256, 256, 3e-4),
                                          (3, 16, 1024, 2e4)])
def test_random_matrices(seed, n, k, std):
    r = np.random.default_rng(seed)
    _same((r.standard_normal((n, k)) * std).astype(np.float32))


def test_ties_constant_and_huge_groups():
    r = np.random.default_rng(9)
    W = (r.standard_normal((40, 256)) * 0.05).astype(np.float32)
    # a constant group (scale 2^-24, z = 0)
    W[0, :128] = 0.3
    # codes exactly on a half step: s = 0.5, values at (j + 0.5) * 0.5
    W[1, :128] = ((np.arange(128) % 15) * 0.5 + 0.25).astype(np.float32)
    W[1, 0], W[1, 1] = 0.0, 7.5
    # range beyond fp16 (scale clamps to 65504)
    W[2, 128:] = np.linspace(-1e6, 1e6, 128, dtype=np.float32)
    # range / 15 right at an fp16 rounding boundary: 2^-10 * (1 + 2^-11) and one fp32 ulp either side
    mid = np.float32(2.0 ** -10 * (1 + 2.0 ** -11))
    for i, q15 in enumerate((np.nextafter(mid, np.float32(0)), mid, np.nextafter(mid, np.float32(1)))):
        W[3 + i, :128] = np.linspace(0, np.float32(15.0) * q15, 128, dtype=np.float32)
    # the symmetric special case z = 8
    q = r.integers(0, 16, size=128)
    q[0], q[1] = 0, 15
    W[6, 128:] = ((q - 8) * 0.25).astype(np.float32)
    _same(W)


def test_dense_layer_matches_oracle_layer():
    from oracle import model as om
    r = np.random.default_rng(4)
    raw = {"qkv": (r.standard_normal((64, 256)) * 0.02).astype(np.float32),
           "o": (r.standard_normal((256, 128)) * 0.02).astype(np.float32),
           "gate_up": (r.standard_normal((512, 256)) * 0.02).astype(np.float32),
           "down": (r.standard_normal((256, 256)) * 0.02).astype(np.float32),
           "q_norm": r.standard_normal(32), "k_norm": r.standard_normal(16),
           "post_attn_norm": r.standard_normal(256), "post_ffn_norm": r.standard_normal(256)}
    a = fast.dense_layer(raw)
    b = om.DenseLayer(om.OracleLayer.from_float(raw))
    for name in ("Wqkv", "Wo", "Wgu", "Wd", "q_norm", "k_norm", "post_attn_norm", "post_ffn_norm"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
