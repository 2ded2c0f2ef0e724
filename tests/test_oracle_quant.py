"""Pins for the oracle's int4 quantizer, packing and dequantization (CPU only).

Each check ties the oracle to something other than itself: the packing order
printed on the model card ("Quantization recipe"), the nearest-code property
of round-to-nearest (brute force over all 16 codes), the error bound, the
symmetric special case z = 8, and closed-form degenerate groups.
"""
import json
from pathlib import Path

import numpy as np
import pytest

from oracle import quant

GOLD = Path(__file__).parent / "golden"


def _rng(seed):
    return np.random.default_rng(seed)


def test_known_pattern_words():
    gold = json.loads((GOLD / "known_pattern_words.json").read_text())
    want = [int(w, 16) for w in gold["codes_k_mod_16_words"]]
    K = 256
    # codes q = k % 16 arise from a group spanning [0, 7.5] in steps of 0.5:
    # s = 7.5 / 15 = 0.5 exactly, z = 0.
    W = np.tile((np.arange(K) % 16) * 0.5, (8, 1)).astype(np.float32)
    codes, s16, z = quant.quantize(W)
    assert np.all(codes == (np.arange(K) % 16)[None, :])
    assert np.all(s16.astype(np.float32) == 0.5) and np.all(z == 0)
    qw, _, _ = quant.pack(codes, s16, z)
    assert qw.dtype == np.uint32 and qw.shape == (8, K // 8)
    for row in qw:
        assert list(row) == want * (K // 16)


def test_pack_unpack_roundtrip():
    r = _rng(1)
    codes = r.integers(0, 16, size=(24, 384)).astype(np.uint8)
    assert np.array_equal(quant.unpack_rows(quant.pack_rows(codes), 384), codes)
    # nibble j of word w is column 8w + j
    words = quant.pack_rows(codes)
    assert (int(words[3, 5]) >> 4 * 6) & 15 == codes[3, 8 * 5 + 6]


def test_symmetric_special_case_z8():
    """A group spanning exactly [-8 s, 7 s] gets z = 8, so w~ = (q - 8) s: the
    pages' symmetric format with stored nibble q + 8."""
    r = _rng(2)
    s = np.float32(0.25)
    q = r.integers(0, 16, size=(16, 128))
    q[:, 0], q[:, 1] = 0, 15
    W = ((q - 8) * s).astype(np.float32)
    codes, s16, z = quant.quantize(W)
    assert np.all(z == 8)
    assert np.all(s16.astype(np.float32) == s)
    assert np.array_equal(codes, q.astype(np.uint8))
    qw, sb, qz = quant.pack(codes, s16, z)
    assert np.array_equal(quant.dequantize(qw, sb, qz, 16, 128), W.astype(np.float64))


def test_nearest_code_brute_force():
    """Every unclamped code is a nearest grid point (q - z) s to w among all 16."""
    r = _rng(3)
    W = (r.standard_normal((32, 256)) * 0.02).astype(np.float32)
    codes, s16, z = quant.quantize(W)
    s = s16.astype(np.float64).T          # [N, G]
    zz = z.astype(np.float64).T
    grid = (np.arange(16)[None, None, :] - zz[:, :, None]) * s[:, :, None]   # [N, G, 16]
    w = W.astype(np.float64).reshape(32, 2, 128)
    c = codes.reshape(32, 2, 128).astype(np.int64)
    err_chosen = np.abs(w - np.take_along_axis(grid, c, axis=2))
    err_best = np.min(np.abs(w[..., None] - grid[:, :, None, :]), axis=3)
    # ties at exactly half a step may go either way under round-half-even
    assert np.all(err_chosen <= err_best + 1e-6 * s[:, :, None])


def test_error_bound_and_scale():
    r = _rng(4)
    W = (r.standard_normal((16, 512)) * 0.02).astype(np.float32)
    codes, s16, z = quant.quantize(W)
    qw, sb, qz = quant.pack(codes, s16, z)
    Wt = quant.dequantize(qw, sb, qz, 16, 512)
    s = np.repeat(s16.astype(np.float64).T, 128, axis=1)
    unclamped = (codes > 0) & (codes < 15)
    assert np.all(np.abs(W - Wt)[unclamped] <= 0.5 * s[unclamped] * (1 + 1e-6))
    # the scale is (max - min) / 15 up to fp32 and fp16 rounding
    G = W.reshape(16, 4, 128)
    rng = (G.max(axis=2) - G.min(axis=2)) / 15.0
    assert np.allclose(s16.astype(np.float64).T, rng, rtol=2 ** -10)


def test_idempotent_on_full_range_groups():
    r = _rng(5)
    W = (r.standard_normal((16, 256)) * 0.02).astype(np.float32)
    codes, s16, z = quant.quantize(W)
    qw, sb, qz = quant.pack(codes, s16, z)
    Wt = quant.dequantize(qw, sb, qz, 16, 256).astype(np.float32)
    codes2, s2, z2 = quant.quantize(Wt)
    full = (codes.reshape(16, 2, 128).min(axis=2) == 0) & (codes.reshape(16, 2, 128).max(axis=2) == 15)
    assert full.sum() > 10
    assert np.array_equal(s2.T[full], s16.T[full]) and np.array_equal(z2.T[full], z.T[full])
    assert np.array_equal(codes2.reshape(16, 2, 128)[full], codes.reshape(16, 2, 128)[full])


def test_degenerate_and_overflow_groups():
    W = np.zeros((8, 384), dtype=np.float32)
    W[:, 128:256] = 3.0        # constant positive group
    W[:, 256:384] = np.linspace(-1e6, 1e6, 128, dtype=np.float32)   # range beyond fp16
    codes, s16, z = quant.quantize(W)
    sbits = s16.view(np.uint16)
    assert np.all(sbits[0] == 0x0001) and np.all(sbits[1] == 0x0001)   # 2**-24
    assert np.all(s16[2].astype(np.float32) == 65504.0)
    assert np.all(z[0] == 0) and np.all(codes[:, :128] == 0)            # zero group -> exact zeros
    assert np.all(z[1] == 0) and np.all(codes[:, 128:256] == 15)        # clamped
    qw, sb, qz = quant.pack(codes, s16, z)
    Wt = quant.dequantize(qw, sb, qz, 8, 384)
    assert np.all(Wt[:, :128] == 0.0)


def test_dequant_exact_in_fp32():
    r = _rng(6)
    W = (r.standard_normal((8, 256)) * 0.02).astype(np.float32)
    qw, sb, qz = quant.quantize_pack(W)
    Wt = quant.dequantize(qw, sb, qz, 8, 256)
    assert np.array_equal(Wt.astype(np.float32).astype(np.float64), Wt)


def test_rounding_half_even_in_fp32():
    """Code decisions use binary32 division and ties-to-even: w / s = 2.5 -> 2."""
    s = np.float32(0.5)
    row = np.zeros(128, np.float32)
    row[0], row[1] = 0.0, 7.5           # min 0, max 7.5 -> s = 0.5, z = 0
    row[2] = 1.25                       # 2.5 steps -> 2
    row[3] = 1.75                       # 3.5 steps -> 4
    codes, s16, z = quant.quantize(row[None, :])
    assert s16[0, 0] == s and z[0, 0] == 0
    assert codes[0, 2] == 2 and codes[0, 3] == 4


# ---- the model card's symmetric group-32 checkpoint format -----------------------
def _bf16_bits(x):
    """Round float32 values to bf16 (nearest-even) and return the bits."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def test_sym32_known_pattern_and_offset():
    """Stored nibbles k % 16 (the page's packing: column j in word j / 8,
    nibble j % 8) decode to q = k % 16 - 8, from -8 to 7."""
    gold = json.loads((GOLD / "known_pattern_words.json").read_text())
    want = [int(w, 16) for w in gold["codes_k_mod_16_words"]]
    K = 64
    qw = quant.pack_rows(np.tile(np.arange(K) % 16, (2, 1)))
    assert list(qw[0][:2]) == want
    s = _bf16_bits(np.full((2, K // 32), 0.5, np.float32))
    w = quant.dequantize_sym32(qw, s, 2, K)
    assert np.array_equal(w[0], ((np.arange(K) % 16) - 8) * 0.5)
    assert w.min() == -4.0 and w.max() == 3.5


def test_sym32_equals_asymmetric_with_zero_8():
    """The symmetric format is the asymmetric dequantization with every zero
    point 8 and group 32 (scales that fp16 holds exactly)."""
    r = _rng(11)
    N, K = 16, 256
    codes = r.integers(0, 16, size=(N, K))
    qw = quant.pack_rows(codes)
    sf = (r.random((N, K // 32)) * 0.01 + 1e-3).astype(np.float32)
    sb = _bf16_bits(sf)
    sv = quant.bf16_bits_to_f64(sb)
    s16 = sv.astype(np.float16)
    assert np.array_equal(s16.astype(np.float64), sv)  # bf16 values in the fp16 range are fp16 values
    zeros = quant.pack_rows(np.full((K // 32, N), 8))
    asym = quant.dequantize(qw, np.ascontiguousarray(s16.T).view(np.uint16), zeros, N, K, group=32)
    assert np.array_equal(quant.dequantize_sym32(qw, sb, N, K), asym)


def test_sym32_brute_force():
    r = _rng(12)
    N, K = 3, 64
    codes = r.integers(0, 16, size=(N, K))
    sb = _bf16_bits(r.random((N, K // 32)).astype(np.float32))
    w = quant.dequantize_sym32(quant.pack_rows(codes), sb, N, K)
    for n in range(N):
        for k in range(K):
            bits = int(sb[n, k // 32]) << 16
            s = float(np.array([bits], dtype=np.uint32).view(np.float32)[0])
            assert w[n, k] == (int(codes[n, k]) - 8) * s
