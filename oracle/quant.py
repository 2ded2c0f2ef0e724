"""Oracle: int4 weight-only quantization, canonical packing and dequantization.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Source: ATLAS-OLMo-3-32B-Think-v4 model card, section "Quantization recipe":
weights are stored 4 bits per value, packed eight to a 32-bit word with
column j of a row landing in word j // 8, little-endian nibble order (nibble
j % 8 occupies bits 4*(j % 8) .. 4*(j % 8) + 3), rows being output channels
(the kernel there walks one row per warp).  The page's checkpoint is symmetric
with a fixed stored offset of 8; the format this library implements is the
asymmetric group-128 variant with an fp16 scale and a 4-bit zero per
(row, group), dequantized as w = (q - z) * s.  With z == 8 for every group the
two coincide, which the tests check.

The page's own checkpoint format (symmetric, group 32, bf16 scales, stored
nibble q + 8, no zero points) is dequantized by ``dequantize_sym32``: the same
packing, w = (nibble - 8) * s with s the bf16 scale of (row, 32-column
group).  Its scales come from an MSE observer and AWQ's search, which need
calibration data; checkpoints of this format are therefore taken as given
(seeded random nibbles and scales), not produced here.

Readings taken where the pages are silent:

* The page's AWQ scale search needs calibration data and trained weights; the
  quantizer here is round-to-nearest min/max asymmetric (reading D1).
* Scales are laid out [K/group, N] in fp16; zeros are packed eight rows to a
  word along N, [K/group, N/8], same nibble order as the weights (D3).
* A group whose max equals its min gets the smallest fp16 subnormal 2**-24 as
  its scale (D4); a scale above the fp16 range is clamped to 65504.
* The code decision is taken in IEEE binary32 arithmetic, each operation
  rounded to nearest-even, so that it is reproducible bit for bit by a CUDA
  kernel that uses correctly rounded fp32 division and ``rintf``.

Parity status: pinned (known-pattern words, nearest-code brute force, error
bound, idempotence, degenerate group, the z == 8 special case).
"""
from __future__ import annotations

import numpy as np

FP16_MAX = np.float16(65504.0)
FP16_MIN_SUBNORMAL = np.float16(2.0 ** -24)


def quantize(W, group: int = 128):
    """Quantize a float32 matrix W [N, K] group-wise along K.

    Per (row n, group g) of ``group`` consecutive columns, in binary32:
        mn, mx = min, max of the group
        s32    = fl32(fl32(mx - mn) / 15)
        s      = fp16(s32) (nearest-even; 0 -> 2**-24; overflow -> 65504)
        z      = clamp(rint(fl32(-mn / s)), 0, 15)
        q      = clamp(rint(fl32(w / s)) + z, 0, 15)
    Returns (codes uint8 [N, K], scales float16 [K/group, N], zeros uint8 [K/group, N]).
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = W.reshape(N, K // group, group)
    mn = G.min(axis=2)
    mx = G.max(axis=2)
    rng = np.subtract(mx, mn, dtype=np.float32)
    s32 = np.divide(rng, np.float32(15.0), dtype=np.float32)
    with np.errstate(over="ignore"):
        s16 = s32.astype(np.float16)
    s16 = np.where(np.isinf(s16), FP16_MAX, s16)
    s16 = np.where(s16 == 0, FP16_MIN_SUBNORMAL, s16).astype(np.float16)
    s = s16.astype(np.float32)
    zf = np.rint(np.divide(-mn, s, dtype=np.float32))
    z = np.clip(zf, 0, 15).astype(np.int64)
    r = np.rint(np.divide(G, s[:, :, None], dtype=np.float32)).astype(np.int64)
    q = np.clip(r + z[:, :, None], 0, 15)
    codes = q.reshape(N, K).astype(np.uint8)
    return codes, np.ascontiguousarray(s16.T), np.ascontiguousarray(z.T.astype(np.uint8))


def pack_rows(codes):
    """Pack 4-bit values [R, C] (C % 8 == 0) eight per uint32 along C.

    Value at column j goes to word j // 8, bits 4*(j % 8) .. +3.
    """
    codes = np.asarray(codes, dtype=np.uint32)
    R, C = codes.shape
    if C % 8:
        raise ValueError("packed dimension must be a multiple of 8")
    c = codes.reshape(R, C // 8, 8)
    words = np.zeros((R, C // 8), dtype=np.uint32)
    for j in range(8):
        words |= (c[:, :, j] & np.uint32(0xF)) << np.uint32(4 * j)
    return words


def unpack_rows(words, C: int):
    """Inverse of ``pack_rows``: uint32 [R, C/8] -> uint8 [R, C]."""
    words = np.asarray(words, dtype=np.uint32)
    R = words.shape[0]
    out = np.zeros((R, C // 8, 8), dtype=np.uint8)
    for j in range(8):
        out[:, :, j] = (words >> np.uint32(4 * j)) & np.uint32(0xF)
    return out.reshape(R, C)


def pack(codes, scales16, zeros):
    """Canonical storage: qweight uint32 [N, K/8], scales uint16 (fp16 bits)
    [K/g, N], qzeros uint32 [K/g, N/8]."""
    qweight = pack_rows(codes)
    sbits = np.ascontiguousarray(np.asarray(scales16, dtype=np.float16)).view(np.uint16)
    qzeros = pack_rows(zeros)
    return qweight, sbits, qzeros


def quantize_pack(W, group: int = 128):
    """quantize() followed by pack(): the canonical triple for W [N, K]."""
    return pack(*quantize(W, group))


def unpack(qweight, scales_bits, qzeros, N: int, K: int, group: int = 128):
    """Canonical triple -> (codes [N, K] uint8, scales float16 [K/g, N], zeros uint8 [K/g, N])."""
    codes = unpack_rows(qweight, K)
    s16 = np.asarray(scales_bits, dtype=np.uint16).view(np.float16).reshape(K // group, N)
    z = unpack_rows(qzeros, N)
    return codes, s16, z


def dequantize(qweight, scales_bits, qzeros, N: int, K: int, group: int = 128):
    """Exact dequantized matrix W~[n, k] = (q - z) * s as float64 [N, K].

    (q - z) is an integer in [-15, 15] and s an fp16 value, so the product is
    exact in float64 (and in float32).
    """
    codes, s16, z = unpack(qweight, scales_bits, qzeros, N, K, group)
    s = s16.astype(np.float64).T            # [N, K/g]
    zz = z.astype(np.int64).T               # [N, K/g]
    q = codes.astype(np.int64).reshape(N, K // group, group)
    w = (q - zz[:, :, None]).astype(np.float64) * s[:, :, None]
    return w.reshape(N, K)


def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> their exact values as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def dequantize_sym32(qweight, scale_bits, N: int, K: int, group: int = 32):
    """The model card's checkpoint format ("Quantization recipe": symmetric,
    no zero points, group 32, stored nibble q + 8, bf16 scales).

    qweight uint32 [N, K/8] packed as ``pack_rows`` packs; scale_bits bf16
    bits [N, K/group] (one scale per output row and group of inputs).
    Returns the exact float64 W~[n, k] = (nibble - 8) * s[n, k // group]."""
    nib = unpack_rows(qweight, K).astype(np.int64)
    s = bf16_bits_to_f64(scale_bits).reshape(N, K // group)
    w = (nib - 8).reshape(N, K // group, group).astype(np.float64) * s[:, :, None]
    return w.reshape(N, K)
