"""GPU codec parity: w4a_pack / w4a_unpack / w4a_tile against the oracle,
bit for bit (integer and byte work), plus KV row copies."""
import numpy as np
import pytest
import torch

from oracle import quant
from w4_weight_only_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from w4_weight_only_b200 import api
    return api


def _as_u32(t):
    return t.cpu().numpy().view(np.uint32)


def _as_u16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("n,k", [(8, 128), (48, 1536), (768, 512), (7168, 5120), (5120, 27648)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_bit_exact(built_lib, cuda, n, k, dtype):
    api = _api()
    W, _ = synth.gemv_case(10, n, k, 1, "cpu")
    W = W.to(dtype)
    qw, sc, qz = api.pack(W.to(cuda))
    oqw, osb, oqz = quant.quantize_pack(W.to(torch.float32).numpy())
    assert np.array_equal(_as_u32(qw), oqw)
    assert np.array_equal(_as_u16(sc), osb)
    assert np.array_equal(_as_u32(qz), oqz)


def _special_matrix():
    r = np.random.default_rng(7)
    W = np.zeros((16, 768), np.float32)
    W[:, 0:128] = np.tile((np.arange(128) % 16) * 0.5, (16, 1))            # known pattern, s = 0.5
    q = r.integers(0, 16, size=(16, 128))
    q[:, 0], q[:, 1] = 0, 15
    W[:, 128:256] = (q - 8) * 0.25                                           # z = 8
    W[:, 256:384] = 3.0                                                      # constant group
    W[:, 384:512] = np.linspace(-1e6, 1e6, 128, dtype=np.float32)           # scale overflow
    W[:, 512:640] = np.float32(1.25) * (np.arange(128) % 3)                 # exact ties
    W[:, 640:768] = r.standard_normal((16, 128)).astype(np.float32) * 1e-30  # subnormal-range scale
    return W


def test_pack_special_groups(built_lib, cuda):
    api = _api()
    W = _special_matrix()
    qw, sc, qz = api.pack(torch.from_numpy(W).to(cuda))
    oqw, osb, oqz = quant.quantize_pack(W)
    assert np.array_equal(_as_u32(qw), oqw)
    assert np.array_equal(_as_u16(sc), osb)
    assert np.array_equal(_as_u32(qz), oqz)
    assert _as_u32(qw)[0, 0] == 0x76543210 and _as_u32(qw)[0, 1] == 0xFEDCBA98


@pytest.mark.parametrize("n,k", [(48, 1536), (7168, 5120)])
def test_unpack_exact(built_lib, cuda, n, k):
    api = _api()
    W, _ = synth.gemv_case(11, n, k, 1, "cpu")
    qw, sc, qz = api.pack(W.to(cuda))
    got = api.unpack_canonical(qw, sc, qz, n, k).cpu().numpy()
    ref = quant.dequantize(_as_u32(qw), _as_u16(sc), _as_u32(qz), n, k)
    assert np.array_equal(got.astype(np.float64), ref)


@pytest.mark.parametrize("n,k,inter", [(48, 1536, False), (64, 1024, True), (3072, 512, True), (5120, 27648, False)])
def test_tile_roundtrip_exact(built_lib, cuda, n, k, inter):
    api = _api()
    W, _ = synth.gemv_case(12, n, k, 1, "cpu")
    qw, sc, qz = api.pack(W.to(cuda))
    lin = api.tile(qw, sc, qz, n, k, row_interleave=inter)
    got = api.unpack_tiled(lin).cpu().numpy()
    ref = quant.dequantize(*quant.quantize_pack(W.numpy()), n, k)
    assert np.array_equal(got.astype(np.float64), ref)


def test_tile_bf16_layout(built_lib, cuda):
    """Reassemble the documented lm_head unit layout by hand and compare bits."""
    api = _api()
    n, k = 37, 256                                    # ragged rows: padded to 48 with zeros
    W = (torch.randn(n, k, generator=torch.Generator().manual_seed(3)) * 0.02).to(torch.bfloat16)
    blob = api.tile_bf16(W.to(cuda)).cpu().numpy().view(np.uint16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    nkc = k // 128
    full = np.zeros((48, k), np.uint16)
    full[:n] = Wb
    for rb in range(3):
        for kc in range(nkc):
            u = blob[(rb * nkc + kc) * 2048:(rb * nkc + kc + 1) * 2048].reshape(8, 32, 8)
            for s in range(8):
                for lane in range(32):
                    g, t = lane // 4, lane % 4
                    # k-step s = 2m + e of thread-in-quad t reads columns 32m + 8t + 4e .. +3
                    k0 = kc * 128 + 32 * (s // 2) + 8 * t + 4 * (s % 2)
                    r0, r1 = rb * 16 + g, rb * 16 + g + 8
                    want = [full[r0, k0], full[r0, k0 + 1], full[r1, k0], full[r1, k0 + 1],
                            full[r0, k0 + 2], full[r0, k0 + 3], full[r1, k0 + 2], full[r1, k0 + 3]]
                    assert list(u[s, lane]) == want


def test_tile_w4_layout(built_lib, cuda):
    """Reassemble the documented int4 unit layout by hand (codes, scales, zeros)."""
    api = _api()
    n, k = 32, 1024
    W, _ = synth.gemv_case(13, n, k, 1, "cpu")
    qw, sc, qz = api.pack(W.to(cuda))
    lin = api.tile(qw, sc, qz, n, k, row_interleave=False)
    blob = lin.blob.cpu().numpy().view(np.uint8)
    q, _, Z = quant.unpack(_as_u32(qw), _as_u16(sc), _as_u32(qz), n, k)   # codes [n, k], zeros [k/128, n]
    S = _as_u16(sc)                                                       # fp16 bits [k/128, n]
    nkc = k // 512
    for rb in range(n // 16):
        for kc in range(nkc):
            u = blob[(rb * nkc + kc) * 4256:(rb * nkc + kc + 1) * 4256]
            words = u[:4096].view(np.uint32).reshape(8, 32, 4)      # [s // 4][lane][s % 4]
            for s in range(32):
                for lane in range(32):
                    g, t = lane // 4, lane % 4
                    c = kc * 512 + 32 * (s // 2) + 8 * t + 4 * (s % 2)
                    r0, r1 = rb * 16 + g, rb * 16 + g + 8
                    # nibble j: row (j odd ? r1 : r0), column c + (2 if j & 2) + (1 if j & 4)
                    want = 0
                    for j in range(8):
                        r = r1 if j & 1 else r0
                        cc = c + (2 if j & 2 else 0) + (1 if j & 4 else 0)
                        want |= int(q[r, cc]) << (4 * j)
                    assert int(words[s // 4, lane, s % 4]) == want
            scales = u[4096:4224].view(np.uint16).reshape(8, 4, 2)   # [row % 8][group][row / 8]
            zeros = u[4224:4256].view(np.uint32).reshape(4, 2)       # [group][row / 8], nibble row % 8
            for grp in range(4):
                gi = kc * 4 + grp
                for i in range(16):
                    row = rb * 16 + i
                    assert scales[i % 8, grp, i // 8] == S[gi, row]
                    assert (int(zeros[grp, i // 8]) >> (4 * (i % 8))) & 15 == int(Z[gi, row])


def test_kv_write_read_roundtrip(built_lib, cuda):
    api = _api()
    from w4_weight_only_b200 import config
    cfg = config.tiny()
    kv = api.KVCache(cfg, 2, 96)
    for layer in (0, 3):
        k, v = synth.kv_rows(5, layer, 1, cfg.n_kv_heads, 40, cfg.head_dim, "cpu")
        kv.write(layer, 1, 17, k.to(cuda), v.to(cuda))
        k2, v2 = kv.read(layer, 1, 17, 40)
        assert torch.equal(k2.cpu(), k) and torch.equal(v2.cpu(), v)
        # documented storage order: chunk c of slot s sits at chunk c ^ (s & 7)
        kc, _ = kv.layer_views(layer)
        s, d = 17 + 5, 19
        raw = kc[1, 0, s].cpu()
        assert raw[((d // 8) ^ (s & 7)) * 8 + d % 8].item() == k[0, 5, d].item()
