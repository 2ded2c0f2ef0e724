"""The model card's own checkpoint format on the GPU: symmetric int4, group 32,
bf16 scales, stored nibble q + 8 (ATLAS-OLMo-3-32B-Think-v4 model card,
"Quantization recipe"), ingested as stored and compared with the oracle's
reading of the format (``oracle.quant.dequantize_sym32``).

* tiling into the kernel's group-32 units and unpacking: bit-exact (the
  product of a 4-bit integer and a bf16 scale is exact in fp32);
* the decode GEMV (the engine's group-32 unit: q - 8 formed in fp16 exactly,
  every 32-column group closed with its scale): 2e-3 * RMS(y_ref), as for the
  group-128 format; the SwiGLU epilogue element-wise;
* the prefill GEMM on these weights (expanded to fp16): 3e-3 * RMS;
* a decode step of the small decoder (prompt prefill, then greedy steps) and
  of a two-layer model of the full 32B shape at 4,096 cached positions: the
  residual after every layer within 2e-2 * RMS, logits within 3e-2.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import quant
from w4_weight_only_b200 import config as wc
from w4_weight_only_b200 import synth
from helpers import Sym32Pair, max_rel_to_rms, np64

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3
GEMM_TOL = 3e-3
HID_TOL = 2e-2
LOGIT_TOL = 3e-2


def _api():
    from w4_weight_only_b200 import api, _abi
    return api, _abi


def _oracle_dense(qw, sc):
    n, k = qw.shape[0], qw.shape[1] * 8
    return quant.dequantize_sym32(qw.cpu().numpy().view(np.uint32), sc.cpu().view(torch.int16).numpy().view(np.uint16),
                                  n, k)


@pytest.mark.parametrize("n,k,inter", [(16, 256, False), (768, 512, False), (3072, 512, True), (512, 1536, False),
                                       (5120, 27648, False), (55296, 5120, True)])
def test_tile_unpack_bit_exact(built_lib, cuda, n, k, inter):
    api, _ = _api()
    qw, sc = synth.sym32_matrix(80, n, k, "cuda")
    ref = _oracle_dense(qw, sc)
    assert np.array_equal(api.unpack_sym32(qw, sc).cpu().numpy().astype(np.float64), ref)
    lin = api.tile_sym32(qw, sc, row_interleave=inter)
    assert lin.nbytes == (n // 16) * (k // 256) * 2304
    assert np.array_equal(api.unpack_tiled(lin).cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("n,k", [(768, 512), (1024, 1536), (7168, 5120), (5120, 5120), (5120, 27648)])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_gemv_sym32(built_lib, cuda, n, k, batch):
    api, _ = _api()
    qw, sc = synth.sym32_matrix(81, n, k, "cuda")
    x = synth.normal((batch, k), "cuda", 1.0, 0.0, 81, "sym32_x", n, k, batch).to(torch.bfloat16)
    lin = api.tile_sym32(qw, sc)
    ws = api.gemv_workspace(lin, batch)
    y = api.gemv(lin, x, ws=ws).cpu().numpy()
    api.check(ws)
    ref = np64(x) @ _oracle_dense(qw, sc).T
    assert max_rel_to_rms(y, ref) <= GEMV_TOL


@pytest.mark.parametrize("ffn,k,batch", [(1536, 512, 3), (27648, 5120, 1)])
def test_gemv_sym32_silu(built_lib, cuda, ffn, k, batch):
    api, abi = _api()
    qw, sc = synth.sym32_matrix(82, 2 * ffn, k, "cuda")
    x = synth.normal((batch, k), "cuda", 1.0, 0.0, 82, "sym32_x", ffn, k, batch).to(torch.bfloat16)
    lin = api.tile_sym32(qw, sc, row_interleave=True)
    h = api.gemv(lin, x, epilogue=abi.EPI_SILU_MUL).float().cpu().numpy()
    gu = np64(x) @ _oracle_dense(qw, sc).T
    ref = gu[:, :ffn] / (1.0 + np.exp(-gu[:, :ffn])) * gu[:, ffn:]
    slack = 1e-3 * np.sqrt(np.mean(ref * ref))
    assert np.all(np.abs(h - ref) <= 2.0 ** -8 * np.abs(ref) + slack)


@pytest.mark.parametrize("n,k,M", [(768, 512, 77), (7168, 5120, 300)])
def test_gemm_sym32(built_lib, cuda, n, k, M):
    api, _ = _api()
    qw, sc = synth.sym32_matrix(83, n, k, "cuda")
    x = synth.normal((M, k), "cuda", 1.0, 0.0, 83, "sym32_gx", M, k).to(torch.float16)
    lin = api.tile_sym32(qw, sc)
    ws = api.gemm_workspace(lin)
    y = api.gemm(lin, x, ws=ws).cpu().numpy()
    api.check(ws)
    ref = np64(x) @ _oracle_dense(qw, sc).T
    err = np.abs(y - ref) / np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    assert float(err.max()) <= GEMM_TOL


def _check(cfg, lg, dump, ref_lg, ref_hid, what):
    for l in range(cfg.n_layers + 1):
        assert max_rel_to_rms(dump[l], ref_hid[l]) <= HID_TOL, (what, l)
    assert float(np.max(np.abs(lg - ref_lg))) <= LOGIT_TOL, what


def test_decode_sym32_tiny(built_lib, cuda):
    """The small decoder with group-32 weights: a 40-token prompt (the dense
    prefill), then 4 greedy steps checked layer by layer."""
    from w4_weight_only_b200 import api
    cfg = wc.tiny()
    cfg.group = 32
    P = Sym32Pair(cfg, seed=6)
    prompt = synth.token_ids(6, 40, cfg.vocab, "cpu")
    kv = api.KVCache(cfg, 1, 64)
    okv = om.OracleKV(P.ocfg, 1, 64)
    last = P.gpu.prefill(kv, prompt.to("cuda"))
    ref_last = om.prefill(P.oracle, okv, prompt.numpy())
    P.gpu.check()
    assert float(np.max(np.abs(last.cpu().numpy() - ref_last))) <= LOGIT_TOL
    tok = int(np.argmax(ref_last))
    for step in range(4):
        pos = 40 + step
        dump = torch.zeros((cfg.n_layers + 1, 1, cfg.d_model), dtype=torch.float32, device="cuda")
        lg, _ = P.gpu.decode_step(kv, torch.tensor([tok], dtype=torch.int32, device="cuda"),
                                  torch.tensor([pos], dtype=torch.int32, device="cuda"), hidden_dump=dump)
        ref_lg, ref_hid = om.decode_step(P.oracle, okv, [tok], [pos])
        P.gpu.check()
        _check(cfg, lg[0].cpu().numpy(), dump[:, 0].cpu().numpy(), ref_lg[0], ref_hid[:, 0], f"step {step}")
        tok = int(om.argmax(ref_lg[0]))


def test_decode_sym32_32b_shape(built_lib, cuda):
    """Two layers of the full 32B shape (sliding-window, then full with YaRN)
    in the group-32 format, batch 1, 4,096 cached positions."""
    from w4_weight_only_b200 import api
    cfg = wc.olmo3_32b(2)
    cfg.full_layers = [False, True]
    cfg.group = 32
    P = Sym32Pair(cfg, seed=7, gen_device="cuda")
    ctx = 4096
    kv = api.KVCache(cfg, 1, ctx + 16)
    okv = om.OracleKV(P.ocfg, 1, ctx + 16)
    for l in range(cfg.n_layers):
        k, v = synth.kv_rows(7, l, 0, cfg.n_kv_heads, ctx, cfg.head_dim, "cuda")
        kv.fill_history(l, 0, k, v)
        okv.fill(l, 0, 0, k.cpu().double().numpy(), v.cpu().double().numpy())
    tok = int(synth.token_ids(7, 1, cfg.vocab, "cpu")[0])
    dump = torch.zeros((cfg.n_layers + 1, 1, cfg.d_model), dtype=torch.float32, device="cuda")
    lg, nxt = P.gpu.decode_step(kv, torch.tensor([tok], dtype=torch.int32, device="cuda"),
                                torch.tensor([ctx], dtype=torch.int32, device="cuda"), hidden_dump=dump)
    ref_lg, ref_hid = om.decode_step(P.oracle, okv, [tok], [ctx])
    P.gpu.check()
    _check(cfg, lg[0].cpu().numpy(), dump[:, 0].cpu().numpy(), ref_lg[0], ref_hid[:, 0], "32b sym32")
    top2 = np.sort(ref_lg[0])[-2:]
    if top2[1] - top2[0] >= 2 * LOGIT_TOL:
        assert int(nxt[0]) == int(np.argmax(ref_lg[0]))
