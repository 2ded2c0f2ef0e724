"""Torch-facing binding of libw4a: argument marshalling only.

Every function here checks dtypes/devices, passes raw device pointers and the
current CUDA stream through ctypes, and returns torch tensors that own the
outputs.  All arithmetic runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes as C
from typing import Dict, List, Optional, Sequence

import torch

from . import _abi
from ._abi import call
from .config import Config


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def _size_out(fn, *args) -> int:
    out = C.c_size_t(0)
    call(fn, *args, C.byref(out))
    return out.value


def zeros_workspace(nbytes: int, device=None) -> torch.Tensor:
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------------------
# int4 codec
# ---------------------------------------------------------------------------
def pack(W: torch.Tensor, group: int = 128):
    """Quantize W [n, k] (fp32 or bf16, CUDA) -> canonical (qweight int32 [n, k/8],
    scales int16 fp16-bits [k/g, n], qzeros int32 [k/g, n/8])."""
    if W.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("pack: W must be float32 or bfloat16")
    _need(W, W.dtype, "W")
    n, k = W.shape
    dev = W.device
    qw = torch.empty((n, k // 8), dtype=torch.int32, device=dev)
    sc = torch.empty((k // group, n), dtype=torch.int16, device=dev)
    qz = torch.empty((k // group, n // 8), dtype=torch.int32, device=dev)
    call("w4a_pack", _p(W), _abi.F32 if W.dtype == torch.float32 else _abi.BF16, n, k, group,
         _p(qw), _p(sc), _p(qz), _stream())
    return qw, sc, qz


def canonical(qw, sc, qz, n: int, k: int, group: int = 128) -> _abi.W4ATensor:
    t = _abi.W4ATensor()
    t.n, t.k, t.group, t.layout, t.row_interleave = n, k, group, _abi.LAYOUT_CANONICAL, 0
    t.qweight, t.scales, t.qzeros = qw.data_ptr(), sc.data_ptr(), qz.data_ptr()
    return t


class W4Linear:
    """An int4 matrix in the kernel (tiled) layout; owns its device buffer."""

    def __init__(self, blob: torch.Tensor, n: int, k: int, row_interleave: bool, group: int = 128):
        self.blob, self.n, self.k, self.row_interleave, self.group = blob, n, k, row_interleave, group

    def tensor(self) -> _abi.W4ATensor:
        t = _abi.W4ATensor()
        t.n, t.k, t.group, t.layout = self.n, self.k, self.group, _abi.LAYOUT_TILED
        t.row_interleave = 1 if self.row_interleave else 0
        t.qweight = self.blob.data_ptr()
        return t

    @property
    def nbytes(self) -> int:
        return self.blob.numel()


def tile(qw, sc, qz, n: int, k: int, row_interleave: bool = False, group: int = 128) -> W4Linear:
    nbytes = _size_out("w4a_tiled_bytes", n, k, group)
    blob = torch.empty(nbytes, dtype=torch.uint8, device=qw.device)
    can = canonical(qw, sc, qz, n, k, group)
    call("w4a_tile", C.byref(can), 1 if row_interleave else 0, _p(blob), nbytes, _stream())
    return W4Linear(blob, n, k, row_interleave, group)


def tile_sym32(qweight: torch.Tensor, scales: torch.Tensor, row_interleave: bool = False) -> W4Linear:
    """The model card's checkpoint format (symmetric int4, group 32, stored
    nibble q + 8): qweight int32 [n, k/8], scales bf16 [n, k/32], as stored,
    rewritten into the kernel's group-32 units."""
    _need(qweight, torch.int32, "qweight")
    _need(scales, torch.bfloat16, "scales")
    n, k = qweight.shape[0], qweight.shape[1] * 8
    nbytes = _size_out("w4a_tiled_bytes", n, k, 32)
    blob = torch.empty(nbytes, dtype=torch.uint8, device=qweight.device)
    t = _abi.W4ATensor()
    t.n, t.k, t.group, t.layout, t.row_interleave = n, k, 32, _abi.LAYOUT_SYM32, 0
    t.qweight, t.scales, t.qzeros = qweight.data_ptr(), scales.data_ptr(), None
    call("w4a_tile", C.byref(t), 1 if row_interleave else 0, _p(blob), nbytes, _stream())
    return W4Linear(blob, n, k, row_interleave, 32)


def unpack_sym32(qweight: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """Exact fp32 dequantization of a symmetric group-32 checkpoint matrix."""
    n, k = qweight.shape[0], qweight.shape[1] * 8
    out = torch.empty((n, k), dtype=torch.float32, device=qweight.device)
    t = _abi.W4ATensor()
    t.n, t.k, t.group, t.layout, t.row_interleave = n, k, 32, _abi.LAYOUT_SYM32, 0
    t.qweight, t.scales, t.qzeros = qweight.data_ptr(), scales.data_ptr(), None
    call("w4a_unpack", C.byref(t), _p(out), _stream())
    return out


def quantize_linear(W: torch.Tensor, row_interleave: bool = False, group: int = 128) -> W4Linear:
    """pack() then tile(): the kernel-layout int4 form of W [n, k]."""
    n, k = W.shape
    qw, sc, qz = pack(W, group)
    return tile(qw, sc, qz, n, k, row_interleave, group)


def unpack_canonical(qw, sc, qz, n: int, k: int, group: int = 128) -> torch.Tensor:
    out = torch.empty((n, k), dtype=torch.float32, device=qw.device)
    can = canonical(qw, sc, qz, n, k, group)
    call("w4a_unpack", C.byref(can), _p(out), _stream())
    return out


def unpack_tiled(lin: W4Linear) -> torch.Tensor:
    out = torch.empty((lin.n, lin.k), dtype=torch.float32, device=lin.blob.device)
    t = lin.tensor()
    call("w4a_unpack", C.byref(t), _p(out), _stream())
    return out


def tile_bf16(W: torch.Tensor) -> torch.Tensor:
    _need(W, torch.bfloat16, "W")
    n, k = W.shape
    nbytes = _size_out("w4a_tiled_bf16_bytes", n, k)
    blob = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    call("w4a_tile_bf16", _p(W), n, k, _p(blob), nbytes, _stream())
    return blob


# ---------------------------------------------------------------------------
# GEMV
# ---------------------------------------------------------------------------
def gemv_workspace(lin: W4Linear, batch: int) -> torch.Tensor:
    t = lin.tensor()
    return zeros_workspace(_size_out("w4a_gemv_workspace_bytes", C.byref(t), batch), lin.blob.device)


def gemv(lin: W4Linear, x: torch.Tensor, epilogue: int = _abi.EPI_NONE, ws: Optional[torch.Tensor] = None,
         out: Optional[torch.Tensor] = None, aux: Optional[torch.Tensor] = None):
    """y = W~ x for x bf16 [B, k].  Returns out (and aux for EPI_SUMSQ)."""
    _need(x, torch.bfloat16, "x")
    B = x.shape[0]
    if x.shape[1] != lin.k:
        raise ValueError("x has the wrong width")
    if ws is None:
        ws = gemv_workspace(lin, B)
    if out is None:
        if epilogue == _abi.EPI_SILU_MUL:
            out = torch.empty((B, lin.n // 2), dtype=torch.bfloat16, device=x.device)
        else:
            out = torch.empty((B, lin.n), dtype=torch.float32, device=x.device)
    if epilogue == _abi.EPI_SUMSQ and aux is None:
        aux = torch.empty((lin.n // 16, B), dtype=torch.float32, device=x.device)
    t = lin.tensor()
    call("w4a_gemv", C.byref(t), _p(x), B, _p(out), epilogue, _p(aux), _p(ws), ws.numel(), _stream())
    return (out, aux) if epilogue == _abi.EPI_SUMSQ else out


def gemv_noalloc(lin: W4Linear, x: torch.Tensor, epilogue: int = _abi.EPI_NONE,
                 out: Optional[torch.Tensor] = None, aux: Optional[torch.Tensor] = None):
    """As gemv(), with the library's fixed scratch instead of a workspace
    (w4a_gemv_noalloc): calls must not overlap in time."""
    _need(x, torch.bfloat16, "x")
    B = x.shape[0]
    if x.shape[1] != lin.k:
        raise ValueError("x has the wrong width")
    if out is None:
        if epilogue == _abi.EPI_SILU_MUL:
            out = torch.empty((B, lin.n // 2), dtype=torch.bfloat16, device=x.device)
        else:
            out = torch.empty((B, lin.n), dtype=torch.float32, device=x.device)
    if epilogue == _abi.EPI_SUMSQ and aux is None:
        aux = torch.empty((lin.n // 16, B), dtype=torch.float32, device=x.device)
    t = lin.tensor()
    call("w4a_gemv_noalloc", C.byref(t), _p(x), B, _p(out), epilogue, _p(aux), _stream())
    return (out, aux) if epilogue == _abi.EPI_SUMSQ else out


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def attn_workspace(batch: int, n_heads: int, n_kv_heads: int, head_dim: int, device=None) -> torch.Tensor:
    return zeros_workspace(_size_out("w4a_attn_workspace_bytes", batch, n_heads, n_kv_heads, head_dim), device)


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, n_kv_heads: int, slots: int,
                pos: torch.Tensor, window: int = 0, ws: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """GQA decode attention; q bf16 [B, n_heads, hd] already normed and rotated."""
    _need(q, torch.bfloat16, "q")
    _need(pos, torch.int32, "pos")
    B, nq, hd = q.shape
    if ws is None:
        ws = attn_workspace(B, nq, n_kv_heads, hd, q.device)
    if out is None:
        out = torch.empty_like(q)
    call("w4a_attn_decode", _p(q), _p(k_cache), _p(v_cache), B, nq, n_kv_heads, hd, slots, _p(pos), window,
         _p(out), _p(ws), ws.numel(), _stream())
    return out


def qk_prep(cfg: Config, full: bool, q_raw, k_raw, v_raw, q_gain, k_gain, pos, k_cache, v_cache, slots: int):
    for name, t in (("q_raw", q_raw), ("k_raw", k_raw), ("v_raw", v_raw), ("q_gain", q_gain), ("k_gain", k_gain)):
        _need(t, torch.float32, name)
    _need(pos, torch.int32, "pos")
    B = q_raw.shape[0]
    q_out = torch.empty((B, cfg.n_heads, cfg.head_dim), dtype=torch.bfloat16, device=q_raw.device)
    c = cfg.to_c()
    call("w4a_qk_prep", C.byref(c), 1 if full else 0, _p(q_raw), _p(k_raw), _p(v_raw), _p(q_gain), _p(k_gain),
         _p(pos), B, _p(q_out), _p(k_cache), _p(v_cache), slots, _stream())
    return q_out


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------
class KVCache:
    """One zero-filled device allocation holding every layer's K and V."""

    def __init__(self, cfg: Config, batch: int, max_ctx: int, device=None):
        self.cfg, self.batch, self.max_ctx = cfg, batch, max_ctx
        c = cfg.to_c()
        nbytes = _size_out("w4a_kv_bytes", C.byref(c), batch, max_ctx)
        self.mem = torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.regions = []
        for l in range(cfg.n_layers):
            ko, vo, sl = C.c_size_t(0), C.c_size_t(0), C.c_int(0)
            call("w4a_kv_layer", C.byref(c), batch, max_ctx, l, C.byref(ko), C.byref(vo), C.byref(sl))
            self.regions.append((ko.value, vo.value, sl.value))

    def c(self) -> _abi.W4AKVCache:
        s = _abi.W4AKVCache()
        s.base, s.batch, s.max_ctx = self.mem.data_ptr(), self.batch, self.max_ctx
        return s

    def slots(self, layer: int) -> int:
        return self.regions[layer][2]

    def layer_views(self, layer: int):
        """(K, V) as bf16 tensors [batch, n_kv, slots, hd] in storage order (rows chunk-permuted)."""
        ko, vo, sl = self.regions[layer]
        cfg = self.cfg
        n = self.batch * cfg.n_kv_heads * sl * cfg.head_dim
        k = self.mem[ko:ko + 2 * n].view(torch.bfloat16).view(self.batch, cfg.n_kv_heads, sl, cfg.head_dim)
        v = self.mem[vo:vo + 2 * n].view(torch.bfloat16).view(self.batch, cfg.n_kv_heads, sl, cfg.head_dim)
        return k, v

    def write(self, layer: int, b: int, slot0: int, k: torch.Tensor, v: torch.Tensor):
        """Store logical rows k, v bf16 [n_kv, n, hd] at slots [slot0, slot0 + n) of sequence b."""
        _need(k, torch.bfloat16, "k")
        _need(v, torch.bfloat16, "v")
        kc, vc = self.layer_views(layer)
        cfg = self.cfg
        call("w4a_kv_write", _p(kc), _p(vc), self.batch, cfg.n_kv_heads, cfg.head_dim, self.slots(layer), b, slot0,
             k.shape[1], _p(k), _p(v), _stream())

    def fill_history(self, layer: int, b: int, k: torch.Tensor, v: torch.Tensor):
        """Store the rows of positions 0 .. n-1 (k, v bf16 [n_kv, n, hd]) of
        sequence b as the cache holds them: at their own slots in a layer with
        room for all of them, else (a sliding-window ring) the last `slots`
        positions at slot position % slots."""
        n, sl = k.shape[1], self.slots(layer)
        if n <= sl:
            self.write(layer, b, 0, k, v)
            return
        p0 = n - sl  # first position still held
        s0 = p0 % sl
        first = sl - s0  # positions p0 .. p0 + first - 1 go to slots s0 .. sl - 1
        self.write(layer, b, s0, k[:, p0:p0 + first].contiguous(), v[:, p0:p0 + first].contiguous())
        if first < sl:
            self.write(layer, b, 0, k[:, p0 + first:].contiguous(), v[:, p0 + first:].contiguous())

    def read(self, layer: int, b: int, slot0: int, n: int):
        cfg = self.cfg
        k = torch.empty((cfg.n_kv_heads, n, cfg.head_dim), dtype=torch.bfloat16, device=self.mem.device)
        v = torch.empty_like(k)
        kc, vc = self.layer_views(layer)
        call("w4a_kv_read", _p(kc), _p(vc), self.batch, cfg.n_kv_heads, cfg.head_dim, self.slots(layer), b, slot0,
             n, _p(k), _p(v), _stream())
        return k, v


def kv_write_region(k_region, v_region, batch: int, n_kv: int, hd: int, slots: int, b: int, slot0: int, k, v):
    """w4a_kv_write on a bare layer region (standalone attention)."""
    call("w4a_kv_write", _p(k_region), _p(v_region), batch, n_kv, hd, slots, b, slot0, k.shape[1], _p(k), _p(v),
         _stream())


# ---------------------------------------------------------------------------
# model
# ---------------------------------------------------------------------------
class Model:
    """Device weights of the decoder (tiled int4 body, bf16 embedding/lm_head)
    plus the library handle.  Build with ``Model.from_float``."""

    def __init__(self, cfg: Config, embed: torch.Tensor, lm_head_blob: torch.Tensor,
                 final_norm: Optional[torch.Tensor], layers: List[Dict[str, object]]):
        self.cfg, self.embed, self.lm_head, self.final_norm, self.layers = cfg, embed, lm_head_blob, final_norm, layers
        arr = (_abi.W4ALayerWeights * cfg.n_layers)()
        for l, L in enumerate(layers):
            a = arr[l]
            a.qkv, a.o = L["qkv"].blob.data_ptr(), L["o"].blob.data_ptr()
            a.gate_up, a.down = L["gate_up"].blob.data_ptr(), L["down"].blob.data_ptr()
            a.q_norm, a.k_norm = L["q_norm"].data_ptr(), L["k_norm"].data_ptr()
            a.post_attn_norm, a.post_ffn_norm = L["post_attn_norm"].data_ptr(), L["post_ffn_norm"].data_ptr()
        w = _abi.W4AModelWeights()
        w.embed, w.lm_head = embed.data_ptr(), lm_head_blob.data_ptr()
        w.final_norm = final_norm.data_ptr() if final_norm is not None else None
        w.layers = arr
        self._c_cfg = cfg.to_c()
        h = C.c_void_p()
        call("w4a_model_create", C.byref(self._c_cfg), C.byref(w), C.byref(h))
        self.handle = h
        self._ws = {}

    @classmethod
    def from_float(cls, cfg: Config, embed: torch.Tensor, lm_head: torch.Tensor, final_norm, layer_fn):
        """layer_fn(l) -> dict of fp32 CUDA tensors qkv, o, gate_up, down, q_norm,
        k_norm, post_attn_norm, post_ffn_norm (the float weights of layer l).
        Quantizes and tiles each matrix on the device."""
        layers = []
        for l in range(cfg.n_layers):
            raw = layer_fn(l)
            L = {"qkv": quantize_linear(raw["qkv"]), "o": quantize_linear(raw["o"]),
                 "gate_up": quantize_linear(raw["gate_up"], row_interleave=True),
                 "down": quantize_linear(raw["down"])}
            for g in ("q_norm", "k_norm", "post_attn_norm", "post_ffn_norm"):
                L[g] = raw[g].float().contiguous()
            del raw
            layers.append(L)
        return cls(cfg, embed.contiguous(), tile_bf16(lm_head.contiguous()),
                   None if final_norm is None else final_norm.float().contiguous(), layers)

    @classmethod
    def from_sym32(cls, cfg: Config, embed: torch.Tensor, lm_head: torch.Tensor, final_norm, layer_fn):
        """layer_fn(l) -> dict of (qweight int32, scales bf16) checkpoint pairs
        for qkv, o, gate_up, down in the symmetric group-32 format (cfg.group
        must be 32) and the four fp32 gains."""
        if cfg.group != 32:
            raise ValueError("from_sym32 needs cfg.group == 32")
        layers = []
        for l in range(cfg.n_layers):
            raw = layer_fn(l)
            L = {"qkv": tile_sym32(*raw["qkv"]), "o": tile_sym32(*raw["o"]),
                 "gate_up": tile_sym32(*raw["gate_up"], row_interleave=True), "down": tile_sym32(*raw["down"])}
            for g in ("q_norm", "k_norm", "post_attn_norm", "post_ffn_norm"):
                L[g] = raw[g].float().contiguous()
            del raw
            layers.append(L)
        return cls(cfg, embed.contiguous(), tile_bf16(lm_head.contiguous()),
                   None if final_norm is None else final_norm.float().contiguous(), layers)

    def __del__(self):
        try:
            if getattr(self, "handle", None) is not None and _abi._LIB is not None:
                _abi.lib().w4a_model_destroy(self.handle)
        except Exception:
            pass

    def workspace(self, batch: int) -> torch.Tensor:
        if batch not in self._ws:
            out = C.c_size_t(0)
            call("w4a_decode_workspace_bytes", self.handle, batch, C.byref(out))
            self._ws[batch] = zeros_workspace(out.value, self.embed.device)
        return self._ws[batch]

    def decode_step(self, kv: KVCache, tokens: torch.Tensor, pos: torch.Tensor, seq0: int = 0,
                    logits: Optional[torch.Tensor] = None, next_token: Optional[torch.Tensor] = None,
                    hidden_dump: Optional[torch.Tensor] = None, want_next: bool = True):
        _need(tokens, torch.int32, "tokens")
        _need(pos, torch.int32, "pos")
        B = tokens.shape[0]
        cfg = self.cfg
        if logits is None:
            logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device=tokens.device)
        if want_next and next_token is None:
            next_token = torch.empty((B,), dtype=torch.int32, device=tokens.device)
        ws = self.workspace(B)
        kvc = kv.c()
        call("w4a_decode_step", self.handle, _p(tokens), C.byref(kvc), seq0, B, _p(pos), _p(logits),
             _p(next_token) if want_next else None, _p(hidden_dump), _p(ws), ws.numel(), _stream())
        return logits, next_token

    def prefill_workspace(self, T: int) -> torch.Tensor:
        """Zero-filled scratch for w4a_prefill of T tokens (kept and reused
        while large enough; its leading part is a batch-1 decode workspace)."""
        out = C.c_size_t(0)
        call("w4a_prefill_workspace_bytes", self.handle, T, C.byref(out))
        cur = getattr(self, "_pf_ws", None)
        if cur is None or cur.numel() < out.value:
            self._pf_ws = None
            self._pf_ws = zeros_workspace(out.value, self.embed.device)
        return self._pf_ws

    def prefill(self, kv: KVCache, tokens: torch.Tensor, seq: int = 0, start_pos: int = 0,
                want_logits: bool = True) -> Optional[torch.Tensor]:
        _need(tokens, torch.int32, "tokens")
        last = torch.empty((self.cfg.vocab,), dtype=torch.float32, device=tokens.device) if want_logits else None
        ws = self.prefill_workspace(tokens.shape[0])
        kvc = kv.c()
        call("w4a_prefill", self.handle, _p(tokens), tokens.shape[0], C.byref(kvc), seq, start_pos, _p(last),
             _p(ws), ws.numel(), _stream())
        return last

    def check(self, batch: int = 1):
        ws = self.workspace(batch)
        check(ws)
        if batch == 1 and getattr(self, "_pf_ws", None) is not None:
            check(self._pf_ws)


class Trace:
    """Per-phase, per-CTA device timestamps of decode launches (w4a_trace)."""

    def __init__(self, n_phases: int, device=None):
        self.n_sms = torch.cuda.get_device_properties(device or 0).multi_processor_count
        self.buf = torch.zeros((n_phases, self.n_sms, 8), dtype=torch.int64, device=device or "cuda")
        call("w4a_trace", _p(self.buf), self.buf.numel() * 8)

    def stop(self):
        call("w4a_trace", None, 0)
        return self.buf.cpu()


def gemm_workspace(lin: W4Linear) -> torch.Tensor:
    t = lin.tensor()
    return zeros_workspace(_size_out("w4a_gemm_workspace_bytes", C.byref(t)), lin.blob.device)


def gemm(lin: W4Linear, x16: torch.Tensor, epilogue: int = _abi.EPI_NONE, row_scale: Optional[torch.Tensor] = None,
         ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = x16 . W~^T for many tokens (w4a_gemm): x16 fp16 [M, k]; fp32
    [M, n] out, or fp16 [M, n/2] silu(gate) * up with EPI_SILU_MUL."""
    _need(x16, torch.float16, "x16")
    M = x16.shape[0]
    if x16.shape[1] != lin.k:
        raise ValueError("x has the wrong width")
    if row_scale is not None:
        _need(row_scale, torch.float32, "row_scale")
    if ws is None:
        ws = gemm_workspace(lin)
    if out is None:
        if epilogue == _abi.EPI_SILU_MUL:
            out = torch.empty((M, lin.n // 2), dtype=torch.float16, device=x16.device)
        else:
            out = torch.empty((M, lin.n), dtype=torch.float32, device=x16.device)
    t = lin.tensor()
    call("w4a_gemm", C.byref(t), _p(x16), M, _p(row_scale), _p(out), epilogue, _p(ws), ws.numel(), _stream())
    return out


def attn_prefill(q: torch.Tensor, k_region: torch.Tensor, v_region: torch.Tensor, k_new: torch.Tensor,
                 v_new: torch.Tensor, batch: int, seq: int, slots: int, window: int, start_pos: int,
                 ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Causal GQA attention of a prompt (w4a_attn_prefill): q bf16 [T, nq,
    hd], the prompt's keys / values k_new, v_new bf16 [n_kv, T, hd], the
    history in a layer's cache regions; returns fp16 [T, nq, hd]."""
    _need(q, torch.bfloat16, "q")
    _need(k_new, torch.bfloat16, "k_new")
    _need(v_new, torch.bfloat16, "v_new")
    T, nq, hd = q.shape
    n_kv = k_new.shape[0]
    if ws is None:
        ws = zeros_workspace(256, q.device)
    if out is None:
        out = torch.empty((T, nq, hd), dtype=torch.float16, device=q.device)
    call("w4a_attn_prefill", _p(q), _p(k_region), _p(v_region), batch, seq, nq, n_kv, hd, slots, window,
         start_pos, T, _p(k_new), _p(v_new), _p(out), _p(ws), ws.numel(), _stream())
    return out


def check(ws: torch.Tensor):
    """Synchronise and raise if the workspace's device error word is set."""
    call("w4a_check", _p(ws), ws.numel(), _stream())


def check_noalloc():
    """Synchronise and raise if the error word of the fixed scratch that
    gemv_noalloc uses on the current device is set (w4a_check with no
    workspace).  Call it after a gemv_noalloc call and before the next one."""
    call("w4a_check", None, 0, _stream())


def sample(logits: torch.Tensor, temperature: float, top_p: float, u: torch.Tensor) -> torch.Tensor:
    """Temperature / top-p sampling of one token per row (w4a_sample): logits
    fp32 [B, V], draws u fp32 [B] in [0, 1); returns int32 [B]."""
    _need(logits, torch.float32, "logits")
    _need(u, torch.float32, "u")
    B, V = logits.shape
    ws = torch.empty(_size_out("w4a_sample_workspace_bytes", B, V), dtype=torch.uint8, device=logits.device)
    out = torch.empty((B,), dtype=torch.int32, device=logits.device)
    call("w4a_sample", _p(logits), B, V, C.c_float(temperature), C.c_float(top_p), _p(u), _p(out), _p(ws), ws.numel(),
         _stream())
    return out
