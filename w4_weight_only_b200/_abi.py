"""ctypes view of include/w4a.h: structs, prototypes and the library handle.

The library is loaded on first use.  There is no fallback: if libw4a.so is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes as C
from pathlib import Path

MAX_LAYERS = 128

OK, ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_KERNEL, ERR_TIMEOUT = (
    0, -1, -2, -3, -4, -5, -6, -7, -8)
F32, BF16 = 0, 1
LAYOUT_CANONICAL, LAYOUT_TILED, LAYOUT_SYM32 = 0, 1, 2
EPI_NONE, EPI_SUMSQ, EPI_SILU_MUL = 0, 1, 2
NOALLOC_SCRATCH_BYTES = 4194304

ERROR_NAMES = {OK: "OK", ERR_ARG: "ERR_ARG", ERR_SHAPE: "ERR_SHAPE", ERR_ALIGN: "ERR_ALIGN",
               ERR_UNSUPPORTED: "ERR_UNSUPPORTED", ERR_CUDA: "ERR_CUDA", ERR_WORKSPACE: "ERR_WORKSPACE",
               ERR_KERNEL: "ERR_KERNEL", ERR_TIMEOUT: "ERR_TIMEOUT"}


class W4AConfig(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("n_layers", C.c_int32), ("n_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("ffn", C.c_int32),
                ("vocab", C.c_int32), ("window", C.c_int32),
                ("full_layers", C.c_uint8 * MAX_LAYERS),
                ("rope_theta", C.c_double), ("yarn_factor", C.c_double),
                ("yarn_orig_ctx", C.c_int32), ("group", C.c_int32),
                ("yarn_beta_fast", C.c_double), ("yarn_beta_slow", C.c_double),
                ("eps", C.c_double), ("final_norm", C.c_int32), ("reserved", C.c_int32)]


class W4ATensor(C.Structure):
    _fields_ = [("n", C.c_int64), ("k", C.c_int64), ("group", C.c_int32), ("layout", C.c_int32),
                ("row_interleave", C.c_int32), ("reserved", C.c_int32),
                ("qweight", C.c_void_p), ("scales", C.c_void_p), ("qzeros", C.c_void_p)]


class W4ALayerWeights(C.Structure):
    _fields_ = [("qkv", C.c_void_p), ("o", C.c_void_p), ("gate_up", C.c_void_p), ("down", C.c_void_p),
                ("q_norm", C.c_void_p), ("k_norm", C.c_void_p),
                ("post_attn_norm", C.c_void_p), ("post_ffn_norm", C.c_void_p)]


class W4AModelWeights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(W4ALayerWeights))]


class W4AKVCache(C.Structure):
    _fields_ = [("base", C.c_void_p), ("batch", C.c_int32), ("max_ctx", C.c_int32)]


_P = C.c_void_p
_I = C.c_int
_I64 = C.c_int64
_SZ = C.c_size_t
_SZP = C.POINTER(C.c_size_t)
_IP = C.POINTER(C.c_int)

PROTOTYPES = {
    "w4a_last_error": (C.c_char_p, []),
    "w4a_version": (_I, []),
    "w4a_pack": (_I, [_P, _I, _I64, _I64, _I, _P, _P, _P, _P]),
    "w4a_unpack": (_I, [C.POINTER(W4ATensor), _P, _P]),
    "w4a_tiled_bytes": (_I, [_I64, _I64, _I, _SZP]),
    "w4a_tile": (_I, [C.POINTER(W4ATensor), _I, _P, _SZ, _P]),
    "w4a_tiled_bf16_bytes": (_I, [_I64, _I64, _SZP]),
    "w4a_tile_bf16": (_I, [_P, _I64, _I64, _P, _SZ, _P]),
    "w4a_gemv_workspace_bytes": (_I, [C.POINTER(W4ATensor), _I, _SZP]),
    "w4a_gemv": (_I, [C.POINTER(W4ATensor), _P, _I, _P, _I, _P, _P, _SZ, _P]),
    "w4a_gemv_noalloc": (_I, [C.POINTER(W4ATensor), _P, _I, _P, _I, _P, _P]),
    "w4a_attn_workspace_bytes": (_I, [_I, _I, _I, _I, _SZP]),
    "w4a_attn_decode": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "w4a_qk_prep": (_I, [C.POINTER(W4AConfig), _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _P]),
    "w4a_kv_bytes": (_I, [C.POINTER(W4AConfig), _I, _I, _SZP]),
    "w4a_kv_layer": (_I, [C.POINTER(W4AConfig), _I, _I, _I, _SZP, _SZP, _IP]),
    "w4a_kv_write": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "w4a_kv_read": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "w4a_model_create": (_I, [C.POINTER(W4AConfig), C.POINTER(W4AModelWeights), C.POINTER(_P)]),
    "w4a_model_destroy": (_I, [_P]),
    "w4a_decode_workspace_bytes": (_I, [_P, _I, _SZP]),
    "w4a_decode_step": (_I, [_P, _P, C.POINTER(W4AKVCache), _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "w4a_prefill": (_I, [_P, _P, _I, C.POINTER(W4AKVCache), _I, _I, _P, _P, _SZ, _P]),
    "w4a_prefill_workspace_bytes": (_I, [_P, _I, _SZP]),
    "w4a_gemm_workspace_bytes": (_I, [C.POINTER(W4ATensor), _SZP]),
    "w4a_gemm": (_I, [C.POINTER(W4ATensor), _P, _I, _P, _P, _I, _P, _SZ, _P]),
    "w4a_attn_prefill": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "w4a_trace": (_I, [_P, _SZ]),
    "w4a_check": (_I, [_P, _SZ, _P]),
    "w4a_sample_workspace_bytes": (_I, [_I, _I, C.POINTER(C.c_size_t)]),
    "w4a_sample": (_I, [_P, _I, _I, C.c_float, C.c_float, _P, _P, _P, _SZ, _P]),
}

_LIB = None


def lib_path() -> Path:
    return Path(__file__).resolve().parent / "libw4a.so"


def lib():
    """The loaded library (raises if it is not built)."""
    global _LIB
    if _LIB is None:
        p = lib_path()
        if not p.exists():
            raise RuntimeError(f"{p} is not built; run `python -m w4_weight_only_b200.build` "
                               "(there is no CPU fallback)")
        L = C.CDLL(str(p))
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


class W4AError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def call(name: str, *args) -> int:
    rc = getattr(lib(), name)(*args)
    if rc != OK:
        msg = lib().w4a_last_error().decode(errors="replace")
        raise W4AError(rc, name, msg)
    return rc
