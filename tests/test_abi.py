"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, loads, exports every entry point declared in include/w4a.h, its struct
layouts match the ctypes binding, and the size queries and argument checks
behave."""
import ctypes as C
import re
import subprocess
from pathlib import Path

import pytest

from oracle import counts, model as om

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "w4a.h"


def declared_functions():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"W4A_API\s+[\w\s\*]+?\b(w4a_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("w4a_pack", "w4a_unpack", "w4a_gemv", "w4a_attn_decode", "w4a_decode_step", "w4a_prefill",
                 "w4a_model_create", "w4a_kv_bytes", "w4a_check"):
        assert must in names


def test_library_exports_every_declared_symbol(built_lib):
    lib = C.CDLL(str(built_lib))
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", str(built_lib)], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(w4a_\w+)", out))
    assert set(declared_functions()) <= exported


def test_binding_prototypes_cover_header(built_lib):
    from w4_weight_only_b200 import _abi
    assert set(_abi.PROTOTYPES) == set(declared_functions())


def test_struct_layouts_match_c(tmp_path):
    from w4_weight_only_b200 import _abi
    src = tmp_path / "sz.c"
    src.write_text(f"""
#include <stdio.h>
#include <stddef.h>
#include "{HEADER}"
int main(void) {{
  printf("%zu %zu %zu %zu %zu\\n", sizeof(W4AConfig), sizeof(W4ATensor), sizeof(W4ALayerWeights),
         sizeof(W4AModelWeights), sizeof(W4AKVCache));
  printf("%zu %zu %zu\\n", offsetof(W4AConfig, rope_theta), offsetof(W4AConfig, eps), offsetof(W4ATensor, qweight));
  return 0;
}}""")
    exe = tmp_path / "sz"
    subprocess.run(["gcc", "-O0", "-o", str(exe), str(src)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = [int(v) for v in lines[0].split()]
    offs = [int(v) for v in lines[1].split()]
    assert sizes == [C.sizeof(_abi.W4AConfig), C.sizeof(_abi.W4ATensor), C.sizeof(_abi.W4ALayerWeights),
                     C.sizeof(_abi.W4AModelWeights), C.sizeof(_abi.W4AKVCache)]
    assert offs == [_abi.W4AConfig.rope_theta.offset, _abi.W4AConfig.eps.offset, _abi.W4ATensor.qweight.offset]


def _size(fn, *args):
    from w4_weight_only_b200 import _abi
    out = C.c_size_t(0)
    rc = getattr(_abi.lib(), fn)(*args, C.byref(out))
    return rc, out.value


def test_size_queries(built_lib):
    from w4_weight_only_b200 import _abi, config
    # 16 x 512 int4 unit = 4096 B codes + 128 B scales + 32 B zeros
    assert _size("w4a_tiled_bytes", 16, 512, 128) == (0, 4256)
    assert _size("w4a_tiled_bytes", 7168, 5120, 128) == (0, 7168 // 16 * 10 * 4256)
    rc, _ = _size("w4a_tiled_bytes", 16, 500, 128)
    assert rc == _abi.ERR_SHAPE
    assert _size("w4a_tiled_bf16_bytes", 100278, 5120) == (0, 6268 * 40 * 4096)
    # tiled int4 bytes equal the canonical storage (codes + fp16 scales + int4 zeros)
    assert _size("w4a_tiled_bytes", 55296, 5120, 128)[1] == counts.w4_bytes(55296, 5120)
    # the cache of the 32B shape equals the pages' SWA-aware count
    c = config.olmo3_32b().to_c()
    for ctx in (4096, 16384, 65536):
        rc, b = _size("w4a_kv_bytes", C.byref(c), 1, ctx)
        assert rc == 0 and b == counts.kv_bytes_at_context(om.olmo3_32b_config(), ctx, 2)


def test_argument_errors_without_gpu(built_lib):
    from w4_weight_only_b200 import _abi, config
    lib = _abi.lib()
    assert lib.w4a_pack(None, 0, 16, 128, 128, None, None, None, None) == _abi.ERR_ARG
    assert b"null" in lib.w4a_last_error()
    assert lib.w4a_pack(C.c_void_p(16), 7, 16, 128, 128, C.c_void_p(16), C.c_void_p(16), C.c_void_p(16),
                        None) == _abi.ERR_ARG
    assert lib.w4a_pack(C.c_void_p(16), 0, 16, 128, 64, C.c_void_p(16), C.c_void_p(16), C.c_void_p(16),
                        None) == _abi.ERR_UNSUPPORTED
    assert lib.w4a_pack(C.c_void_p(16), 0, 12, 128, 128, C.c_void_p(16), C.c_void_p(16), C.c_void_p(16),
                        None) == _abi.ERR_SHAPE
    assert lib.w4a_pack(C.c_void_p(18), 0, 16, 128, 128, C.c_void_p(16), C.c_void_p(16), C.c_void_p(16),
                        None) == _abi.ERR_ALIGN
    bad = config.tiny()
    bad.head_dim = 96
    c = bad.to_c()
    out = C.c_size_t(0)
    assert lib.w4a_kv_bytes(C.byref(c), 1, 64, C.byref(out)) == _abi.ERR_UNSUPPORTED
    c = config.tiny().to_c()
    assert lib.w4a_kv_bytes(C.byref(c), 1, 70, C.byref(out)) == _abi.ERR_SHAPE
    t = _abi.W4ATensor()
    t.n, t.k, t.group, t.layout, t.qweight = 16, 512, 128, _abi.LAYOUT_TILED, 16
    assert lib.w4a_gemv(C.byref(t), None, 1, None, 0, None, None, 0, None) == _abi.ERR_ARG
    assert lib.w4a_gemv_workspace_bytes(C.byref(t), 17, C.byref(out)) == _abi.ERR_SHAPE
    assert lib.w4a_gemv_workspace_bytes(C.byref(t), 1, C.byref(out)) == 0 and out.value >= 256


def test_model_create_validates(built_lib):
    from w4_weight_only_b200 import _abi, config
    lib = _abi.lib()
    c = config.tiny().to_c()
    arr = (_abi.W4ALayerWeights * 4)()
    w = _abi.W4AModelWeights()
    w.embed, w.lm_head, w.final_norm, w.layers = 16, 16, 16, arr
    h = C.c_void_p()
    assert lib.w4a_model_create(C.byref(c), C.byref(w), C.byref(h)) == _abi.ERR_ARG   # null layer pointers
    for a in arr:
        a.qkv = a.o = a.gate_up = a.down = 16
        a.q_norm = a.k_norm = a.post_attn_norm = a.post_ffn_norm = 16
    assert lib.w4a_model_create(C.byref(c), C.byref(w), C.byref(h)) == 0
    out = C.c_size_t(0)
    assert lib.w4a_decode_workspace_bytes(h, 1, C.byref(out)) == 0 and out.value > 0
    assert lib.w4a_decode_workspace_bytes(h, 17, C.byref(out)) == _abi.ERR_SHAPE
    assert lib.w4a_model_destroy(h) == 0


def test_no_cpu_fallback_when_library_missing(tmp_path, monkeypatch):
    from w4_weight_only_b200 import _abi
    monkeypatch.setattr(_abi, "_LIB", None)
    monkeypatch.setattr(_abi, "lib_path", lambda: tmp_path / "missing.so")
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _abi.lib()
