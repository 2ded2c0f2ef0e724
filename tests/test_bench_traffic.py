"""The DRAM-traffic figure that bench.py reports is tied to the engine code
the counters were taken on: a change of comments or layout keeps it, a change
of code drops it (reported as null)."""
import importlib.util
import pathlib

ROOT = pathlib.Path(__file__).resolve().parents[1]


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", ROOT / "bench.py")
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_code_hash_ignores_comments_and_layout():
    b = _bench()
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    c = "// header\nint f(int x)\n{\n    return x + 1;\n}\n"
    assert b.engine_code_hash(a) == b.engine_code_hash(c)
    assert b.engine_code_hash(a) != b.engine_code_hash(a.replace("x + 1", "x + 2"))


def test_traffic_matches_current_engine_code():
    b = _bench()
    src = (ROOT / "w4_weight_only_b200" / "csrc" / "engine.cuh").read_text()
    if b.engine_code_hash(src) == b.TRAFFIC_ENGINE_CODE:
        t = b.measured_traffic(64)
        assert t is not None and abs(t / 18.3177e9 - 1) < 0.02  # within 2 % of the algorithmic bytes
    else:
        assert b.measured_traffic(64) is None
