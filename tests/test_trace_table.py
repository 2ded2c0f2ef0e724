"""Host-side reduction of the engine's per-phase stamps (w4_weight_only_b200.trace)."""
import torch

from w4_weight_only_b200.trace import STEPS, phase_table


def _stamps(n_layers, ctas, step_ns, gap_ns):
    n = 5 * n_layers + 2
    t = torch.zeros(n, ctas, 8, dtype=torch.int64)
    base = 10_000_000
    period = 6 * step_ns + gap_ns
    for p in range(n):
        for c in range(ctas):
            for i in range(7):
                t[p, c, i] = base + p * period + i * step_ns + c  # CTAs 1 ns apart
    return t


def test_phase_table_steps_and_kinds():
    t = _stamps(n_layers=3, ctas=5, step_ns=2000, gap_ns=7000)
    res = phase_table(t, 3)
    assert list(res) == ["qkv", "attn", "o", "gate_up", "down", "lm_head", "argmax"]
    for kind, (n, span, steps) in res.items():
        assert n == (3 if kind not in ("lm_head", "argmax") else 1)
        assert len(steps) == len(STEPS)
        for a, b in steps[:6]:
            assert abs(a - 2.0) < 1e-9 and abs(b - 2.0) < 1e-9
        wait = steps[6][0]
        assert abs(wait - (0.0 if kind == "argmax" else 7.0)) < 1e-9
        assert abs(span - (12.0 + 0.004)) < 1e-9  # 6 steps + the CTA skew


def test_phase_table_skips_unstamped_steps():
    t = _stamps(n_layers=1, ctas=2, step_ns=1000, gap_ns=1000)
    t[0, :, 1] = 0  # step "desc" not stamped: its time moves to the next step
    res = phase_table(t, 1)
    steps = res["qkv"][2]
    assert steps[0] == (0.0, 0.0)
    assert abs(steps[1][0] - 2.0) < 1e-9
