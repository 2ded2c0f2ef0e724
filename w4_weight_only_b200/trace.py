"""Per-phase timeline of one decode step of the persistent engine.

    python -m w4_weight_only_b200.trace [--layers L] [--batch B] [--ctx C]

Builds the OLMo-3-32B-shaped synthetic model (the benchmark's shapes, seeds
and KV fill), runs a few decode steps, then one step with the device trace
on (`w4a_trace`: eight %globaltimer stamps per phase and CTA) and prints, per
phase kind, the median and maximum over CTAs of each step of the phase:

    desc     phase start (descriptor ready)        -> marks 0..1
    pass1    first pass of the input staging        -> 1..2
    staged   input staged in shared memory          -> 2..3
    units    weight / key units streamed            -> 3..4
    combine  pieces combined, rows written          -> 4..5
    arrive   CTA barrier + release to the grid      -> 5..6
    wait     until the next phase starts            -> 6..next 0

averaged over the layers.  The globaltimer ticks in 256 ns steps on this
part, so sub-microsecond entries are coarse.
"""
import argparse
import os

import torch

from . import api, synth
from . import config as wc

STEPS = ("desc", "pass1", "staged", "units", "combine", "arrive", "wait")


def phase_table(t: torch.Tensor, n_layers: int):
    """Median / max over CTAs of each step, averaged per phase kind.

    t: [phases][ctas][8] int64 stamps (0 = not stamped)."""
    names = ["qkv", "attn", "o", "gate_up", "down"]
    nph = t.shape[0]
    rows = {}
    t = t.double()
    for p in range(nph):
        kind = names[p % 5] if p < 5 * n_layers else ("lm_head" if p == 5 * n_layers else "argmax")
        x = t[p]
        ok = x[:, 0] > 0
        if not ok.any():
            continue
        span = (x[ok, 6].max() - x[ok, 0].min()).item() / 1000
        steps = []
        prev = x[:, 0]
        for i in (1, 2, 3, 4, 5, 6):
            cur = x[:, i]
            m = ok & (cur > 0)
            if m.any():
                dd = (cur - prev)[m] / 1000
                steps.append((dd.median().item(), dd.max().item()))
                prev = torch.where(cur > 0, cur, prev)
            else:
                steps.append((0.0, 0.0))
        if p + 1 < nph:
            w = (t[p + 1, :, 0] - x[:, 6])[ok & (t[p + 1, :, 0] > 0)] / 1000
            steps.append((w.median().item(), w.max().item()) if w.numel() else (0.0, 0.0))
        else:
            steps.append((0.0, 0.0))
        r = rows.setdefault(kind, [0, 0.0, [[0.0, 0.0] for _ in STEPS]])
        r[0] += 1
        r[1] += span
        for i, (a, b) in enumerate(steps):
            r[2][i][0] += a
            r[2][i][1] += b
    return {k: (n, span / n, [(a / n, b / n) for a, b in st]) for k, (n, span, st) in rows.items()}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--ctx", type=int, default=4096)
    ap.add_argument("--seed", type=int, default=3)
    args = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("a CUDA device is required")
    cfg = wc.olmo3_32b(args.layers)
    B, ctx = args.batch, args.ctx
    emb, head, fin = synth.embed_head(cfg, args.seed, "cuda")
    model = api.Model.from_float(cfg, emb, head, fin, lambda l: synth.layer_float(cfg, args.seed, l, "cuda"))
    kv = api.KVCache(cfg, B, ctx + 64)
    for l in range(cfg.n_layers):
        for b in range(B):
            k, v = synth.kv_rows(args.seed, l, b, cfg.n_kv_heads, ctx, cfg.head_dim, "cuda")
            kv.fill_history(l, b, k, v)
    tok = torch.ones(B, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(B, dtype=torch.int32, device="cuda")

    def pos(i):
        return torch.full((B,), ctx + i, dtype=torch.int32, device="cuda")

    for i in range(4):
        model.decode_step(kv, tok, pos(i), next_token=nxt)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(5):
        model.decode_step(kv, tok, pos(4 + i), next_token=nxt)
    e1.record()
    torch.cuda.synchronize()
    untraced = e0.elapsed_time(e1) / 5
    nph = 5 * cfg.n_layers + 2
    tr = api.Trace(nph)
    e0.record()
    model.decode_step(kv, tok, pos(9), next_token=nxt)
    e1.record()
    torch.cuda.synchronize()
    t = tr.stop()
    model.check(B)
    print(f"step: {untraced:.3f} ms untraced, {e0.elapsed_time(e1):.3f} ms traced "
          f"({cfg.n_layers} layers, batch {B}, ctx {ctx})")
    print("per phase kind: span, then median/max over CTAs of each step, us")
    t0 = t.double()
    ok = (t0[0, :, 7] > 0) & (t0[0, :, 0] > 0)
    if ok.any():
        su = (t0[0, ok, 0] - t0[0, ok, 7]) / 1000
        print(f"setup (CTA start to its first phase): median {su.median().item():.2f} us, max {su.max().item():.2f} us")
    print(f"{'kind':8s} {'n':>3s} {'span':>7s} " + " ".join(f"{s:>13s}" for s in STEPS))
    for k, (n, span, st) in phase_table(t, cfg.n_layers).items():
        print(f"{k:8s} {n:3d} {span:7.2f} " + " ".join(f"{a:6.2f}/{b:6.2f}" for a, b in st))


if __name__ == "__main__":
    main()
