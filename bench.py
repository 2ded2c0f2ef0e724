"""Benchmark: batch-1 decode of the 64-layer OLMo-3-32B-shaped int4 model at 4K context.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl w4a|reference]

One step = one decode token through the whole hot path (embedding, 64 x [QKV
GEMV, QK-norm + RoPE/YaRN + KV append, GQA attention, O GEMV, post-norm,
gate/up GEMV + SwiGLU, down GEMV, post-norm], final norm, lm_head, argmax), run
as one persistent kernel launch.  Greedy: each step consumes the previous
step's argmax on the device.  The KV cache is pre-filled with N(0,1) bf16 rows
for positions 0..4095 (sliding-window rings full); timed steps decode positions
4096 + warmup .. onward.  Weights are random-init (seeded), streamed from HBM
every token (16.2 GB of int4 + 1.03 GB lm_head, far above the 126 MB L2).

With --gpus N > 1 (launched by torchrun) every rank runs an independent replica
(the method has no data-path exchange); value = total tokens / max-over-ranks
device time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "decode tok/s @bs1, 32B-shape W4, 4K ctx; % of B200 HBM roofline"
CTX = 4096
SEED = 3
NOMINAL_HBM_GBS = 8000.0


# DRAM traffic of the engine from ncu: 4- and 8-layer launches of the
# benchmark model at ctx 4096 give the bytes per layer and the fixed part;
# valid only for the engine code they were taken on (its hash with comments
# and whitespace stripped).
TRAFFIC_ENGINE_CODE = "fd2d498d3fad205a"
TRAFFIC_FIXED = 1.033945e9
TRAFFIC_PER_LAYER = 0.270434e9


def engine_code_hash(text: str) -> str:
    """sha256 prefix of the engine source without // comments and whitespace:
    edits of comments or layout do not change the kernel."""
    import hashlib
    import re
    kept = []
    for line in text.splitlines():
        i = line.find("//")
        kept.append(re.sub(r"\s+", "", line if i < 0 else line[:i]))
    return hashlib.sha256("".join(kept).encode()).hexdigest()[:16]


def measured_traffic(n_layers: int):
    src = ROOT / "w4_weight_only_b200" / "csrc" / "engine.cuh"
    if not src.exists() or engine_code_hash(src.read_text()) != TRAFFIC_ENGINE_CODE:
        return None
    return int(TRAFFIC_FIXED + n_layers * TRAFFIC_PER_LAYER)


def measured_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes of one decode token (the roofline numerator)
# ---------------------------------------------------------------------------
def w4_bytes(n, k):
    return n * k // 2 + (k // 128) * n * 2 + (k // 128) * n // 2


def step_bytes(cfg, pos: int) -> int:
    """HBM bytes one batch-1 token must move: all int4 matrices (codes, fp16
    scales, int4 zeros), the bf16 lm_head, K and V of every visible key, the new
    K/V row per layer, norm gains and the embedding row."""
    d = cfg.d_model
    per_layer = (w4_bytes(cfg.qkv_dim, d) + w4_bytes(d, cfg.q_dim) + w4_bytes(2 * cfg.ffn, d)
                 + w4_bytes(d, cfg.ffn))
    kv_row = 2 * cfg.kv_dim * 2
    kv = 0
    for full in cfg.full_layers:
        keys = pos + 1 if full else min(pos + 1, cfg.window)
        kv += (keys - 1) * kv_row + kv_row          # read the old keys, write the new one
    gains = cfg.n_layers * (cfg.q_dim + cfg.kv_dim + 2 * d) * 4 + d * 4
    return cfg.n_layers * per_layer + cfg.vocab * d * 2 + kv + gains + d * 2


def linear_params_per_layer(cfg) -> int:
    d = cfg.d_model
    return cfg.qkv_dim * d + d * cfg.q_dim + 2 * cfg.ffn * d + d * cfg.ffn


def prefill_flops(cfg, T: int, start: int = 0) -> int:
    """Algorithmic FLOPs of a prompt of T tokens at positions start ..: the
    linear layers (2 per weight per token), QK^T and PV over each token's
    visible keys (causal; the window on SWA layers), the lm_head on the last
    token."""
    lin = 2 * T * cfg.n_layers * linear_params_per_layer(cfg) + 2 * cfg.vocab * cfg.d_model
    att = 0
    for full in cfg.full_layers:
        keys = 0
        for p in range(start, start + T):
            keys += p + 1 if full else min(p + 1, cfg.window)
        att += 4 * cfg.n_heads * cfg.head_dim * keys
    return lin + att


def measured_tensor_peak(sustained: bool):
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    return (1400.0 if sustained else 1590.0), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------
SAMPLE_ROWS = 256


def oracle_config_of(cfg):
    from oracle import model as om
    return om.OracleConfig(d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                           n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                           window=cfg.window, full_layers=list(cfg.full_layers), rope_theta=cfg.rope_theta,
                           yarn_factor=cfg.yarn_factor, yarn_orig_ctx=cfg.yarn_orig_ctx,
                           beta_fast=cfg.yarn_beta_fast, beta_slow=cfg.yarn_beta_slow, eps=cfg.eps,
                           group=cfg.group, final_norm=cfg.final_norm)


class OracleSample:
    """A bounded sample of one decode token through the float64 oracle: the
    first SAMPLE_ROWS rows of each of a layer's four int4 GEMVs (dequantize +
    matvec, the oracle's W4Matrix) and of the lm_head, one full-layer QK-prep +
    GQA attention over 4096 cached keys; the per-token time scales each GEMV by
    its rows / SAMPLE_ROWS and the layer by the layer count."""

    def __init__(self, cfg):
        import numpy as np
        from oracle import model as om
        from w4_weight_only_b200 import synth
        self.cfg, self.om, self.np = cfg, om, np
        self.ocfg = oracle_config_of(cfg)
        d, qd, kvd, f = cfg.d_model, cfg.q_dim, cfg.kv_dim, cfg.ffn
        shapes = {"qkv": (qd + 2 * kvd, d), "o": (d, qd), "gate_up": (2 * f, d), "down": (d, f)}
        r = SAMPLE_ROWS
        self.mats, self.xs, self.scale = {}, {}, {}
        for name, (n, k) in shapes.items():
            W = synth.normal((r, k), "cpu", 0.02, 0.0, SEED, "oracle_sample", name).numpy()
            self.mats[name] = om.W4Matrix.from_float(W, cfg.group)
            self.xs[name] = synth.normal((k,), "cpu", 1.0, 0.0, SEED, "oracle_sample_x", name).double().numpy()
            self.scale[name] = n / r
        self.head = synth.normal((r, d), "cpu", 0.02, 0.0, SEED, "oracle_sample", "head").to(
            __import__("torch").bfloat16).double().numpy()
        self.head_scale = cfg.vocab / r
        self.x = self.xs["qkv"]
        # one full layer's attention inputs at ctx 4096
        kcfg = om.OracleConfig(**{**self.ocfg.__dict__, "n_layers": 1, "full_layers": [True]})
        self.kv = om.OracleKV(kcfg, 1, CTX + 1)
        k, v = synth.kv_rows(SEED, 0, 0, cfg.n_kv_heads, CTX, cfg.head_dim, "cpu")
        self.kv.fill(0, 0, 0, k.double().numpy(), v.double().numpy())
        self.qr = synth.normal((qd,), "cpu", 1.0, 0.0, SEED, "oracle_sample_q").double().numpy()
        self.kr = synth.normal((kvd,), "cpu", 1.0, 0.0, SEED, "oracle_sample_k").double().numpy()
        self.qg = synth.normal((qd,), "cpu", 0.1, 1.0, SEED, "oracle_sample_qg").double().numpy()
        self.kg = synth.normal((kvd,), "cpu", 0.1, 1.0, SEED, "oracle_sample_kg").double().numpy()

    def _attention(self) -> None:
        q, k = self.om.qk_prep(self.ocfg, self.qr, self.kr, self.qg, self.kg, CTX, True)
        self.om.gqa_decode(self.ocfg, q, self.kv.K[0][0], self.kv.V[0][0], CTX - 1, True)

    def layer_seconds(self) -> float:
        """Seconds of one layer, projected from one pass over the sample."""
        t_layer = 0.0
        for name, W in self.mats.items():
            t0 = time.perf_counter()
            W.matvec(self.xs[name])
            t_layer += (time.perf_counter() - t0) * self.scale[name]
        t0 = time.perf_counter()
        self._attention()
        return t_layer + time.perf_counter() - t0

    def step(self) -> float:
        """Seconds of one token, estimated from one pass over the sample."""
        t_layer = self.layer_seconds()
        t0 = time.perf_counter()
        _ = self.head @ self.x[: self.cfg.d_model]
        t_head = (time.perf_counter() - t0) * self.head_scale
        return self.cfg.n_layers * t_layer + t_head

    def full_token_check(self) -> dict:
        """One token's work measured rather than projected by rows: one whole
        layer through the oracle (each int4 matrix at its full size,
        dequantize + float64 matvec, one at a time, then the layer's
        attention over CTX keys) and the whole bf16 lm_head, timed once; the
        token is that layer times the layer count (every layer has the same
        shapes, and at CTX = the window a sliding-window layer attends as many
        keys as a full one) plus the head.  Also returns the ratio to the
        sample's projection (median of three), which the reference arm uses
        to calibrate its per-step samples."""
        from w4_weight_only_b200 import synth
        projected = statistics.median(self.step() for _ in range(3))
        cfg = self.cfg
        d, qd, kvd, f = cfg.d_model, cfg.q_dim, cfg.kv_dim, cfg.ffn
        shapes = {"qkv": (qd + 2 * kvd, d), "o": (d, qd), "gate_up": (2 * f, d), "down": (d, f)}
        layer = 0.0
        for name, (n, k) in shapes.items():
            qw, sb, qz = (t.numpy() for t in synth.g128_storage(SEED, n, k, "oracle_full_layer", name))
            W = self.om.W4Matrix(qw, sb.view(self.np.uint16), qz, n, k, cfg.group)
            x = synth.normal((k,), "cpu", 1.0, 0.0, SEED, "oracle_full_layer_x", name).double().numpy()
            t0 = time.perf_counter()
            W.matvec(x)
            layer += time.perf_counter() - t0
            del W, qw, sb, qz
        t0 = time.perf_counter()
        self._attention()
        layer += time.perf_counter() - t0
        import torch
        head = synth.normal((cfg.vocab, d), "cpu", 0.02, 0.0, SEED, "oracle_full_head").to(
            torch.bfloat16).double().numpy()
        t0 = time.perf_counter()
        _ = head @ self.x[:d]
        t_head = time.perf_counter() - t0
        del head
        token = cfg.n_layers * layer + t_head
        return {"full_layer_s": round(layer, 3), "full_lm_head_s": round(t_head, 3), "token_s": round(token, 3),
                "sample_projected_token_s": round(projected, 3),
                "measured_over_projected": round(token / projected, 3)}

    def describe(self, steps: int) -> str:
        return (f"{steps} passes over a sample of one ctx-{CTX} token: the first {SAMPLE_ROWS} rows of each "
                f"int4 GEMV (dequantize + float64 matvec) and of the lm_head, one layer's QK-prep + GQA "
                f"attention over {CTX} keys; the token's time is projected from the sample by rows and by "
                f"{self.cfg.n_layers} layers")

    def sample_seconds(self) -> float:
        """Wall time of one pass over the sample itself (what is measured)."""
        t0 = time.perf_counter()
        for name, W in self.mats.items():
            W.matvec(self.xs[name])
        self._attention()
        _ = self.head @ self.x[: self.cfg.d_model]
        return time.perf_counter() - t0


def oracle_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        import torch
        return torch.get_num_threads()


def cpu_baseline(cfg):
    S = OracleSample(cfg)
    S.step()
    chk = S.full_token_check()
    return {"value": 1.0 / chk["token_s"], "unit": "tok/s", "cores": oracle_threads(), "kind": "oracle",
            "projected": "by layer count only", "full_token": chk,
            "sample": f"one whole layer of the ctx-{CTX} token (the four int4 GEMVs at full size, dequantize + "
                      f"float64 matvec, and the layer's QK-prep + GQA attention over {CTX} keys) and the whole "
                      f"lm_head, timed once; the token is {cfg.n_layers} such layers plus the head; "
                      f"host has {len(os.sched_getaffinity(0))} cores"}


# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    """--impl reference: the oracle on this host's cores, same metric and config."""
    from w4_weight_only_b200 import config as wc
    if rank != 0:
        return
    cfg = wc.olmo3_32b(args.layers)
    S = OracleSample(cfg)
    S.step()
    chk = S.full_token_check()          # once, before the steps: the calibration
    factor = chk["measured_over_projected"]
    for _ in range(args.warmup):
        S.step()
    t_region = time.perf_counter()
    ts = [S.step() * factor for _ in range(args.steps)]
    t_region = time.perf_counter() - t_region
    per_token = sum(ts) / len(ts)
    v = 1.0 / per_token
    base = {"value": v, "unit": "tok/s", "cores": oracle_threads(), "kind": "oracle", "projected": True,
            "measured_sample_s": round(S.sample_seconds(), 4), "full_token": chk,
            "sample": S.describe(args.steps) + f", times the ratio {factor} of one measured whole-layer token "
                                                f"to its projection; host has {len(os.sched_getaffinity(0))} cores"}
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * per_token,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "projected": True, "timed_region_wall_s": round(t_region, 3),
            "config": {"workload": f"OLMo-3-32B-shaped int4 (g128, fp16 scale, int4 zero) decode, "
                                   f"{cfg.n_layers} layers, batch 1, ctx {CTX}, greedy",
                       "batch": 1, "ctx": CTX, "layers": cfg.n_layers, "parallelism": "host cores"},
            "cpu_baseline": base,
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (device time of the timed region);
    every rank takes the same collective step."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tok_s(ms_max: float, steps: int, world: int) -> float:
    """Whole-job throughput: every replica decodes `steps` tokens; the job
    takes as long as its slowest rank."""
    return world * steps / (ms_max / 1000.0)


def measure_prefill(model, cfg, dev, lengths, repeats: int = 3):
    """Time to first token of prompts of uniform ids from position 0 through
    the public prefill call (CUDA events around the call; device-resident
    token ids, the last token's logits out), best of `repeats` after one
    untimed call; and the int4 GEMM alone (the gate/up matrix of layer 0,
    its fp16 expansion included) at the longest prompt's M."""
    import torch
    from w4_weight_only_b200 import api, synth
    out = {"workload": f"{cfg.n_layers}-layer model, prompts of " + " and ".join(str(T) for T in lengths)
                       + " uniform token ids from position 0; best of %d after a warm-up" % repeats,
           "ttft_ms": {}, "tflop": {}, "tflops": {}}
    for T in lengths:
        kv = api.KVCache(cfg, 1, (T + 16) // 16 * 16, device=dev)
        toks = synth.token_ids(SEED, T, cfg.vocab, dev, "prompt")
        model.prefill(kv, toks)
        torch.cuda.synchronize()
        best = None
        for _ in range(repeats):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            model.prefill(kv, toks)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        model.check()
        fl = prefill_flops(cfg, T)
        out["ttft_ms"][str(T)] = round(best, 2)
        out["tflop"][str(T)] = round(fl / 1e12, 2)
        out["tflops"][str(T)] = round(fl / (best / 1e3) / 1e12, 1)
        del kv
    M = max(lengths)
    lin = model.layers[0]["gate_up"]
    ws = api.gemm_workspace(lin)
    x = torch.randn((M, cfg.d_model), device=dev).to(torch.float16)
    api.gemm(lin, x, epilogue=2, ws=ws)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(repeats):
        api.gemm(lin, x, epilogue=2, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    api.check(ws)
    ms = e0.elapsed_time(e1) / repeats
    peak, src = measured_tensor_peak(sustained=False)
    ach = 2.0 * M * lin.n * lin.k / (ms / 1e3) / 1e12
    out["gemm"] = {"call": "w4a_gemm (fp16 expansion of the int4 matrix + tcgen05 GEMM)",
                   "shape": f"gate/up {lin.n}x{lin.k}, M={M}, SwiGLU epilogue", "ms": round(ms, 3),
                   "bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                   "frac": round(ach / peak, 4), "peak_source": src + " bf16 burst (fp16 has the same dense rate)"}
    del ws, x
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="w4a", choices=["w4a", "reference"])
    ap.add_argument("--layers", type=int, default=64, help="model depth (64 = the benchmark model)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill (TTFT) measurement")
    ap.add_argument("--no-sampled", action="store_true", help="skip the sampled-decode measurement")
    ap.add_argument("--mode", default="decode", choices=["decode", "prefill", "sample", "attn"],
                    help="prefill / sample: only that measurement (for profiling)")
    ap.add_argument("--prefill-tokens", default="1200,8192", help="prompt lengths of the prefill measurement")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    from w4_weight_only_b200 import api, synth
    from w4_weight_only_b200 import config as wc
    cfg = wc.olmo3_32b(args.layers)

    if args.mode == "attn":
        # the prompt attention alone at the 32B shape: 8,192 tokens from
        # position 0 through a 4,096 window, and through full attention
        out = {}
        nq, nkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
        T = max(int(t) for t in args.prefill_tokens.split(",") if t)
        for window in (cfg.window, 0):
            slots = window if window else (T + 15) // 16 * 16
            kreg = torch.zeros((1, nkv, slots, hd), dtype=torch.bfloat16, device=dev)
            vreg = torch.zeros_like(kreg)
            K = synth.normal((nkv, T, hd), str(dev), 1.0, 0.0, SEED, "attn_k", T).to(torch.bfloat16)
            V = synth.normal((nkv, T, hd), str(dev), 1.0, 0.0, SEED, "attn_v", T).to(torch.bfloat16)
            q = synth.normal((T, nq, hd), str(dev), 1.0, 0.0, SEED, "attn_q", T).to(torch.bfloat16)
            ws = torch.zeros(256, dtype=torch.uint8, device=dev)
            o = torch.empty((T, nq, hd), dtype=torch.float16, device=dev)
            for _ in range(args.warmup):
                api.attn_prefill(q, kreg, vreg, K, V, 1, 0, slots, window, 0, ws=ws, out=o)
            torch.cuda.synchronize()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record()
            for _ in range(args.steps):
                api.attn_prefill(q, kreg, vreg, K, V, 1, 0, slots, window, 0, ws=ws, out=o)
            c1.record()
            torch.cuda.synchronize()
            api.check(ws)
            ms = c0.elapsed_time(c1) / args.steps
            vis = sum(min(t + 1, window) if window else t + 1 for t in range(T))
            fl = 4.0 * hd * nq * vis
            out["window %d" % window if window else "full"] = {"ms": round(ms, 4), "tflop": round(fl / 1e12, 4),
                                                              "tflops": round(fl / (ms / 1e3) / 1e12, 1)}
        if rank == 0:
            print(json.dumps({"mode": "attn", "tokens": T, "heads": [nq, nkv, hd], "attention": out}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    if args.mode == "sample":
        # the sampler alone over the full vocabulary (temperature 0.6, top-p 0.95)
        out = {}
        for Bs in (1, 16):
            lgs = synth.logits_rows(SEED, Bs, cfg.vocab, 3.0, str(dev))
            us = synth.uniforms(SEED + 1, Bs, str(dev))
            for _ in range(args.warmup):
                api.sample(lgs, 0.6, 0.95, us)
            torch.cuda.synchronize()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record()
            for _ in range(args.steps):
                api.sample(lgs, 0.6, 0.95, us)
            c1.record()
            torch.cuda.synchronize()
            out[str(Bs)] = round(1000.0 * c0.elapsed_time(c1) / args.steps, 1)
        if rank == 0:
            print(json.dumps({"mode": "sample", "vocab": cfg.vocab, "us_per_call": out}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # ---- model and cache (not timed) ----
    emb, head, fin = synth.embed_head(cfg, SEED, "cuda")

    def layer_fn(l):
        return synth.layer_float(cfg, SEED, l, "cuda")

    model = api.Model.from_float(cfg, emb, head, fin, layer_fn)
    del head
    lengths = [int(t) for t in args.prefill_tokens.split(",") if t]
    if args.mode == "prefill":
        pf = measure_prefill(model, cfg, dev, lengths, repeats=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"mode": "prefill", "n_gpus": world, "prefill": pf}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    total = args.warmup + args.steps
    max_ctx = ((CTX + total + 1 + 15) // 16) * 16
    kv = api.KVCache(cfg, 1, max_ctx)
    for l in range(cfg.n_layers):
        k, v = synth.kv_rows(SEED, l, 0, cfg.n_kv_heads, CTX, cfg.head_dim, "cuda")
        if cfg.full_layers[l]:
            kv.write(l, 0, 0, k, v)
        else:
            W = cfg.window     # positions [0, 4096) fill the ring exactly once
            kv.write(l, 0, 0, k[:, CTX - W:].contiguous(), v[:, CTX - W:].contiguous())
        del k, v
    torch.cuda.synchronize()
    ws = model.workspace(1)
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device=dev)
    toks = torch.zeros((total + 1,), dtype=torch.int32, device=dev)
    toks[0] = 1
    positions = torch.arange(CTX, CTX + total, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        model.decode_step(kv, toks[i:i + 1], positions[i:i + 1], logits=logits, next_token=toks[i + 1:i + 2])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    api.check(ws)

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.warmup, total):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    api.check(ws)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world, dev)
    ms_step = ms_max / args.steps
    tok_s = job_tok_s(ms_max, args.steps, world)

    # roofline of the (only) kernel: algorithmic bytes per launch / its device time
    bytes_avg = sum(step_bytes(cfg, CTX + i) for i in range(args.warmup, total)) / args.steps
    peak, peak_src = measured_peaks()
    achieved = bytes_avg / (ms / args.steps / 1000.0) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": measured_traffic(cfg.n_layers), "peak_source": peak_src,
            "bytes_per_launch": int(bytes_avg), "frac_of_8000_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "kernel": "w4a_engine_kernel<1,128> (one launch per token)"}

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        h_tok = torch.zeros((1,), dtype=torch.int32).pin_memory()
        h_pos = torch.zeros((1,), dtype=torch.int32).pin_memory()
        h_next = torch.zeros((1,), dtype=torch.int32).pin_memory()
        d_tok = torch.zeros((1,), dtype=torch.int32, device=dev)
        d_pos = torch.zeros((1,), dtype=torch.int32, device=dev)
        d_next = torch.zeros((1,), dtype=torch.int32, device=dev)
        h_tok[0] = 1
        n_e2e = args.steps
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(n_e2e):
            h_pos[0] = CTX + i
            d_tok.copy_(h_tok, non_blocking=True)
            d_pos.copy_(h_pos, non_blocking=True)
            model.decode_step(kv, d_tok, d_pos, logits=logits, next_token=d_next)
            h_next.copy_(d_next, non_blocking=True)
            stream.synchronize()
            h_tok[0] = int(h_next[0])
        t1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(t0.elapsed_time(t1), world, dev)
        e2e = {"value": job_tok_s(te, n_e2e, world), "unit": "tok/s",
               "h2d_bytes_per_step": 8, "d2h_bytes_per_step": 4}

    # ---- sampled decode: the same steps with temperature 0.6 / top-p 0.95 ----
    sampled = None
    if not args.no_sampled:
        u_all = synth.uniforms(SEED, args.steps, str(dev)).contiguous()
        lg1 = torch.empty((1, cfg.vocab), dtype=torch.float32, device=dev)
        stok = torch.zeros((args.steps + 1,), dtype=torch.int32, device=dev)
        stok[0] = 1
        spos = torch.arange(CTX, CTX + args.steps, dtype=torch.int32, device=dev)

        def sstep(i):
            model.decode_step(kv, stok[i:i + 1], spos[i:i + 1], logits=lg1, want_next=False)
            stok[i + 1:i + 2].copy_(api.sample(lg1, 0.6, 0.95, u_all[i:i + 1]))

        for i in range(3):
            sstep(i)
        torch.cuda.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(args.steps):
            sstep(i)
        s1.record(stream)
        torch.cuda.synchronize()
        api.check(ws)
        ms_s = max_over_ranks(s0.elapsed_time(s1), world, dev)
        # the sampler alone at batch 1 and 16 over the full vocabulary
        per_call = {}
        for Bs in (1, 16):
            lgs = synth.logits_rows(SEED, Bs, cfg.vocab, 3.0, str(dev))
            us = synth.uniforms(SEED + 1, Bs, str(dev))
            api.sample(lgs, 0.6, 0.95, us)
            torch.cuda.synchronize()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(20):
                api.sample(lgs, 0.6, 0.95, us)
            c1.record(stream)
            torch.cuda.synchronize()
            per_call[str(Bs)] = round(1000.0 * c0.elapsed_time(c1) / 20, 1)
        sampled = {"value": job_tok_s(ms_s, args.steps, world), "unit": "tok/s",
                   "how": "each step: decode_step (logits) then w4a_sample (temperature 0.6, top-p 0.95, seeded "
                          "draws) feeding the next token, device-timed like the greedy steps",
                   "sample_us_per_call": per_call}

    pf = None
    if not args.no_prefill:
        del kv
        torch.cuda.empty_cache()
        pf = measure_prefill(model, cfg, dev, lengths)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            base = cpu_baseline(cfg)
        except Exception as ex:  # reported, never silently dropped
            base = {"error": repr(ex)}

    if rank == 0:
        line = {"metric": METRIC, "value": round(tok_s, 2), "unit": "tok/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
                "data": "synthetic",
                "config": {"workload": f"OLMo-3-32B-shaped int4 (g128, fp16 scale, int4 zero) decode, "
                                       f"{cfg.n_layers} layers, batch 1, ctx {CTX}..{CTX + total}, greedy",
                           "batch": 1, "ctx": CTX, "layers": cfg.n_layers,
                           "l2": "inputs larger than L2: 17.2 GB of weights streamed per token",
                           "parallelism": f"replicas x{world}"},
                "roofline": roof, "clocks": clk, "gpu_launches": args.steps,
                "e2e": e2e, "cpu_baseline": base, "sampled_decode": sampled, "prefill": pf}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
