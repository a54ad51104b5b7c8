"""Times one hot-path kernel in isolation on the shapes of a workload.

  python -m quantized_opt_decode_b200.microbench --kernel attn_decode --config opt-30b
  python -m quantized_opt_decode_b200.microbench --kernel all --config opt-30b

Kernels: qkv, out_proj, fc1, fc2 (dequant-fused linear layers at the decode
batch, or --rows for prefill-sized inputs), attn_decode (one layer's 4-bit
cache at KV length s + n/2), attn_topk (the same cache, top-k sparse),
layer_decode (one fused decode layer step), attn_prefill, kv_append,
layernorm, lm_head.
Prints one JSON line per kernel: average device time over --reps launches
(CUDA events on the launching stream, after --warmup launches) and the
achieved rate of the method's algorithmic bytes or FLOPs.  Also the small
case that `ncu` captures of single kernels run (--reps 3).
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from . import build  # noqa: E402

build.build()
from . import flexq as fq  # noqa: E402
from .device_model import KVCache, make_config, workspace  # noqa: E402

GEMMS = {"qkv": ("3h", "h", 0), "out_proj": ("h", "h", fq.EPI_RESIDUAL), "fc1": ("f", "h", fq.EPI_GELU),
         "fc2": ("h", "f", fq.EPI_RESIDUAL)}


def _dim(p, tag):
    return {"h": p["h"], "3h": 3 * p["h"], "f": p["ffn"]}[tag]


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d["hbm_gbs"], d["bf16_tflops"]
    return 6650.0, 1590.0


def _time(fn, reps, warmup, stream):
    for _ in range(warmup):
        fn()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def bench_gemm(p, kind, M, reps, warmup, stream, splits):
    n, k = _dim(p, GEMMS[kind][0]), _dim(p, GEMMS[kind][1])
    seed = synth.config_seed(p)
    w16 = torch.empty(n * k, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(w16, n * k, seed, 999, 0, 0.02, 0.0, stream)
    if p["w_bits"] == 4:
        w = torch.empty(fq.flexq_packed_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
        fq.flexq_quantize_weight_q4(w16, n, k, w, stream)
        del w16
        wbytes = n * k * (0.5 + 4 / 64)
    else:
        w = w16
        wbytes = n * k * 2
    x = torch.empty(M, k, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(x, M * k, seed, 998, 0, 1.0, 0.0, stream)
    bias = torch.zeros(n, dtype=torch.float16, device="cuda")
    res = torch.zeros(M, n, dtype=torch.float16, device="cuda")
    y = torch.empty(M, n, dtype=torch.float16, device="cuda")
    ws_n = max(fq.flexq_linear_workspace(M, n, k, p["w_bits"], splits), 1)
    ws = workspace(ws_n)
    epi = fq.EPI_BIAS | GEMMS[kind][2]

    def run():
        fq.flexq_linear(x, k, w, p["w_bits"], M, n, k, bias, res, n, epi, y, n, ws, ws_n, splits, stream)

    ms = _time(run, reps, warmup, stream)
    flops = 2.0 * M * n * k
    byts = wbytes + M * k * 2 + M * n * 2 * (2 if GEMMS[kind][2] == fq.EPI_RESIDUAL else 1)
    return ms, byts, flops, {"M": M, "N": n, "K": k}


def _filled_cache(p, cfg, b, L, stream):
    """One layer's cache for b sequences holding L seeded rows each."""
    h = p["h"]
    kv = KVCache(cfg, b, L + 1)
    seed = synth.config_seed(p)
    chunk = max(1, (1 << 28) // (b * 3 * h * 2))  # rows of history per fill pass
    rows = torch.empty(b * chunk, 3 * h, dtype=torch.float16, device="cuda")
    for t0 in range(0, L, chunk):
        nt = min(chunk, L - t0)
        fq.flexq_synth_normal_f16(rows, b * nt * 3 * h, seed, 997, t0 * 3 * h, 1.0, 0.0, stream)
        fq.flexq_kv_append(cfg, kv.struct, rows[:, h:], rows[:, 2 * h:], 3 * h, b, t0, nt, stream)
    del rows
    return kv


def bench_attn_decode(p, b, reps, warmup, stream, topk=0):
    cfg = make_config(p)
    h, a = p["h"], p["heads"]
    L = p["s"] + p["n"] // 2
    kv = _filled_cache(p, cfg, b, L, stream)
    seed = synth.config_seed(p)
    q = torch.empty(b, 3 * h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(q, b * 3 * h, seed, 996, 0, 1.0, 0.0, stream)
    out = torch.empty(b, h, dtype=torch.float16, device="cuda")

    kk = max(1, -(-L * topk // 1000))

    def run():
        if topk:
            fq.flexq_attention_decode_topk(cfg, kv.struct, q, 3 * h, b, L, kk, out, h, None, stream)
        else:
            fq.flexq_attention_decode(cfg, kv.struct, q, 3 * h, b, L, out, h, stream)

    ms = _time(run, reps, warmup, stream)
    d = h // a
    row = (d / 2 + 4 * d / 64) if p["kv_bits"] == 4 else 2 * d
    # top-k: every key, the kept keys' values (the method's bytes)
    byts = b * a * (L + (kk if topk else L)) * row + 2 * b * h * 2
    return ms, byts, 2.0 * b * (L + (kk if topk else L)) * h, {"b": b, "L": L, "heads": a, "d": d, "kept": kk}


def bench_layer_decode(p, b, reps, warmup, stream):
    """One fused decode layer step (QKV with the KV append, attention,
    output projection with LN2, FC1, FC2) at KV length s + n/2."""
    from .device_model import DeviceLayer
    cfg = make_config(p)
    h = p["h"]
    L = p["s"] + p["n"] // 2
    seed = synth.config_seed(p)
    layer = DeviceLayer(cfg, seed, 0, None, "cuda", stream)
    kv = _filled_cache(p, cfg, b, L, stream)
    t = torch.empty(b, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(t, b * h, seed, 991, 0, 1.0, 0.0, stream)
    y = torch.empty_like(t)
    ws_n = fq.flexq_layer_workspace(cfg, b, 1)
    ws = workspace(ws_n)

    def run():
        fq.flexq_layer_decode(cfg, layer.struct, t, y, kv.struct, b, L, ws, ws_n, stream)

    ms = _time(run, reps, warmup, stream)
    wb = 0.5 + 4 / 64 if p["w_bits"] == 4 else 2.0
    d = h // p["heads"]
    row = (d / 2 + 4 * d / 64) if p["kv_bits"] == 4 else 2 * d
    byts = (4 * h * h + 2 * h * p["ffn"]) * wb + b * p["heads"] * (L + 1) * 2 * row
    flops = 2.0 * b * (4 * h * h + 2 * h * p["ffn"]) + 4.0 * b * (L + 1) * h
    return ms, byts, flops, {"b": b, "L": L + 1}


def bench_attn_prefill(p, b, reps, warmup, stream):
    cfg = make_config(p)
    h, s = p["h"], p["s"]
    qkv = torch.empty(b * s, 3 * h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(qkv, qkv.numel(), synth.config_seed(p), 995, 0, 1.0, 0.0, stream)
    out = torch.empty(b * s, h, dtype=torch.float16, device="cuda")

    def run():
        fq.flexq_attention_prefill(cfg, qkv, 3 * h, b, s, out, h, stream)

    ms = _time(run, reps, warmup, stream)
    flops = 2.0 * b * s * s * h  # causal: half of 4 b s^2 h
    return ms, b * s * 4 * h * 2, flops, {"b": b, "s": s}


def bench_layernorm(p, M, reps, warmup, stream):
    h = p["h"]
    x = torch.empty(M, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(x, M * h, synth.config_seed(p), 994, 0, 1.0, 0.0, stream)
    g = torch.ones(h, dtype=torch.float16, device="cuda")
    bb = torch.zeros(h, dtype=torch.float16, device="cuda")
    y = torch.empty_like(x)

    def run():
        fq.flexq_layernorm(x, h, g, bb, y, h, M, h, 1e-5, stream)

    ms = _time(run, reps, warmup, stream)
    return ms, M * h * 4, 0.0, {"rows": M, "h": h}


def bench_kv_append(p, b, reps, warmup, stream):
    cfg = make_config(p)
    h = p["h"]
    kv = KVCache(cfg, b, p["s"] + p["n"])
    rows = torch.empty(b, 3 * h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(rows, rows.numel(), synth.config_seed(p), 993, 0, 1.0, 0.0, stream)

    def run():
        fq.flexq_kv_append(cfg, kv.struct, rows[:, h:], rows[:, 2 * h:], 3 * h, b, p["s"], 1, stream)

    ms = _time(run, reps, warmup, stream)
    d = h // p["heads"]
    return ms, b * 2 * h * 2 + b * p["heads"] * 2 * (d / 2 + 4 * d / 64), 0.0, {"b": b}


def bench_lm_head(p, b, reps, warmup, stream):
    h, V = p["h"], p["vocab"]
    E = torch.empty(V, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(E, V * h, synth.config_seed(p), synth.TID_EMBED, 0, 0.02, 0.0, stream)
    x = torch.empty(b, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(x, b * h, synth.config_seed(p), 992, 0, 1.0, 0.0, stream)
    y = torch.empty(b, V, dtype=torch.float32, device="cuda")
    ws_n = max(fq.flexq_linear_workspace(b, V, h, 16, 0), 1)
    ws = workspace(ws_n)

    def run():
        fq.flexq_linear(x, h, E, 16, b, V, h, None, None, 0, fq.EPI_F32_OUT, y, V, ws, ws_n, 0, stream)

    ms = _time(run, reps, warmup, stream)
    return ms, V * h * 2 + b * V * 4, 2.0 * b * V * h, {"b": b, "V": V}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="all")
    ap.add_argument("--config", default="opt-30b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--rows", type=int, default=0, help="GEMM rows (default: the decode batch)")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--topk", type=int, default=100, help="attn_topk: keys kept per mille")
    a = ap.parse_args()
    p = dict(synth.CONFIGS[a.config])
    hbm, tf = _peaks()
    stream = torch.cuda.Stream()
    kinds = ["qkv", "out_proj", "fc1", "fc2", "attn_decode", "kv_append", "layernorm", "lm_head",
             "attn_prefill"] if a.kernel == "all" else a.kernel.split(",")
    for kind in kinds:
        with torch.cuda.stream(stream):
            if kind in GEMMS:
                ms, byts, flops, shape = bench_gemm(p, kind, a.rows or p["gpu_batch"], a.reps, a.warmup,
                                                    stream, a.splits)
            elif kind == "attn_decode":
                ms, byts, flops, shape = bench_attn_decode(p, p["gpu_batch"], a.reps, a.warmup, stream)
            elif kind == "attn_topk":
                ms, byts, flops, shape = bench_attn_decode(p, p["gpu_batch"], a.reps, a.warmup, stream, a.topk)
            elif kind == "layer_decode":
                ms, byts, flops, shape = bench_layer_decode(p, p["gpu_batch"], a.reps, a.warmup, stream)
            elif kind == "attn_prefill":
                ms, byts, flops, shape = bench_attn_prefill(p, max(1, p["gpu_batch"] // 8), a.reps, a.warmup,
                                                            stream)
            elif kind == "layernorm":
                ms, byts, flops, shape = bench_layernorm(p, a.rows or p["gpu_batch"], a.reps, a.warmup, stream)
            elif kind == "kv_append":
                ms, byts, flops, shape = bench_kv_append(p, p["gpu_batch"], a.reps, a.warmup, stream)
            elif kind == "lm_head":
                ms, byts, flops, shape = bench_lm_head(p, p["gpu_batch"], a.reps, a.warmup, stream)
            else:
                raise SystemExit(f"unknown kernel {kind}")
        fq.flexq_device_status(stream)
        s = ms / 1e3
        print(json.dumps({"kernel": kind, "config": a.config, "shape": shape, "avg_us": round(ms * 1e3, 2),
                          "GB_s": round(byts / s / 1e9, 1), "TFLOP_s": round(flops / s / 1e12, 1),
                          "hbm_frac": round(byts / s / 1e9 / hbm, 4),
                          "tensor_frac": round(flops / s / 1e12 / tf, 4)}), flush=True)
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
