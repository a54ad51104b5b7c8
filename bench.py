#!/usr/bin/env python
"""Decode throughput of the group-wise 4-bit OPT-style block on B200.

Default workload: the OPT-30B shape (48 layers, h=7168, 56 heads, FFN 28672,
vocab 50272), weights and KV cache in the group-wise 4-bit format, a block of
144 sequences, prompt length 512, 32 generated tokens, one GPU batch of 144.

One timed step is the decode phase of flexq_generate: the n-1 = 31 decode
columns of the zig-zag block (every layer for every GPU batch, then the tied
LM head and the greedy choice), run through the public entry point
flexq_generate_decode on caches filled by one prefill.  value = b * (n - 1) *
n_gpus / (max over ranks of the step time).  Weights (16.7 GB) and KV (30 GB)
are far larger than L2, so no flush is needed between steps.

Other figures on the same JSON line: the prefill column timed once, the
per-kernel breakdown of one profiled decode step (CUDA events around every
kernel, a separate pass after the timed steps), the roofline of the dominant
kernel against MEASURED_PEAKS.json, SM clocks sampled during the timed
region, an end-to-end run of flexq_generate with the prompts uploaded from
pinned host memory and the tokens read back, and the CPU oracle timed on a
bounded sample (`cpu_baseline`).

`--impl reference` times the CPU oracle alone on the same metric (each step =
one oracle layer decode for a few sequences, extrapolated to tokens/s).
Multi-GPU: one independent replica per rank (weak scaling, no collective on
the data path; torch.distributed only for the barrier and the max-over-ranks
timing).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402


# ---------------------------------------------------------------------------
# common helpers
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def csrc_hash(files=None):
    """Hash of the CUDA sources (all of them, or the named files)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_opt_decode_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# Source files that define each kernel kind's device code: an ncu traffic
# figure stays valid while these are unchanged.
_SHARED = ["common.cuh", "kernels.h"]
_GEMM = ["gemm_tc.cu"] + _SHARED
KERNEL_FILES = {
    # the decode attention kernels quantize the appended token with quant_common.cuh
    "attn_decode": ["attn_decode.cu", "attn_topk.cu", "quant_common.cuh"] + _SHARED,
    "qkv": _GEMM, "out_proj": _GEMM, "fc1": _GEMM, "fc2": _GEMM, "lm_head": _GEMM,
    "kv_append": ["kv_append.cu", "quant_common.cuh"] + _SHARED,
    "layernorm": ["rowwise.cu"] + _SHARED, "embed": ["rowwise.cu"] + _SHARED,
}


def ncu_traffic(kind: str):
    """DRAM bytes per launch of `kind` from the committed ncu summary, or None
    when absent or taken on other sources of that kernel."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path) or kind not in KERNEL_FILES:
        return None
    cur = csrc_hash(KERNEL_FILES[kind])
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kind:
                return float(parts[1]) if parts[2] == cur else None
    return None


def max_over_ranks(x: float, device: str = "cuda") -> float:
    """The largest x over all ranks (all ranks must call it, in the same
    order); x itself when there is no process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def prompt_tensor_id(rank: int) -> int:
    """Each replica generates its own block of prompts."""
    return synth.TID_PROMPT + 7919 * rank


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while active."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = num(rows[0][2])
        load = [v for v in sm if smax and v > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---------------------------------------------------------------------------
# algorithmic work per kernel call (decode step, M = b rows)
# ---------------------------------------------------------------------------
def kernel_work(p: dict, kind: str, M: int, L_avg: float):
    """(bytes, flops) the method must move / compute in one call of `kind`."""
    h, f, a = p["h"], p["ffn"], p["heads"]
    d = h // a
    wb = 0.5 + 4 / 64 if p["w_bits"] == 4 else 2.0
    kvb = (d / 2 + 4 * d / 64) if p["kv_bits"] == 4 else 2 * d  # bytes per cached row
    gemm = {"qkv": (3 * h, h, False), "out_proj": (h, h, True), "fc1": (f, h, False),
            "fc2": (h, f, True)}
    if kind in gemm:
        n, k, res = gemm[kind]
        byts = n * k * wb + M * k * 2 + M * n * 2 * (2 if res else 1) + n * 2
        return byts, 2.0 * M * n * k
    if kind == "attn_decode":
        if p.get("topk_permille", 0) > 0:
            # top-k sparse: every key, and the values of the kept keys only
            kept = max(1.0, math.ceil(L_avg * p["topk_permille"] / 1000.0))
            return M * a * (L_avg + kept) * kvb + 2 * M * h * 2, 2.0 * M * (L_avg + kept) * h
        return M * a * L_avg * 2 * kvb + 2 * M * h * 2, 4.0 * M * L_avg * h
    if kind == "attn_prefill":  # causal: half of the s x s score and value products
        if p.get("prefill_kv_cache"):  # Q and O fp16, K and V read back from the cache
            return M * h * 2 * 2 + 2 * M * a * kvb, 2.0 * M * L_avg * h
        return M * h * 2 * 4, 2.0 * M * L_avg * h
    if kind == "kv_append":
        return M * 2 * h * 2 + M * a * 2 * kvb, 0.0
    if kind == "layernorm":
        return M * h * 4 + 4 * h, 0.0
    if kind == "lm_head":
        eb = 0.5 + 4 / 64 if p.get("embed_bits", 16) == 4 else 2.0
        return p["vocab"] * h * eb + M * h * 2 + M * p["vocab"] * 4, 2.0 * M * p["vocab"] * h
    if kind == "argmax":
        return M * p["vocab"] * 4, 0.0
    if kind == "embed":
        return M * h * 6, 0.0
    return 0.0, 0.0


def roof_time(p, kind, M, L, peaks) -> float:
    """Seconds one call of `kind` takes at its roofline: the larger of its
    algorithmic bytes at the measured HBM copy rate and its flops at the
    measured sustained dense rate."""
    byts, flops = kernel_work(p, kind, M, L)
    return max(byts / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops_sustained"] * 1e12))


def step_ceilings(p: dict, gbs: int, peaks: dict) -> dict:
    """Tokens/s the decode phase and the prefill column would reach if every
    kernel they launch ran at its own roofline (the per-kernel rooflines
    summed over the launches of the step, in the launch order of
    flexq_generate: per column and GPU batch the embedding, l layer steps,
    the final LayerNorm, the tied LM head and the greedy choice)."""
    b, s, n, layers = p["b"], p["s"], p["n"], p["layers"]
    batches = b // gbs

    def column(rows_per_batch, embed_rows, L, attn):
        # embedding over the whole block, then every layer for every GPU
        # batch, then the final LayerNorm, LM head and greedy choice over the
        # block's last rows
        t = roof_time(p, "embed", embed_rows, L, peaks)
        layer = (2 * roof_time(p, "layernorm", rows_per_batch, L, peaks)
                 + roof_time(p, "qkv", rows_per_batch, L, peaks)
                 + roof_time(p, "kv_append", rows_per_batch, L, peaks)
                 + roof_time(p, attn, rows_per_batch, L, peaks)
                 + roof_time(p, "out_proj", rows_per_batch, L, peaks)
                 + roof_time(p, "fc1", rows_per_batch, L, peaks)
                 + roof_time(p, "fc2", rows_per_batch, L, peaks))
        t += layers * batches * layer
        t += (roof_time(p, "layernorm", b, L, peaks) + roof_time(p, "lm_head", b, L, peaks)
              + roof_time(p, "argmax", b, L, peaks))
        return t

    t_dec = sum(column(gbs, b, s + j + 1, "attn_decode") for j in range(1, n))
    t_pre = column(gbs * s, b * s, s, "attn_prefill")
    return {"decode_tokens_per_s": b * (n - 1) / t_dec, "prefill_tokens_per_s": b * s / t_pre}


def phase_work(p: dict, kind: str, calls: int, gbs: int, phase: str, columns: int):
    """(bytes, flops) of all `calls` launches of `kind` in one profiled pass of
    a phase ("decode": the n-1 decode columns; "prefill": the prefill column).
    Inside the layer steps a call covers one GPU batch (gbs rows, or gbs * s
    in the prefill); the embedding, the final LayerNorm, the LM head and the
    argmax cover the whole block once per column (the final LayerNorm shares
    its kind with the layer LayerNorms: `columns` of the calls are final)."""
    b, s, n = p["b"], p["s"], p["n"]
    rows = gbs * s if phase == "prefill" else gbs
    L = s if phase == "prefill" else s + n / 2.0
    if kind in ("lm_head", "argmax"):
        byts, flops = kernel_work(p, kind, b, L)
        return calls * byts, calls * flops
    if kind == "embed":
        byts, flops = kernel_work(p, kind, b * s if phase == "prefill" else b, L)
        return calls * byts, calls * flops
    if kind == "layernorm":
        n_final = min(columns, calls)
        bl, _ = kernel_work(p, kind, rows, L)
        bf, _ = kernel_work(p, kind, b, L)
        return (calls - n_final) * bl + n_final * bf, 0.0
    byts, flops = kernel_work(p, kind, rows, L)
    return calls * byts, calls * flops


def roofline(kind, byts, flops, seconds, peaks):
    """Achieved rate of `kind` (all its launches in a profiled pass) against
    its roof: the tensor pipe when its arithmetic intensity is above the
    ridge of the measured peaks, HBM otherwise."""
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops > 0 and flops / max(byts, 1.0) > ridge:
        ach = flops / seconds / 1e12
        peak = peaks["bf16_tflops_sustained"]
        return {"kernel": kind, "bound": "tensor", "achieved": round(ach, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "peak_note": f"{peaks['source']} dense bf16 sustained (fp16 nominal ratio 1:1)"}
    ach = byts / seconds / 1e9
    peak = peaks["hbm_gbs"]
    return {"kernel": kind, "bound": "hbm", "achieved": round(ach, 1), "peak": peak,
            "unit": "GB/s", "frac": round(ach / peak, 4), "peak_note": f"{peaks['source']} HBM copy"}


def kernel_table(p, prof, gbs, phase, columns, peaks):
    """Per-kind calls, time, share and roofline fraction of one profiled pass."""
    out = {}
    total = sum(v[0] for v in prof.values()) or 1.0
    for kind, (kms, calls) in prof.items():
        if calls == 0:
            continue
        byts, flops = phase_work(p, kind, calls, gbs, phase, columns)
        rl = roofline(kind, byts, flops, kms / 1e3, peaks)
        out[kind] = {"calls": calls, "ms": round(kms, 3), "share": round(kms / total, 4),
                     "avg_us": round(kms / calls * 1e3, 2), "bound": rl["bound"],
                     "achieved": rl["achieved"], "unit": rl["unit"], "frac": rl["frac"],
                     "algorithmic_bytes_per_call": round(byts / calls),
                     "algorithmic_flops_per_call": round(flops / calls)}
    return out


def codec_rates(fq, torch, p, stream, reps=5):
    """GB/s of the quantize/pack kernels (weights: fp16 in, packed 4-bit out;
    2 + 0.5625 bytes per element) and of the dequantizer (0.5625 + 2), on a
    matrix of the workload's FC1 shape [ffn][h], CUDA events on `stream`."""
    n_out, k_in = p["ffn"], p["h"]
    n = n_out * k_in
    w = torch.empty(n, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(w, n, synth.config_seed(p), synth.TID_TEST_BASE + 99, 0, 0.02, 0.0, stream)
    packed = torch.empty(fq.flexq_packed_weight_bytes(n_out, k_in), dtype=torch.uint8, device="cuda")
    codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    mn = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    sc = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    out = torch.empty_like(w)
    ops = {
        "quantize_weight_q4": (lambda: fq.flexq_quantize_weight_q4(w, n_out, k_in, packed, stream), 2.5625),
        "quantize": (lambda: fq.flexq_quantize(w, n, codes, mn, sc, stream), 2.5625),
        "dequantize": (lambda: fq.flexq_dequantize(codes, mn, sc, n, out, stream), 2.5625),
    }
    res = {}
    for name, (fn, bpe) in ops.items():
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        stream.synchronize()
        t = e0.elapsed_time(e1) / reps / 1e3
        res[name] = {"elements": n, "us": round(t * 1e6, 1), "GBps": round(n * bpe / t / 1e9, 1),
                     "frac": round(n * bpe / t / 1e9 / load_peaks()["hbm_gbs"], 4)}
    fq.flexq_device_status(stream)
    del w, packed, codes, mn, sc, out
    return res


# ---------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """One layer of the workload on the CPU oracle: a decode step for b_o
    sequences at the average KV length s + n/2 over a seeded cache."""

    def __init__(self, p: dict, b_o: int):
        from oracle import opt
        self.opt = opt
        self.p = p
        self.b_o = b_o
        self.cfg = opt.Config.from_preset(p)
        seed = synth.config_seed(p)
        self.W = opt.effective_layer(self.cfg, opt.raw_layer(self.cfg, seed, 0))
        self.L = p["s"] + p["n"] // 2
        self.cache = opt.KVCache(self.cfg, b_o, self.L + 1, self.cfg.kv_bits)
        h = p["h"]
        hist = synth.normal_f16(seed, synth.TID_TEST_BASE + 1, b_o * self.L * h, 1.0)
        hist = hist.reshape(b_o, self.L, h)
        self.cache.write("k", hist, 0)
        self.cache.write("v", hist, 0)
        self.t = synth.normal_f16(seed, synth.TID_TEST_BASE + 2, b_o * h, 1.0).reshape(b_o, h)
        self.t = self.t.astype(np.float64)

    def step(self) -> float:
        t0 = time.perf_counter()
        self.opt.layer_decode(self.cfg, self.W, self.t, self.cache, self.L)
        return time.perf_counter() - t0

    def tokens_per_s(self, seconds: float) -> float:
        # one decode token of one sequence needs all l layers
        return self.b_o / (seconds * self.p["layers"])

    def prefill_step(self, s_p: int) -> float:
        """Layer-0 prefill of one sequence's first s_p prompt tokens (causal, so
        it is exactly the prefill of an s_p-token prompt)."""
        x = synth.normal_f16(synth.config_seed(self.p), synth.TID_TEST_BASE + 3, s_p * self.p["h"], 1.0)
        x = x.reshape(1, s_p, self.p["h"]).astype(np.float64)
        t0 = time.perf_counter()
        self.opt.layer_prefill(self.cfg, self.W, x)
        return time.perf_counter() - t0


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(p: dict, budget_s: float = 12.0):
    t_setup = time.perf_counter()
    smp = OracleSample(p, b_o=4)
    setup = time.perf_counter() - t_setup
    smp.step()  # warm
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        times.append(smp.step())
    t = statistics.median(times)
    s_p = min(p["s"], 128)
    t_pre = smp.prefill_step(s_p)
    return {"value": round(smp.tokens_per_s(t), 4), "unit": "tokens/s", "cores": cpu_cores(),
            "kind": "oracle",
            "prefill_value": round(s_p / (t_pre * p["layers"]), 4),
            "sample": (f"oracle (numpy float64) decode of layer 0 for {smp.b_o} sequences at KV "
                       f"length {smp.L + 1}, {len(times)} repetitions, median {t * 1e3:.1f} ms, "
                       f"extrapolated x{p['layers']} layers per token; prefill_value: layer-0 "
                       f"prefill of one {s_p}-token prompt, {t_pre:.2f} s, extrapolated the same "
                       f"way; setup {setup:.0f} s (weights drawn, quantized, dequantized on the host)")}


def run_reference(args, p):
    import torch.distributed as dist  # noqa: F401
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample(p, b_o=4)
    for _ in range(args.warmup):
        smp.step()
    times = [smp.step() for _ in range(args.steps)]
    t = sum(times) / len(times)
    v = smp.tokens_per_s(t)
    line = {"metric": METRIC, "value": round(v, 4), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(args), "global_batch": smp.b_o, "seq_len": p["s"],
                       "gen_tokens": p["n"], "note": "one layer per step, extrapolated"},
            "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": cpu_cores(),
                             "kind": "oracle",
                             "sample": f"layer-0 decode of {smp.b_o} sequences at KV length "
                                       f"{smp.L + 1} per step, x{p['layers']} layers"},
            "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


METRIC = "decode tokens/s, OPT-30B-shape 4-bit W+KV; HBM GB/s & tensor util vs peak"


def workload_name(args) -> str:
    """The configuration's name, plus the variants that change the work."""
    name = args.config
    if args.embed_bits == 4:
        name += "+embed4"
    if args.topk:
        name += f"+topk{args.topk}"
    if args.prefill_kv_cache:
        name += "+prefillkv"
    if args.no_launch_overlap:
        name += "+nooverlap"
    return name


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_flexq(args, p):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    torch.cuda.set_device(local)
    from quantized_opt_decode_b200 import build
    build.build()
    from quantized_opt_decode_b200 import flexq as fq
    from quantized_opt_decode_b200.device_model import DeviceModel, workspace
    fq.flexq_set_launch_overlap(not args.no_launch_overlap)

    b, s, n, gbs = p["b"], p["s"], p["n"], p["gpu_batch"]
    stream = torch.cuda.Stream()
    t_setup = time.perf_counter()
    with torch.cuda.stream(stream):
        dm = DeviceModel(p, b=b, max_len=s + n, stream=stream)
        prompts = torch.empty(b, s, dtype=torch.int32, device="cuda")
        fq.flexq_synth_tokens(prompts, b * s, synth.config_seed(p), prompt_tensor_id(rank),
                              p["vocab"], stream=stream)
        out = torch.zeros(b, n, dtype=torch.int32, device="cuda")
        ws_n = fq.flexq_generate_workspace(dm.struct, b, s, gbs)
        ws = workspace(ws_n)
    stream.synchronize()
    setup_s = time.perf_counter() - t_setup

    def ev():
        return torch.cuda.Event(enable_timing=True)

    # prefill column once (fills every layer's cache)
    e0, e1 = ev(), ev()
    e0.record(stream)
    fq.flexq_generate_prefill(dm.struct, prompts, b, s, n, gbs, out, ws, ws_n, stream)
    e1.record(stream)
    stream.synchronize()
    prefill_ms = e0.elapsed_time(e1)
    fq.flexq_device_status(stream)

    def step():
        fq.flexq_generate_decode(dm.struct, b, s, n, gbs, out, ws, ws_n, stream)

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    fq.flexq_device_status(stream)

    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        l0 = fq.flexq_launch_count()
        t0, t1 = ev(), ev()
        torch.cuda.nvtx.range_push("timed")
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        launches = fq.flexq_launch_count() - l0
        if world > 1:
            dist.barrier()
    clocks = clk.summary()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    fq.flexq_device_status(stream)
    value = world * b * (n - 1) / (ms / 1e3)

    # per-kernel breakdown: one more decode phase with every kernel bracketed
    fq.flexq_profile_start()
    step()
    prof = fq.flexq_profile_stop(stream)
    peaks = load_peaks()
    kernels = kernel_table(p, prof, gbs, "decode", n - 1, peaks)
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    byts, flops = phase_work(p, dom, prof[dom][1], gbs, "decode", n - 1)
    rl = roofline(dom, byts, flops, prof[dom][0] / 1e3, peaks)
    rl["traffic"] = ncu_traffic(dom)
    rl["algorithmic_per_launch"] = {"bytes": round(byts / prof[dom][1]), "flops": round(flops / prof[dom][1])}
    ceil = step_ceilings(p, gbs, peaks)

    # the prefill column once more, every kernel bracketed
    fq.flexq_profile_start()
    fq.flexq_generate_prefill(dm.struct, prompts, b, s, n, gbs, out, ws, ws_n, stream)
    prof_pre = fq.flexq_profile_stop(stream)
    fq.flexq_device_status(stream)
    prefill_kernels = kernel_table(p, prof_pre, gbs, "prefill", 1, peaks)
    codec = None if args.no_codec else codec_rates(fq, torch, p, stream)

    # end to end through flexq_generate: prompts from pinned host memory,
    # tokens back to pinned host memory, all inside the timed region
    e2e = None
    if not args.no_e2e:
        host_prompts = prompts.cpu().pin_memory()
        host_out = torch.empty(b, n, dtype=torch.int32).pin_memory()
        dev_prompts = torch.empty_like(prompts)

        def e2e_step():
            dev_prompts.copy_(host_prompts, non_blocking=True)
            fq.flexq_generate(dm.struct, dev_prompts, b, s, n, gbs, out, ws, ws_n, None, stream)
            host_out.copy_(out, non_blocking=True)

        with torch.cuda.stream(stream):
            e2e_step()
            stream.synchronize()
            a0, a1 = ev(), ev()
            a0.record(stream)
            for _ in range(args.e2e_steps):
                e2e_step()
            a1.record(stream)
        stream.synchronize()
        e_ms = max_over_ranks(a0.elapsed_time(a1) / args.e2e_steps)
        e2e = {"value": round(world * b * n / (e_ms / 1e3), 2), "unit": "tokens/s",
               "h2d_bytes_per_step": b * s * 4, "d2h_bytes_per_step": b * n * 4,
               "ms_per_step": round(e_ms, 2),
               "what": "flexq_generate end to end (prompt upload, prefill column, n-1 decode "
                       "columns, token download): generated tokens b*n per second"}
        fq.flexq_device_status(stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(p)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded splitmix64 draws; weights ~N(0,0.02) quantized to 4-bit)",
            "config": {"workload": workload_name(args), "layers": p["layers"], "h": p["h"],
                       "heads": p["heads"], "ffn": p["ffn"], "vocab": p["vocab"],
                       "global_batch": b * world, "gpu_batch": gbs, "seq_len": s,
                       "gen_tokens": n, "w_bits": p["w_bits"], "kv_bits": p["kv_bits"],
                       "embed_bits": p.get("embed_bits", 16),
                       "attn": (f"top-k sparse, {p['topk_permille'] / 10:g} % of keys"
                                if p.get("topk_permille") else "dense"),
                       "prefill_kv": "read back from the cache" if p.get("prefill_kv_cache") else "the pass's own",
                       "parallelism": f"replicas x{world}",
                       "step": "decode phase: n-1 decode columns x all layers + LM head",
                       "l2": "no flush: inputs far larger than L2 (weights + KV per step)"},
            "roofline": rl,
            "kernels": kernels,
            "prefill": {"ms": round(prefill_ms, 2),
                        "tokens_per_s": round(world * b * s / (prefill_ms / 1e3), 1),
                        "kernels": prefill_kernels,
                        "frac_of_ceiling": round(world * b * s / (prefill_ms / 1e3)
                                                 / (world * ceil["prefill_tokens_per_s"]), 4)},
            "ceiling": {"decode_tokens_per_s": round(world * ceil["decode_tokens_per_s"], 1),
                        "decode_frac": round(value / (world * ceil["decode_tokens_per_s"]), 4),
                        "prefill_tokens_per_s": round(world * ceil["prefill_tokens_per_s"], 1),
                        "what": "every launched kernel at its own roofline (algorithmic bytes at the "
                                "measured HBM copy rate or flops at the measured sustained dense rate, "
                                "whichever is slower), summed over the step"},
            "codec": codec,
            "gpu_launches": int(launches),
            "gpu_launches_per_step": int(launches // max(1, args.steps)),
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "setup_s": round(setup_s, 1),
            "kernel_sources": csrc_hash(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_h2d_gbps(torch, stream, nbytes=1 << 30, reps=5):
    """Page-locked host to device copy rate (GB/s), CUDA events on `stream`."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    with torch.cuda.stream(stream):
        dst.copy_(src, non_blocking=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            dst.copy_(src, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    return nbytes * reps / (e0.elapsed_time(e1) / 1e3) / 1e9


def run_offload(args, p):
    """Decode throughput with the layer weights in page-locked host memory:
    the block (GPU batch x GPU batches) chosen by the library's cost model
    from the measured host-to-device rate and the measured device peaks; one
    step = one flexq_generate_offload (prefill column + n-1 decode columns),
    decode tokens/s from its device-timed decode phase."""
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    from quantized_opt_decode_b200 import build
    build.build()
    from quantized_opt_decode_b200 import flexq as fq
    from quantized_opt_decode_b200.device_model import DeviceModel, workspace
    fq.flexq_set_launch_overlap(not args.no_launch_overlap)

    s, n = p["s"], p["n"]
    stream, copy = torch.cuda.Stream(), torch.cuda.Stream()
    h2d = measure_h2d_gbps(torch, copy)
    t_setup = time.perf_counter()
    with torch.cuda.stream(stream):
        dm = DeviceModel(p, b=0, max_len=s + n, stream=stream, with_kv=False, offload=True)
    stream.synchronize()
    torch.cuda.empty_cache()
    peaks = load_peaks()
    free, _ = torch.cuda.mem_get_info()
    hw = fq.flexq_hw(h2d_gbps=h2d, hbm_gbps=peaks["hbm_gbs"], tensor_tflops=peaks["bf16_tflops_sustained"],
                     device_bytes=free - 6e9)
    ch = fq.flexq_offload_plan(dm.struct, s, n, hw, args.max_block)
    gbs, b = ch.gpu_batch, ch.gpu_batch * ch.num_batches
    dm.alloc_kv(b, s + n)
    prompts = torch.empty(b, s, dtype=torch.int32, device="cuda")
    fq.flexq_synth_tokens(prompts, b * s, synth.config_seed(p), synth.TID_PROMPT, p["vocab"], stream=stream)
    out = torch.zeros(b, n, dtype=torch.int32, device="cuda")
    ws_n = fq.flexq_generate_workspace(dm.struct, b, s, gbs)
    ws = workspace(ws_n)
    slot = fq.flexq_offload_slot_bytes(dm.cfg)
    slots = workspace(2 * slot)
    stream.synchronize()
    setup_s = time.perf_counter() - t_setup

    def step():
        t = fq.flexq_timing()
        fq.flexq_generate_offload(dm.struct, slots, 2 * slot, copy, prompts, b, s, n, gbs, out, ws, ws_n, t, stream)
        return t.prefill_ms, t.decode_ms

    for _ in range(args.warmup):
        step()
    fq.flexq_device_status(stream)
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        torch.cuda.synchronize()
        l0 = fq.flexq_launch_count()
        times = [step() for _ in range(args.steps)]
        launches = fq.flexq_launch_count() - l0
    fq.flexq_device_status(stream)
    pre = sum(t[0] for t in times) / len(times)
    dec = sum(t[1] for t in times) / len(times)
    w_bytes = sum(dm.layers[0].t[k].numel() * dm.layers[0].t[k].element_size() for k in
                  ("w_qkv", "w_o", "w_fc1", "w_fc2")) * p["layers"]
    line = {
        "metric": METRIC, "mode": "offloaded weights", "value": round(b * (n - 1) / (dec / 1e3), 2),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dec, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic (seeded splitmix64 draws; weights ~N(0,0.02) quantized to 4-bit)",
        "config": {"workload": workload_name(args) + "+offload", "layers": p["layers"], "h": p["h"],
                   "global_batch": b, "gpu_batch": gbs, "seq_len": s, "gen_tokens": n,
                   "w_bits": p["w_bits"], "kv_bits": p["kv_bits"],
                   "weights": f"page-locked host memory, {w_bytes / 1e9:.1f} GB, two device slots",
                   "step": "one flexq_generate_offload; value from its decode phase (n-1 columns)"},
        "plan": {"gpu_batch": gbs, "num_batches": ch.num_batches, "max_block": args.max_block,
                 "modelled_decode_tokens_per_s": round(ch.decode_tokens_per_s, 1),
                 "modelled_column_io_s": round(ch.column_io_s, 4),
                 "modelled_column_compute_s": round(ch.column_compute_s, 4),
                 "modelled_device_gb": round(ch.device_bytes / 1e9, 1),
                 "h2d_gbps_measured": round(h2d, 1)},
        "measured_column_ms": round(dec / (n - 1), 2),
        "link_frac": round(w_bytes / (dec / (n - 1) / 1e3) / (h2d * 1e9), 4),
        "generation_tokens_per_s": round(b * n / ((pre + dec) / 1e3), 2),
        "prefill_ms": round(pre, 1),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "setup_s": round(setup_s, 1),
        "kernel_sources": csrc_hash(),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="flexq", choices=["flexq", "reference"])
    ap.add_argument("--config", default="opt-30b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-codec", action="store_true")
    ap.add_argument("--offload", action="store_true",
                    help="layer weights in page-locked host memory, block chosen by the cost model")
    ap.add_argument("--max-block", type=int, default=288, help="largest block the offload plan may choose")
    ap.add_argument("--embed-bits", type=int, default=16, choices=[16, 4],
                    help="4: tied embedding / LM head stored group-wise 4-bit")
    ap.add_argument("--topk", type=int, default=0,
                    help="top-k sparse decode attention keeping ceil(L * TOPK / 1000) keys (100 = 10 %%)")
    ap.add_argument("--prefill-kv-cache", action="store_true",
                    help="prefill attention reads K/V back from the (4-bit) cache")
    ap.add_argument("--no-launch-overlap", action="store_true",
                    help="launch every kernel after its predecessor completes (no programmatic dependent launch)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    p = dict(synth.CONFIGS[args.config])
    if args.embed_bits != 16:
        p["embed_bits"] = args.embed_bits
    if args.topk:
        p["topk_permille"] = args.topk
    if args.prefill_kv_cache:
        p["prefill_kv_cache"] = True
    if args.impl == "reference":
        run_reference(args, p)
    elif args.offload:
        run_offload(args, p)
    else:
        run_flexq(args, p)


if __name__ == "__main__":
    main()
