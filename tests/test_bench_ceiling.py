"""The benchmark's step ceiling (every launched kernel at its own roofline,
summed over the step) against the closed form of the per-layer decode
ceiling: GEMMs max(12 h^2 B_w / BW, 24 b h^2 / P), attention b L 2h B_kv / BW,
plus the tied LM head max(2 V h / BW, 2 b V h / P) per column."""
import importlib.util
import os

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(spec)
spec.loader.exec_module(bench)

PEAKS = {"hbm_gbs": 6545.3, "bf16_tflops": 1661.0, "bf16_tflops_sustained": 1397.6, "source": "test"}


def _closed_form(p):
    """Decode tokens/s at the ceiling: per column, each of the l layers runs
    its GEMMs once per GPU batch (b / gpu_batch of them, weights re-read each
    time) and attends over the KV of all b sequences; the tied LM head runs
    once over the whole block."""
    BW, P = PEAKS["hbm_gbs"] * 1e9, PEAKS["bf16_tflops_sustained"] * 1e12
    b, gbs, s, n, l, h, V = p["b"], p["gpu_batch"], p["s"], p["n"], p["layers"], p["h"], p["vocab"]
    nb = b // gbs
    bw = 0.5625 if p["w_bits"] == 4 else 2.0
    bkv = 0.5625 if p["kv_bits"] == 4 else 2.0
    t = 0.0
    for j in range(1, n):
        L = s + j + 1
        gemm = nb * max(12 * h * h * bw / BW, 24 * gbs * h * h / P)
        t += l * (gemm + b * L * 2 * h * bkv / BW) + max(2 * V * h / BW, 2 * b * V * h / P)
    return b * (n - 1) / t


def test_decode_ceiling_matches_closed_form():
    for name in ("opt-1.3b", "opt-6.7b", "opt-30b", "opt-30b-s1024", "opt-175b"):
        p = dict(synth.CONFIGS[name])
        got = bench.step_ceilings(p, p["gpu_batch"], PEAKS)["decode_tokens_per_s"]
        want = _closed_form(p)
        # the closed form leaves out activations, LayerNorm, the append and the argmax
        assert 0.93 * want < got <= want, (name, got, want)


def test_phase_work_counts_final_layernorm_over_the_block():
    """The final LayerNorm shares its profiler kind with the layer norms but
    covers all b rows, the layer norms one GPU batch each."""
    p = dict(synth.CONFIGS["opt-6.7b"])
    gbs, b, h, l = p["gpu_batch"], p["b"], p["h"], p["layers"]
    cols = p["n"] - 1
    calls = cols * (2 * l * (b // gbs) + 1)
    byts, _ = bench.phase_work(p, "layernorm", calls, gbs, "decode", cols)
    per_row = 4 * h
    want = cols * (2 * l * (b // gbs) * (gbs * per_row + 4 * h) + (b * per_row + 4 * h))
    assert byts == want


def test_prefill_ceiling_is_tensor_bound_at_30b():
    p = dict(synth.CONFIGS["opt-30b"])
    b, s, h, l = p["b"], p["s"], p["h"], p["layers"]
    flops = l * (24 * b * s * h * h + 2 * b * s * s * h)
    want = b * s / (flops / (PEAKS["bf16_tflops_sustained"] * 1e12))
    got = bench.step_ceilings(p, p["gpu_batch"], PEAKS)["prefill_tokens_per_s"]
    assert 0.95 * want < got <= want, (got, want)
