"""Host logic of the offloaded block schedule's cost model
(flexq_offload_plan): it runs without a GPU, so it is checked here on the
benchmark shapes for the properties the model implies ("FlexGen" walk-through,
sections "Search Space" and "Cost Model": per column and layer the time is the
larger of the weight copy and the block's compute; a larger block amortises
the copy until memory runs out)."""
import ctypes as C

import pytest

import synth

fq = pytest.importorskip("quantized_opt_decode_b200.flexq")


def _model(name, embed_bits=16):
    p = synth.CONFIGS[name]
    cfg = fq.flexq_config(h=p["h"], heads=p["heads"], ffn=p["ffn"], w_bits=p["w_bits"], kv_bits=p["kv_bits"],
                          ln_eps=1e-5)
    ptrs = [0x10000 * (i + 1) for i in range(12)]
    layers = (fq.flexq_layer * p["layers"])(*[fq.flexq_layer(*ptrs) for _ in range(p["layers"])])
    kv = (fq.flexq_kv * p["layers"])()
    m = fq.flexq_model(cfg, p["layers"], p["vocab"], p["s"] + p["n"], layers, kv, 0x1000, 0x2000, 0x3000,
                       0x4000, embed_bits)
    m._keep = (layers, kv)
    return p, m


def _mem(m, p, b, gbs):
    """Device bytes of a block of b sequences, as the header states them."""
    cfg = m.cfg
    kv = p["layers"] * fq._lib.flexq_kv_bytes(C.byref(cfg), b, p["s"] + p["n"])
    return kv + fq._lib.flexq_generate_workspace(C.byref(m), b, p["s"], gbs)


def test_io_bound_plan_fills_memory():
    """Over a slow host link every column waits for the weights, so the best
    block is as large as memory allows (within one GPU batch of the limit)."""
    p, m = _model("opt-30b")
    hw = fq.flexq_hw(h2d_gbps=50.0, hbm_gbps=6545.0, tensor_tflops=1397.0, device_bytes=170e9)
    ch = fq.flexq_offload_plan(m, p["s"], p["n"], hw, 100000)
    b = ch.gpu_batch * ch.num_batches
    assert ch.device_bytes <= hw.device_bytes
    assert ch.column_io_s > ch.column_compute_s  # copy-bound
    assert _mem(m, p, b + ch.gpu_batch, ch.gpu_batch) > hw.device_bytes - 2e9
    # weights of 48 layers at 50 GB/s per column
    w = sum(fq.flexq_packed_weight_bytes(no, ki) for no, ki in
            ((3 * p["h"], p["h"]), (p["h"], p["h"]), (p["ffn"], p["h"]), (p["h"], p["ffn"])))
    assert abs(ch.column_io_s - p["layers"] * w / 50e9) < 1e-9 * p["layers"]
    # every layer waits for its copy: a column is the copies plus the LM head
    assert ch.decode_tokens_per_s == pytest.approx(b / (ch.column_io_s + _head(p, m, hw, b)), rel=1e-9)


def _head(p, m, hw, b):
    e = p["vocab"] * p["h"] * 2 if m.embed_bits == 16 else fq.flexq_packed_weight_bytes(p["vocab"], p["h"])
    return max(e / (hw.hbm_gbps * 1e9), 2.0 * b * p["vocab"] * p["h"] / (hw.tensor_tflops * 1e12))


def test_fast_link_plan_is_compute_bound_and_respects_max_block():
    p, m = _model("opt-30b")
    hw = fq.flexq_hw(h2d_gbps=1e6, hbm_gbps=6545.0, tensor_tflops=1397.0, device_bytes=170e9)
    ch = fq.flexq_offload_plan(m, p["s"], p["n"], hw, 1024)
    assert ch.column_compute_s > ch.column_io_s
    assert ch.gpu_batch * ch.num_batches <= 1024
    small = fq.flexq_offload_plan(m, p["s"], p["n"], hw, 64)
    assert small.gpu_batch * small.num_batches <= 64
    assert small.decode_tokens_per_s <= ch.decode_tokens_per_s


def test_more_memory_never_lowers_the_modelled_throughput():
    p, m = _model("opt-175b")
    last = 0.0
    for gb in (40e9, 80e9, 160e9):
        hw = fq.flexq_hw(h2d_gbps=50.0, hbm_gbps=6545.0, tensor_tflops=1397.0, device_bytes=gb)
        ch = fq.flexq_offload_plan(m, p["s"], p["n"], hw, 100000)
        assert ch.decode_tokens_per_s >= last and ch.device_bytes <= gb
        last = ch.decode_tokens_per_s


def test_plan_rejects_impossible_requests():
    p, m = _model("opt-30b")
    hw = fq.flexq_hw(h2d_gbps=50.0, hbm_gbps=6545.0, tensor_tflops=1397.0, device_bytes=1e9)
    with pytest.raises(fq.FlexqError) as ei:
        fq.flexq_offload_plan(m, p["s"], p["n"], hw, 1000)
    assert ei.value.status == 1 and "fits" in str(ei.value)
    hw.device_bytes = 170e9
    hw.h2d_gbps = 0.0
    with pytest.raises(fq.FlexqError):
        fq.flexq_offload_plan(m, p["s"], p["n"], hw, 1000)
