"""GPU parity of whole layer steps and of generation against the oracle.

Layer steps (prefill over b x s tokens, then decode of one token) on the tiny
configuration and on a d = 128 variant, 4-bit and fp16 weights/KV, against the
oracle with the LN1 output rounded to fp16 (the projection input of a layer
that computes in fp16, as for every shape): max relative Frobenius error 2e-3
on the layer output and the element-wise bound of gpu_helpers.assert_close,
and on the layer's residual branch
(y - x) a bound of 2e-3 relative to the output norm as well.  Cached codes are
compared element by element: the K/V rows come out of a GEMM on each side, so
a value sitting on a rounding boundary may land one code apart; at least 99%
must be identical and none may differ by more than one step.

Generation: tokens are a greedy choice, several of which can be right when two
logits tie within rounding, so each GPU token is checked against the oracle
run teacher-forced on the GPU's own tokens: it must be the oracle's argmax or
within 2e-3 * max|logit| of it."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import synth  # noqa: E402
from oracle import opt  # noqa: E402
from gpu_helpers import assert_close, fq, rel_fro, to_dev, to_host  # noqa: E402
from quantized_opt_decode_b200.device_model import DeviceModel, workspace  # noqa: E402

TOL = 2e-3


def _preset(name, **over):
    p = dict(synth.CONFIGS[name])
    p.update(over)
    return p


def _layer_roundtrip(p, b, s):
    """Runs prefill then one decode through layer 0 on both sides."""
    dm = DeviceModel(p, b=b, max_len=s + 4, layers=1)
    cfg = opt.Config.from_preset(p, ln1_f16=True)
    seed = synth.config_seed(p)
    W = opt.effective_layer(cfg, opt.raw_layer(cfg, seed, 0))
    rng = np.random.default_rng(b * s + p["h"])
    x = rng.standard_normal((b, s, p["h"])).astype(np.float16)
    t = rng.standard_normal((b, p["h"])).astype(np.float16)
    h = p["h"]
    ws_n = max(fq.flexq_layer_workspace(dm.cfg, b * s, 0), fq.flexq_layer_workspace(dm.cfg, b, 1))
    ws = workspace(ws_n)
    xd = to_dev(x.reshape(b * s, h))
    yd = torch.empty_like(xd)
    L, kv = dm.layers[0].struct, dm.kv[0].struct
    fq.flexq_layer_prefill(dm.cfg, L, xd, yd, kv, b, s, ws, ws_n)
    td = to_dev(t)
    t2 = torch.empty_like(td)
    fq.flexq_layer_decode(dm.cfg, L, td, t2, kv, b, s, ws, ws_n)
    fq.flexq_device_status()
    y_ref, K16, V16 = opt.layer_prefill(cfg, W, x.astype(np.float64))
    cache = opt.KVCache(cfg, b, s + 4, cfg.kv_bits)
    cache.write("k", K16, 0)
    cache.write("v", V16, 0)
    t_ref = opt.layer_decode(cfg, W, t.astype(np.float64), cache, s)
    return dm, (to_host(yd).reshape(b, s, h), y_ref, x), (to_host(t2), t_ref, t), cache


def _check_out(got, ref, x):
    assert_close(got, ref, TOL)
    branch = np.linalg.norm(got.astype(np.float64) - ref) / np.linalg.norm(ref - x.astype(np.float64))
    assert branch < 1e-2, branch  # error relative to the layer's own contribution


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("tiny16", {}),
    ("tiny", dict(h=512, heads=4, ffn=2048)),      # d = 128
    ("tiny16", dict(h=512, heads=4, ffn=2048)),
    ("tiny", dict(prefill_kv_cache=True)),         # prefill attention reads the 4-bit cache back
    ("tiny", dict(h=512, heads=4, ffn=2048, prefill_kv_cache=True)),
    ("tiny16", dict(prefill_kv_cache=True)),
])
def test_layer_prefill_and_decode(name, over):
    p = _preset(name, **over)
    dm, (y, y_ref, x), (t2, t_ref, t), cache = _layer_roundtrip(p, b=4, s=32)
    _check_out(y, y_ref, x)
    _check_out(t2, t_ref, t)
    # cached K: element-wise comparison of codes (or fp16 values)
    b, s, a, d = 4, 32, p["heads"], p["h"] // p["heads"]
    if p["kv_bits"] == 4:
        kc = to_host(dm.kv[0].k).reshape(b, a, s + 4, d // 2)
        got = np.stack([kc & 15, kc >> 4], -1).astype(int)
        oc = cache.t["k_codes"]
        want = np.stack([oc & 15, oc >> 4], -1).astype(int)
        diff = np.abs(got[:, :, :s + 1] - want[:, :, :s + 1])
        assert diff.max() <= 1 and (diff == 0).mean() > 0.99
    else:
        kc = to_host(dm.kv[0].k).reshape(b, a, s + 4, d).astype(np.float64)
        assert rel_fro(kc[:, :, :s + 1], cache.t["k"][:, :, :s + 1].astype(np.float64)) < TOL


@pytest.mark.parametrize("name,over", [("tiny", {}), ("tiny16", {}),
                                       ("tiny", dict(embed_bits=4)),        # 4-bit tied embedding / LM head
                                       ("tiny", dict(topk_permille=100)),   # top-10 % sparse decode attention
                                       ("tiny", dict(prefill_kv_cache=True))])  # prefill reads the 4-bit cache
def test_generate_tokens_valid_under_oracle(name, over):
    p = _preset(name, **over)
    b, s, n = p["b"], p["s"], p["n"]
    dm = DeviceModel(p, b=b, max_len=s + n)
    seed = synth.config_seed(p)
    prompts = synth.tokens(seed, synth.TID_PROMPT, b * s, p["vocab"]).reshape(b, s)
    out = torch.zeros(b, n, dtype=torch.int32, device="cuda")
    ws_n = fq.flexq_generate_workspace(dm.struct, b, s, p["gpu_batch"])
    ws = workspace(ws_n)
    timing = fq.flexq_timing()
    fq.flexq_generate(dm.struct, to_dev(prompts), b, s, n, p["gpu_batch"], out, ws, ws_n, timing)
    fq.flexq_device_status()
    toks = to_host(out)
    m = opt.build_model(opt.Config.from_preset(p, ln1_f16=True), seed, s + n)
    own, _ = opt.generate(m, prompts, n)
    _, logits = opt.generate(m, prompts, n, forced=toks)
    for j in range(n):
        for i in range(b):
            lg = logits[j, i]
            assert lg[toks[i, j]] >= lg.max() - 2e-3 * np.abs(lg).max(), (i, j)
    assert (toks == own).mean() > 0.5
    assert timing.prefill_ms > 0 and timing.decode_ms > 0


def test_block_schedule_gpu_batches_agree():
    """The zig-zag block order with GPU batches of b, b/2 and b/4 sequences
    produces the same tokens (sequences are independent)."""
    p = _preset("tiny", b=8)
    b, s, n = 8, p["s"], 6
    dm = DeviceModel(p, b=b, max_len=s + n)
    seed = synth.config_seed(p)
    prompts = to_dev(synth.tokens(seed, synth.TID_PROMPT, b * s, p["vocab"]).reshape(b, s))
    results = []
    for gbs in (8, 4, 2):
        out = torch.zeros(b, n, dtype=torch.int32, device="cuda")
        ws_n = fq.flexq_generate_workspace(dm.struct, b, s, gbs)
        ws = workspace(ws_n)
        fq.flexq_generate(dm.struct, prompts, b, s, n, gbs, out, ws, ws_n)
        results.append(to_host(out))
    assert np.array_equal(results[0], results[1]) and np.array_equal(results[0], results[2])


def test_sequence_subset_matches_block():
    """A GPU batch run alone yields the tokens it yields inside the block."""
    p = _preset("tiny", b=4)
    b, s, n = 4, p["s"], 5
    dm = DeviceModel(p, b=b, max_len=s + n)
    seed = synth.config_seed(p)
    pr = synth.tokens(seed, synth.TID_PROMPT, b * s, p["vocab"]).reshape(b, s)
    out = torch.zeros(b, n, dtype=torch.int32, device="cuda")
    ws_n = fq.flexq_generate_workspace(dm.struct, b, s, b)
    ws = workspace(ws_n)
    fq.flexq_generate(dm.struct, to_dev(pr), b, s, n, b, out, ws, ws_n)
    full = to_host(out)
    out2 = torch.zeros(2, n, dtype=torch.int32, device="cuda")
    fq.flexq_generate(dm.struct, to_dev(pr[1:3]), 2, s, n, 2, out2, ws, ws_n)
    assert np.array_equal(to_host(out2), full[1:3])


@pytest.mark.parametrize("name,over,b", [
    ("tiny", {}, 5),
    ("tiny", dict(h=512, heads=4, ffn=2048), 3),     # d = 128
    ("tiny16", {}, 5),
    ("tiny", dict(h=512, heads=8, ffn=1024), 37),    # three 16-token chunks, the last ragged
])
def test_fused_decode_append_bit_exact(name, over, b):
    """The decode step appends the token's K/V from inside the QKV projection
    (quantize on append in its epilogue).  The cache slot it writes must be
    exactly what the oracle's quantizer makes of the fp16 K/V rows of the
    same projection run unfused (LayerNorm, then the linear layer alone: same
    kernel, same K split, so the same fp16 rows); fp16 caches hold those rows."""
    from gpu_helpers import v_words_to_canonical
    from oracle import q64
    p = _preset(name, **over)
    h, a = p["h"], p["heads"]
    d = h // a
    pos = 11
    dm = DeviceModel(p, b=b, max_len=pos + 3, layers=1)
    rng = np.random.default_rng(b + h)
    t = rng.standard_normal((b, h)).astype(np.float16)
    td = to_dev(t)
    t2 = torch.empty_like(td)
    ws_n = fq.flexq_layer_workspace(dm.cfg, b, 1)
    ws = workspace(ws_n)
    L, kv = dm.layers[0].struct, dm.kv[0].struct
    fq.flexq_layer_decode(dm.cfg, L, td, t2, kv, b, pos, ws, ws_n)
    fq.flexq_device_status()
    # unfused: LN1, then the QKV linear layer alone
    lw = dm.layers[0].t
    u = torch.empty_like(td)
    fq.flexq_layernorm(td, h, lw["ln1_g"], lw["ln1_b"], u, h, b, h, 1e-5)
    qkv = torch.empty(b, 3 * h, dtype=torch.float16, device="cuda")
    lin_ws = fq.flexq_linear_workspace(b, 3 * h, h, p["w_bits"], 0)
    lws = workspace(lin_ws)
    fq.flexq_linear(u, h, lw["w_qkv"], p["w_bits"], b, 3 * h, h, lw["b_qkv"], None, 0, fq.EPI_BIAS, qkv, 3 * h,
                    lws, lin_ws, 0)
    rows = to_host(qkv)
    K = rows[:, h:2 * h].reshape(b, a, d)
    V = rows[:, 2 * h:].reshape(b, a, d)
    L_ = pos + 3
    if p["kv_bits"] == 4:
        kc = to_host(dm.kv[0].k).reshape(b, a, L_, d // 2)[:, :, pos]
        km = to_host(dm.kv[0].k_meta).reshape(b, a, L_, d // 64, 2)[:, :, pos]
        vm = to_host(dm.kv[0].v_meta).reshape(b, a, L_, d // 64, 2)[:, :, pos]
        vc = v_words_to_canonical(to_host(dm.kv[0].v), b, a, L_, d)[:, :, pos]
        for got_c, got_m, rows16 in ((kc, km, K), (vc, vm, V)):
            c, m, s = q64.quantize_rows(rows16)
            assert np.array_equal(got_c, c)
            assert np.array_equal(got_m[..., 0].view(np.uint16), m.view(np.uint16))
            assert np.array_equal(got_m[..., 1].view(np.uint16), s.view(np.uint16))
    else:
        kc = to_host(dm.kv[0].k).reshape(b, a, L_, d)[:, :, pos]
        vc = to_host(dm.kv[0].v).reshape(b, a, L_, d)[:, :, pos]
        assert np.array_equal(kc.view(np.uint16), K.view(np.uint16))
        assert np.array_equal(vc.view(np.uint16), V.view(np.uint16))


@pytest.mark.parametrize("name,over,b,length", [
    ("tiny", dict(h=512, heads=4, ffn=1024), 2, 1100),   # d = 128, cache split over 5 CTAs
    ("tiny", {}, 3, 1056),                                # d = 64
    ("tiny", dict(h=512, heads=4, ffn=1024), 1, 300),     # a ragged 128-token chunk per split
])
def test_layer_decode_long_cache(name, over, b, length):
    """Decode over a long 4-bit cache with so few (sequence, head) pairs that
    the attention splits each head's cache across CTAs and merges the partial
    softmax results.  The cache is filled from seeded fp16 rows on both sides
    through the quantizer (bit-exact), then one decode step appends slot
    `length` and attends over length + 1 slots."""
    p = _preset(name, **over)
    h = p["h"]
    cfg = opt.Config.from_preset(p, ln1_f16=True)
    seed = synth.config_seed(p)
    W = opt.effective_layer(cfg, opt.raw_layer(cfg, seed, 0))
    dm = DeviceModel(p, b=b, max_len=length + 2, layers=1)
    rng = np.random.default_rng(length + b)
    rows = rng.standard_normal((b * length, 2 * h)).astype(np.float16)
    t = rng.standard_normal((b, h)).astype(np.float16)
    rd = to_dev(rows)
    kv = dm.kv[0].struct
    fq.flexq_kv_append(dm.cfg, kv, rd[:, :h], rd[:, h:], 2 * h, b, 0, length)
    ws_n = fq.flexq_layer_workspace(dm.cfg, b, 1)
    ws = workspace(ws_n)
    td = to_dev(t)
    t2 = torch.empty_like(td)
    fq.flexq_layer_decode(dm.cfg, dm.layers[0].struct, td, t2, kv, b, length, ws, ws_n)
    fq.flexq_device_status()
    cache = opt.KVCache(cfg, b, length + 2, 4)
    cache.write("k", rows[:, :h].reshape(b, length, h), 0)
    cache.write("v", rows[:, h:].reshape(b, length, h), 0)
    ref = opt.layer_decode(cfg, W, t.astype(np.float64), cache, length)
    _check_out(to_host(t2), ref, t)


def test_layer_decode_topk_sparse_attention():
    """A decode step whose attention keeps the top 10 % of the cache (the
    configuration's attn_topk_permille), against the oracle's decode with the
    same option."""
    p = _preset("tiny", h=512, heads=4, ffn=1024, topk_permille=100)
    h, b, length = p["h"], 3, 700
    cfg = opt.Config.from_preset(p, ln1_f16=True)
    seed = synth.config_seed(p)
    W = opt.effective_layer(cfg, opt.raw_layer(cfg, seed, 0))
    dm = DeviceModel(p, b=b, max_len=length + 2, layers=1)
    rng = np.random.default_rng(71)
    rows = rng.standard_normal((b * length, 2 * h)).astype(np.float16)
    t = rng.standard_normal((b, h)).astype(np.float16)
    rd = to_dev(rows)
    kv = dm.kv[0].struct
    fq.flexq_kv_append(dm.cfg, kv, rd[:, :h], rd[:, h:], 2 * h, b, 0, length)
    ws_n = fq.flexq_layer_workspace(dm.cfg, b, 1)
    ws = workspace(ws_n)
    td = to_dev(t)
    t2 = torch.empty_like(td)
    fq.flexq_layer_decode(dm.cfg, dm.layers[0].struct, td, t2, kv, b, length, ws, ws_n)
    fq.flexq_device_status()
    cache = opt.KVCache(cfg, b, length + 2, 4)
    cache.write("k", rows[:, :h].reshape(b, length, h), 0)
    cache.write("v", rows[:, h:].reshape(b, length, h), 0)
    ref = opt.layer_decode(cfg, W, t.astype(np.float64), cache, length)
    _check_out(to_host(t2), ref, t)


@pytest.mark.parametrize("gbs", [4, 2])
def test_offloaded_weights_match_resident(gbs):
    """Generation with the layer weights in page-locked host memory, copied
    into two device slots on a second stream ahead of the compute, gives the
    tokens of the resident run bit for bit (same kernels, same weights; only
    where the weights come from differs)."""
    p = _preset("tiny", b=4)
    b, s, n = 4, p["s"], 6
    seed = synth.config_seed(p)
    prompts = to_dev(synth.tokens(seed, synth.TID_PROMPT, b * s, p["vocab"]).reshape(b, s))
    res = DeviceModel(p, b=b, max_len=s + n)
    off = DeviceModel(p, b=b, max_len=s + n, offload=True)
    assert off.layers[0].t["w_qkv"].device.type == "cpu" and off.layers[0].t["w_qkv"].is_pinned()
    ws_n = fq.flexq_generate_workspace(res.struct, b, s, gbs)
    ws = workspace(ws_n)
    out_r = torch.zeros(b, n, dtype=torch.int32, device="cuda")
    fq.flexq_generate(res.struct, prompts, b, s, n, gbs, out_r, ws, ws_n)
    slot = fq.flexq_offload_slot_bytes(off.cfg)
    slots = workspace(2 * slot)
    copy = torch.cuda.Stream()
    out_o = torch.zeros(b, n, dtype=torch.int32, device="cuda")
    timing = fq.flexq_timing()
    fq.flexq_generate_offload(off.struct, slots, 2 * slot, copy, prompts, b, s, n, gbs, out_o, ws, ws_n, timing)
    fq.flexq_device_status()
    assert np.array_equal(to_host(out_o), to_host(out_r))
    assert timing.prefill_ms > 0 and timing.decode_ms > 0
    # weights that are not page-locked host memory are refused
    with pytest.raises(fq.FlexqError) as ei:
        fq.flexq_generate_offload(res.struct, slots, 2 * slot, copy, prompts, b, s, n, gbs, out_o, ws, ws_n)
    assert ei.value.status == 1 and "page-locked" in str(ei.value)


def test_layer_decode_long_fp16_cache():
    """The fp16-cache decode attention over a long cache split across CTAs
    (b * heads = 4 pairs), against the oracle's decode on the same fp16 rows."""
    p = _preset("tiny16", h=256, heads=4, ffn=1024)
    h, b, length = p["h"], 1, 900
    cfg = opt.Config.from_preset(p, ln1_f16=True)
    seed = synth.config_seed(p)
    W = opt.effective_layer(cfg, opt.raw_layer(cfg, seed, 0))
    dm = DeviceModel(p, b=b, max_len=length + 2, layers=1)
    rng = np.random.default_rng(91)
    rows = rng.standard_normal((b * length, 2 * h)).astype(np.float16)
    t = rng.standard_normal((b, h)).astype(np.float16)
    rd = to_dev(rows)
    kv = dm.kv[0].struct
    fq.flexq_kv_append(dm.cfg, kv, rd[:, :h], rd[:, h:], 2 * h, b, 0, length)
    ws_n = fq.flexq_layer_workspace(dm.cfg, b, 1)
    ws = workspace(ws_n)
    td = to_dev(t)
    t2 = torch.empty_like(td)
    fq.flexq_layer_decode(dm.cfg, dm.layers[0].struct, td, t2, kv, b, length, ws, ws_n)
    fq.flexq_device_status()
    cache = opt.KVCache(cfg, b, length + 2, 16)
    cache.write("k", rows[:, :h].reshape(b, length, h), 0)
    cache.write("v", rows[:, h:].reshape(b, length, h), 0)
    ref = opt.layer_decode(cfg, W, t.astype(np.float64), cache, length)
    _check_out(to_host(t2), ref, t)
