"""Parity at the full sizes of the five benchmark shapes, in the launch
configuration the benchmark times.

For each shape (OPT-1.3B fp16 W+KV, OPT-6.7B / OPT-30B / OPT-175B 4-bit W+KV,
and OPT-30B at a 1024-token prompt) one decoder layer at full width runs a
prefill over a whole GPU batch of prompt-length sequences and then one decode
step for the whole GPU batch, exactly the kernels and shapes of the benchmark's
prefill and decode columns.

The float64 oracle (with the LN1 output rounded to fp16, the projection input
of a layer that computes in fp16; the same reading for every shape) evaluates
sampled outputs, since a whole GPU batch at these widths would take it hours:
the first, a middle and the last sequence of the batch, each at three prompt
positions (first, middle, last), their cached K codes after the prefill, and
their decode outputs and appended K codes.  Every output feature is checked
for each sampled sequence.  At these sizes the token tiles are full (b*s and
b are multiples of the token tile), so ragged tiles are covered by the
small-shape tests; what covers the other sequences here is a property that
holds at any size: the kernels treat sequences independently and identically,
so running the batch with its sequences rotated must give the rotated outputs
(prefill rotated by one sequence, decode by 17 sequences, which moves every
token to another 16-token chunk of the GEMM epilogue), equal up to the order
in which split tiles sum their fp32 partials (8 ulps + 1e-3 of the rms).

The decode step reads a cache that both sides fill from the same seeded fp16
K/V rows through the quantizer (bit-exact, as the KV-append tests show):
after a prefill each side quantizes its own GEMM output, and a code that lands
one step apart moves a 4-bit element by a whole quantization step, more than
the layer tolerance.  The prefill's cache is checked code by code instead.

Inputs are seeded draws of the shared generator, made on the device for the
GPU and regenerated on the host, for the sampled sequences only, for the
oracle.  Bars: layer outputs within 2e-3 relative Frobenius error, every
element within the element-wise bound of gpu_helpers.assert_close, and within
1e-2 of the layer's own contribution (y - x); cached codes at least 99 %
identical and never more than one step apart; fp16 caches within 2e-3.  The
decode output is also held against the plain float64 oracle (LN1 not rounded
to fp16) within 5e-2 relative Frobenius error (OPT-175B was 2.1 % off it), so
both readings' gaps are tracked."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import synth  # noqa: E402
from oracle import opt, q64  # noqa: E402
from gpu_helpers import assert_close, fq, rel_fro, to_host, ulp16  # noqa: E402
from quantized_opt_decode_b200.device_model import DeviceModel, workspace  # noqa: E402

TOL = 2e-3
TID_X = synth.TID_TEST_BASE + 11  # prefill inputs [gpu_batch * s][h]
TID_T = synth.TID_TEST_BASE + 12  # decode inputs [gpu_batch][h]
TID_KV = synth.TID_TEST_BASE + 13  # cache rows for the decode [gpu_batch * s][K | V]
ROLL_DECODE = 17
PLAIN_GAP = 5e-2  # decode output against the plain float64 oracle (relative Frobenius error)


def _oracle_weights(cfg, seed):
    """Layer 0's weights as the oracle computes with them: the dequantized 4-bit
    codes (exact in fp16, held as float32 to keep host memory near 10 GB at
    OPT-175B width; every product is still formed in float64) or the fp16
    values.  Tensors are drawn one at a time, and the quantizer runs on blocks
    of whole rows (its groups lie inside a row, so blocks give the same codes)."""
    W = {}
    for name in synth.LAYER_TENSORS:
        shape, sigma, mean = synth.layer_tensor_spec(name, cfg.h, cfg.ffn)
        v = synth.normal_f16(seed, synth.layer_tensor_id(0, name), int(np.prod(shape)), sigma, mean).reshape(shape)
        if name in opt.LINEAR and cfg.w_bits == 4:
            out = np.empty(shape, np.float32)
            for r0 in range(0, shape[0], 2048):
                out[r0:r0 + 2048] = q64.roundtrip(v[r0:r0 + 2048])
            W[name] = out
        elif name in opt.LINEAR:
            W[name] = v.astype(np.float32)
        else:
            W[name] = v.astype(np.float64)
        del v
    return W


def _check_out(got, ref, x, what):
    got = got.astype(np.float64)
    assert_close(got, ref, TOL, what=what)
    branch = np.linalg.norm(got - ref) / np.linalg.norm(ref - x)
    assert branch < 1e-2, (what, branch)


def _check_codes(got_codes, want_codes, what):
    g = np.stack([got_codes & 15, got_codes >> 4], -1).astype(int)
    w = np.stack([want_codes & 15, want_codes >> 4], -1).astype(int)
    diff = np.abs(g - w)
    assert diff.max() <= 1 and (diff == 0).mean() > 0.99, (what, (diff == 0).mean(), diff.max())


def _check_rotation(rot, ref, what):
    """Rotating the batch rotates the outputs.  Where a linear layer splits
    a tile's K range across CTAs (stream-K), the split points depend on the
    tile, so a row that moves to another tile may sum its fp32 partials in
    another order, and the difference passes through LayerNorm, GELU and a
    second split GEMM: allow 8 fp16 ulps plus 1e-3 of the rms, far below the
    O(1) error of a misplaced or wrong row."""
    rot = rot.astype(np.float64)
    ref = ref.astype(np.float64)
    err = np.abs(rot - ref)
    bound = 8 * ulp16(ref) + 1e-3 * float(np.sqrt(np.mean(ref ** 2)))
    k = int(np.argmax(err - bound))
    assert (err <= bound).all(), f"{what} under rotation: element {k} off by {err.flat[k]:.3e}"


@pytest.mark.parametrize("name", ["opt-1.3b", "opt-6.7b", "opt-30b", "opt-30b-s1024", "opt-175b"])
def test_layer_full_size_sampled(name):
    p = dict(synth.CONFIGS[name])
    gb, s, h = p["gpu_batch"], p["s"], p["h"]
    cfg = opt.Config.from_preset(p, ln1_f16=True)
    a, d = cfg.heads, cfg.d
    seed = synth.config_seed(p)
    seqs = sorted({0, gb // 2, gb - 1})
    pos = [0, s // 2, s - 1]

    # ---- GPU: the whole GPU batch through layer 0
    dm = DeviceModel(p, b=gb, max_len=s + 1, layers=1)
    xd = torch.empty(gb * s, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(xd, gb * s * h, seed, TID_X, 0, 1.0, 0.0)
    td = torch.empty(gb, h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(td, gb * h, seed, TID_T, 0, 1.0, 0.0)
    yd = torch.empty_like(xd)
    t2 = torch.empty_like(td)
    ws_n = max(fq.flexq_layer_workspace(dm.cfg, gb * s, 0), fq.flexq_layer_workspace(dm.cfg, gb, 1))
    ws = workspace(ws_n)
    L, kv = dm.layers[0].struct, dm.kv[0].struct
    fq.flexq_layer_prefill(dm.cfg, L, xd, yd, kv, gb, s, ws, ws_n)
    fq.flexq_device_status()
    y_got = to_host(yd.view(gb, s, h)[seqs][:, pos])
    k_shape = (gb, a, s + 1, d // 2) if p["kv_bits"] == 4 else (gb, a, s + 1, d)
    k_pre = to_host(dm.kv[0].k).reshape(k_shape)[seqs, :, :s]
    # rotation by one sequence: the rotated outputs (up to split-tile summation order)
    y_rot = torch.empty_like(xd)
    fq.flexq_layer_prefill(dm.cfg, L, torch.roll(xd, s, 0), y_rot, kv, gb, s, ws, ws_n)
    fq.flexq_device_status()
    _check_rotation(to_host(torch.roll(y_rot, -s, 0)), to_host(yd), "prefill")
    del y_rot
    # the decode reads a cache filled from seeded rows on both sides
    kvd = torch.empty(gb * s, 2 * h, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(kvd, gb * s * 2 * h, seed, TID_KV, 0, 1.0, 0.0)
    fq.flexq_kv_append(dm.cfg, kv, kvd[:, :h], kvd[:, h:], 2 * h, gb, 0, s)
    fq.flexq_layer_decode(dm.cfg, L, td, t2, kv, gb, s, ws, ws_n)
    fq.flexq_device_status()
    t_got = to_host(t2[seqs])
    k_dec = to_host(dm.kv[0].k).reshape(k_shape)[seqs, :, s]
    # rotation of the decode batch (cache rows and tokens) by ROLL_DECODE sequences
    kv_rot = torch.roll(kvd, ROLL_DECODE * s, 0)
    fq.flexq_kv_append(dm.cfg, kv, kv_rot[:, :h], kv_rot[:, h:], 2 * h, gb, 0, s)
    t3 = torch.empty_like(td)
    fq.flexq_layer_decode(dm.cfg, L, torch.roll(td, ROLL_DECODE, 0), t3, kv, gb, s, ws, ws_n)
    fq.flexq_device_status()
    _check_rotation(to_host(torch.roll(t3, -ROLL_DECODE, 0)), to_host(t2), "decode")
    del dm, xd, yd, kvd, kv_rot, ws
    torch.cuda.empty_cache()

    # ---- oracle: the sampled sequences
    W = _oracle_weights(cfg, seed)
    rows, x_rows, k_rows = [], [], []
    for i in seqs:
        x = synth.normal_f16(seed, TID_X, s * h, 1.0, 0.0, start=i * s * h).reshape(s, h).astype(np.float64)
        u = opt.projection_input(cfg, W, x)
        qkv = opt.linear(u, W["w_qkv"], W["b_qkv"])
        Q, K, V = qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:]
        for pp in pos:
            q = Q[pp].reshape(1, a, d)
            kk = K[:pp + 1].reshape(1, pp + 1, a, d).transpose(0, 2, 1, 3)
            vv = V[:pp + 1].reshape(1, pp + 1, a, d).transpose(0, 2, 1, 3)
            rows.append(opt.attention_single(q, kk, vv).reshape(h))
            x_rows.append(x[pp])
        k_rows.append(K.astype(np.float16))
    x_pos = np.stack(x_rows)
    x_out = opt.linear(np.stack(rows), W["w_o"], W["b_o"]) + x_pos
    v2 = opt.layernorm(x_out, W["ln2_g"], W["ln2_b"], cfg.eps)
    y_ref = opt.linear(opt.gelu(opt.linear(v2, W["w_fc1"], W["b_fc1"])), W["w_fc2"], W["b_fc2"]) + x_out
    _check_out(y_got.reshape(-1, h), y_ref, x_pos, f"{name} prefill rows")

    # prefill cache of the sampled sequences, code by code
    cache = opt.KVCache(cfg, len(seqs), s + 1, cfg.kv_bits)
    cache.write("k", np.stack(k_rows), 0)
    if p["kv_bits"] == 4:
        _check_codes(k_pre, cache.t["k_codes"][:, :, :s], f"{name} prefill K codes")
    else:
        assert rel_fro(k_pre.astype(np.float64), cache.t["k"][:, :, :s].astype(np.float64)) < TOL

    # decode on the seeded cache; slot s holds the appended token's K
    kv_rows = np.stack([synth.normal_f16(seed, TID_KV, s * 2 * h, 1.0, 0.0, start=i * s * 2 * h).reshape(s, 2 * h)
                        for i in seqs])
    t = np.stack([synth.normal_f16(seed, TID_T, h, 1.0, 0.0, start=i * h) for i in seqs]).astype(np.float64)
    cache = opt.KVCache(cfg, len(seqs), s + 1, cfg.kv_bits)
    cache.write("k", kv_rows[:, :, :h], 0)
    cache.write("v", kv_rows[:, :, h:], 0)
    t_ref = opt.layer_decode(cfg, W, t, cache, s)
    _check_out(t_got, t_ref, t, f"{name} decode")
    # the plain float64 reading (LN1 not rounded before the projection): the
    # appended token's 4-bit codes may then be decided from a slightly
    # different K/V row, a quantization step on a few elements; tracked at a
    # looser relative bound on the output
    cache_plain = opt.KVCache(cfg, len(seqs), s + 1, cfg.kv_bits)
    cache_plain.write("k", kv_rows[:, :, :h], 0)
    cache_plain.write("v", kv_rows[:, :, h:], 0)
    cfg_plain = opt.Config.from_preset(p, ln1_f16=False)
    t_plain = opt.layer_decode(cfg_plain, W, t, cache_plain, s)
    gap = rel_fro(t_got.astype(np.float64), t_plain)
    assert gap < PLAIN_GAP, (name, gap)
    if p["kv_bits"] == 4:
        _check_codes(k_dec, cache.t["k_codes"][:, :, s], f"{name} appended K codes")
    else:
        assert rel_fro(k_dec.astype(np.float64), cache.t["k"][:, :, s].astype(np.float64)) < TOL
