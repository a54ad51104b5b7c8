"""GPU parity of the layer building blocks against the oracle on the same
seeded fp16 inputs: LayerNorm, the dequant-fused tcgen05 linear layers (4-bit
and fp16 weights, every epilogue, split K), the quantize-on-append KV write
(bit-exact), decode attention over the 4-bit / fp16 cache and causal prefill
attention.  Floating-point tolerance: 2e-3 relative Frobenius error (the
layer-output bar), far above fp16 output rounding (~3e-4) and far below any
indexing or operand mistake; and element by element, one fp16 ulp plus
10 x 2e-3 of the reference's rms (gpu_helpers.assert_close), which a single
wrong element fails."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import opt, q64  # noqa: E402
from gpu_helpers import assert_close, fq, rel_fro, to_dev, to_host  # noqa: E402

TOL = 2e-3
EPI = fq


@pytest.mark.parametrize("rows,h", [(1, 256), (5, 256), (300, 7168), (3, 12288), (64, 2048)])
def test_layernorm(rows, h):
    rng = np.random.default_rng(rows * h)
    x = (rng.standard_normal((rows, h)) * 2 + 0.5).astype(np.float16)
    g = (1 + 0.1 * rng.standard_normal(h)).astype(np.float16)
    b = (0.1 * rng.standard_normal(h)).astype(np.float16)
    y = torch.empty(rows, h, dtype=torch.float16, device="cuda")
    fq.flexq_layernorm(to_dev(x), h, to_dev(g), to_dev(b), y, h, rows, h, 1e-5)
    ref = opt.layernorm(x.astype(np.float64), g.astype(np.float64), b.astype(np.float64), 1e-5)
    assert_close(to_host(y), ref, TOL, what=f"layernorm {rows}x{h}")


def _linear_case(m, n, k, w_bits, epi, splits, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k)).astype(np.float16)
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float16)
    bias = (rng.standard_normal(n) * 0.1).astype(np.float16)
    res = rng.standard_normal((m, n)).astype(np.float16)
    if w_bits == 4:
        wd = torch.empty(fq.flexq_packed_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
        fq.flexq_quantize_weight_q4(to_dev(w), n, k, wd)
        w_eff = q64.roundtrip(w).astype(np.float64)
    else:
        wd = to_dev(w)
        w_eff = w.astype(np.float64)
    f32 = epi == fq.EPI_F32_OUT
    y = torch.empty(m, n, dtype=torch.float32 if f32 else torch.float16, device="cuda")
    ws_bytes = max(fq.flexq_linear_workspace(m, n, k, w_bits, splits), 1)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    fq.flexq_linear(to_dev(x), k, wd, w_bits, m, n, k, to_dev(bias), to_dev(res), n, epi, y, n,
                    ws, ws_bytes, splits)
    ref = x.astype(np.float64) @ w_eff.T
    if epi & fq.EPI_BIAS:
        ref = ref + bias.astype(np.float64)
    if epi & fq.EPI_GELU:
        ref = opt.gelu(ref)
    if epi & fq.EPI_RESIDUAL:
        ref = ref + res.astype(np.float64)
    return to_host(y), ref


LIN_CASES = [
    # m, n, k, epilogue, forced K splits
    (1, 128, 64, 1, 0),
    (4, 384, 256, 1, 0),
    (17, 256, 1024, 1 | 2, 0),
    (144, 512, 512, 1 | 4, 0),
    (144, 256, 2048, 1 | 4, 5),
    (32, 128, 4096, 1, 0),
    (256, 384, 384, 1 | 2, 0),
    (300, 384, 320, 1, 0),
    (600, 256, 128, 1 | 4, 0),
    (1000, 640, 512, 1 | 2, 3),
    (7, 200, 192, 8, 0),
    (3, 130, 64, 8, 0),
]


@pytest.mark.parametrize("m,n,k,epi,splits", LIN_CASES)
def test_linear_q4(m, n, k, epi, splits):
    got, ref = _linear_case(m, n, k, 4, epi, splits, m * 7 + n + k)
    assert_close(got, ref, TOL, what=f"linear q4 {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k,epi,splits", LIN_CASES + [(5, 1000, 256, 8, 0), (64, 50272 // 8, 256, 8, 0)])
def test_linear_f16(m, n, k, epi, splits):
    got, ref = _linear_case(m, n, k, 16, epi, splits, m * 11 + n + k)
    assert_close(got, ref, TOL, what=f"linear f16 {m}x{n}x{k}")


def test_linear_split_k_matches_unsplit():
    a, ref = _linear_case(144, 512, 2048, 4, 1, 1, 3)
    b, _ = _linear_case(144, 512, 2048, 4, 1, 8, 3)
    assert_close(a, ref, TOL, what="unsplit")
    assert_close(b, ref, TOL, what="split")
    assert rel_fro(a, b) < 1e-3


def _cfg(h, heads, kv_bits):
    return fq.flexq_config(h=h, heads=heads, ffn=4 * h, w_bits=4, kv_bits=kv_bits, ln_eps=1e-5)


def _dev_cache(cfg, b, max_len):
    from quantized_opt_decode_b200.device_model import KVCache
    return KVCache(cfg, b, max_len)


@pytest.mark.parametrize("h,heads,pos0,ntok", [(256, 4, 4, 5), (512, 4, 4, 5), (512, 4, 3, 21),
                                                (256, 4, 0, 16), (512, 4, 7, 1), (512, 4, 8, 1)])
def test_kv_append_bit_exact(h, heads, pos0, ntok):
    """Each (sequence, head, token) row quantized exactly as the oracle does;
    covers whole 8-token V blocks, ragged block edges and single tokens."""
    from gpu_helpers import v_words_to_canonical
    cfg = _cfg(h, heads, 4)
    b, L = 3, pos0 + ntok + 3
    rng = np.random.default_rng(h + pos0 * 7 + ntok)
    ld = 3 * h
    rows = rng.standard_normal((b * ntok, ld)).astype(np.float16)
    dev = _dev_cache(cfg, b, L)
    rd = to_dev(rows)
    fq.flexq_kv_append(cfg, dev.struct, rd[:, h:], rd[:, 2 * h:], ld, b, pos0, ntok)
    ocfg = opt.Config(layers=1, h=h, heads=heads, ffn=4 * h, vocab=8, w_bits=4, kv_bits=4)
    oc = opt.KVCache(ocfg, b, L, 4)
    oc.write("k", rows[:, h:2 * h].reshape(b, ntok, h), pos0)
    oc.write("v", rows[:, 2 * h:].reshape(b, ntok, h), pos0)
    d = h // heads
    sl = slice(pos0, pos0 + ntok)
    kc = to_host(dev.k).reshape(b, heads, L, d // 2)
    km = to_host(dev.k_meta).reshape(b, heads, L, d // 64, 2)
    vm = to_host(dev.v_meta).reshape(b, heads, L, d // 64, 2)
    vc = v_words_to_canonical(to_host(dev.v), b, heads, L, d)
    assert np.array_equal(kc[:, :, sl], oc.t["k_codes"][:, :, sl])
    assert np.array_equal(vc[:, :, sl], oc.t["v_codes"][:, :, sl])
    assert np.array_equal(km[:, :, sl, :, 0].view(np.uint16), oc.t["k_min"][:, :, sl].view(np.uint16))
    assert np.array_equal(km[:, :, sl, :, 1].view(np.uint16), oc.t["k_scale"][:, :, sl].view(np.uint16))
    assert np.array_equal(vm[:, :, sl, :, 0].view(np.uint16), oc.t["v_min"][:, :, sl].view(np.uint16))
    assert np.array_equal(vm[:, :, sl, :, 1].view(np.uint16), oc.t["v_scale"][:, :, sl].view(np.uint16))
    # slots outside the written range keep their (zero) codes
    assert not vc[:, :, :pos0].any() and not vc[:, :, pos0 + ntok:].any()


@pytest.mark.parametrize("h,heads,kv_bits,length", [(256, 4, 4, 1), (256, 4, 4, 37), (512, 4, 4, 545),
                                                    (256, 4, 16, 33), (512, 4, 16, 300),
                                                    (1024, 8, 4, 1030), (256, 2, 4, 12000)])
def test_attention_decode(h, heads, kv_bits, length):
    """Dense decode attention against the oracle; d = 64 and 128, ragged
    8-token blocks, and (12000 slots at d = 128) a cache too long for its V
    (min, scale) pairs to be gathered into shared memory."""
    cfg = _cfg(h, heads, kv_bits)
    b, L = 3, length + 3
    rng = np.random.default_rng(length + h)
    hist = rng.standard_normal((b * length, 3 * h)).astype(np.float16)
    dev = _dev_cache(cfg, b, L)
    hd = to_dev(hist)
    fq.flexq_kv_append(cfg, dev.struct, hd[:, h:], hd[:, 2 * h:], 3 * h, b, 0, length)
    q = rng.standard_normal((b, 3 * h)).astype(np.float16)
    out = torch.empty(b, h, dtype=torch.float16, device="cuda")
    fq.flexq_attention_decode(cfg, dev.struct, to_dev(q), 3 * h, b, length, out, h)
    ocfg = opt.Config(layers=1, h=h, heads=heads, ffn=4 * h, vocab=8, w_bits=4, kv_bits=kv_bits)
    oc = opt.KVCache(ocfg, b, L, kv_bits)
    oc.write("k", hist[:, h:2 * h].reshape(b, length, h), 0)
    oc.write("v", hist[:, 2 * h:].reshape(b, length, h), 0)
    qq = q[:, :h].astype(np.float64).reshape(b, heads, h // heads)
    ref = opt.attention_single(qq, oc.read("k", length), oc.read("v", length)).reshape(b, h)
    assert_close(to_host(out), ref, TOL, what=f"decode attention L={length}")


@pytest.mark.parametrize("h,heads,b,s", [(256, 4, 2, 1), (256, 4, 3, 37), (512, 4, 2, 64),
                                         (512, 4, 2, 130), (1024, 8, 1, 257)])
def test_attention_prefill(h, heads, b, s):
    cfg = _cfg(h, heads, 16)
    rng = np.random.default_rng(s + h)
    qkv = rng.standard_normal((b * s, 3 * h)).astype(np.float16)
    out = torch.empty(b * s, h, dtype=torch.float16, device="cuda")
    fq.flexq_attention_prefill(cfg, to_dev(qkv), 3 * h, b, s, out, h)
    x = qkv.astype(np.float64).reshape(b, s, 3 * h)
    Q, K, V = (opt.heads_split(x[..., i * h:(i + 1) * h], heads) for i in range(3))
    ref = opt.heads_merge(opt.attention_causal(Q, K, V)).reshape(b * s, h)
    assert_close(to_host(out), ref, TOL, what=f"prefill attention s={s}")


@pytest.mark.parametrize("h,heads,kv_bits,b,s,pos0", [(512, 4, 4, 2, 200, 0), (256, 4, 4, 3, 64, 0),
                                                      (512, 4, 4, 2, 73, 8), (1024, 8, 4, 1, 130, 0),
                                                      (512, 4, 16, 2, 130, 0), (256, 4, 16, 2, 37, 5)])
def test_attention_prefill_from_cache(h, heads, kv_bits, b, s, pos0):
    """Prefill attention reading K/V back from the cache: query t of the pass
    attends over slots pos0 .. pos0 + t as stored (the oracle's KVCache
    write/read, the decode steps' route), ragged last tiles included; slots
    before pos0 hold other rows and must be ignored."""
    cfg = _cfg(h, heads, kv_bits)
    L = pos0 + s + 3
    rng = np.random.default_rng(s + h + kv_bits + pos0)
    rows = rng.standard_normal((b * s, 3 * h)).astype(np.float16)
    early = rng.standard_normal((b * max(pos0, 1), 3 * h)).astype(np.float16) * 50
    dev = _dev_cache(cfg, b, L)
    rd = to_dev(rows)
    if pos0 > 0:
        ed = to_dev(early)
        fq.flexq_kv_append(cfg, dev.struct, ed[:, h:], ed[:, 2 * h:], 3 * h, b, 0, pos0)
    fq.flexq_kv_append(cfg, dev.struct, rd[:, h:], rd[:, 2 * h:], 3 * h, b, pos0, s)
    out = torch.empty(b * s, h, dtype=torch.float16, device="cuda")
    fq.flexq_attention_prefill_cache(cfg, dev.struct, rd, 3 * h, b, s, pos0, out, h)
    fq.flexq_device_status()
    ocfg = opt.Config(layers=1, h=h, heads=heads, ffn=4 * h, vocab=8, w_bits=4, kv_bits=kv_bits)
    oc = opt.KVCache(ocfg, b, s, kv_bits)
    r3 = rows.reshape(b, s, 3 * h)
    oc.write("k", r3[..., h:2 * h], 0)
    oc.write("v", r3[..., 2 * h:], 0)
    Q = opt.heads_split(r3[..., :h].astype(np.float64), heads)
    ref = opt.heads_merge(opt.attention_causal(Q, oc.read("k", s), oc.read("v", s))).reshape(b * s, h)
    assert_close(to_host(out), ref, TOL, what=f"prefill attention from the {kv_bits}-bit cache s={s}")


@pytest.mark.parametrize("h,heads,length,permille", [(512, 4, 545, 100), (256, 4, 37, 100), (1024, 8, 1030, 100),
                                                     (512, 4, 200, 1000), (256, 4, 64, 10), (512, 4, 1, 100)])
def test_attention_decode_topk(h, heads, length, permille):
    """Top-k sparse attention against the oracle on the same 4-bit cache.
    The kept set is decided from scores, so it is unique only where the k-th
    and (k+1)-th largest scores are apart by more than the scores' rounding:
    for those heads the kept slots must equal the oracle's exactly and the
    output must meet the parity bar; for a head with a near-tie at the
    threshold the kept set must still be a valid top-k (k slots, each scoring
    at least the oracle's k-th score minus the margin; the margin is ten times
    the kernel's score rounding, and most heads have a clear gap)."""
    cfg = _cfg(h, heads, 4)
    b, L = 3, length + 3
    d = h // heads
    rng = np.random.default_rng(length + h + permille)
    hist = rng.standard_normal((b * length, 3 * h)).astype(np.float16)
    dev = _dev_cache(cfg, b, L)
    hd = to_dev(hist)
    fq.flexq_kv_append(cfg, dev.struct, hd[:, h:], hd[:, 2 * h:], 3 * h, b, 0, length)
    q = rng.standard_normal((b, 3 * h)).astype(np.float16)
    kk = opt.topk_count(length, permille)
    out = torch.empty(b, h, dtype=torch.float16, device="cuda")
    idx = torch.full((b, heads, kk), -1, dtype=torch.int32, device="cuda")
    fq.flexq_attention_decode_topk(cfg, dev.struct, to_dev(q), 3 * h, b, length, kk, out, h, idx)
    fq.flexq_device_status()
    ocfg = opt.Config(layers=1, h=h, heads=heads, ffn=4 * h, vocab=8, w_bits=4, kv_bits=4)
    oc = opt.KVCache(ocfg, b, L, 4)
    oc.write("k", hist[:, h:2 * h].reshape(b, length, h), 0)
    oc.write("v", hist[:, 2 * h:].reshape(b, length, h), 0)
    qq = q[:, :h].astype(np.float64).reshape(b, heads, d)
    K, V = oc.read("k", length), oc.read("v", length)
    ref, sel = opt.attention_topk(qq, K, V, kk)
    sc = np.einsum("bad,bald->bal", qq, K) / math.sqrt(d)
    got_idx = to_host(idx)
    got = to_host(out).reshape(b, heads, d)
    clear_got, clear_ref, n_clear = [], [], 0
    for i in range(b):
        for j in range(heads):
            s = np.sort(sc[i, j])[::-1]
            # the kernel's scores differ from float64 by about 2e-5 * max|s|
            # (15-bit fixed-point q); 10x that decides a clear gap
            margin = 2e-4 * np.abs(s).max() + 1e-6
            gi = got_idx[i, j]
            assert np.all(np.diff(gi) > 0) and gi.min() >= 0 and gi.max() < length
            if kk == length or s[kk - 1] - s[kk] > margin:
                assert np.array_equal(gi, sel[i, j]), (i, j)
                clear_got.append(got[i, j])
                clear_ref.append(ref[i, j])
                n_clear += 1
            else:
                assert np.all(sc[i, j][gi] >= s[kk - 1] - margin), (i, j)
    assert n_clear >= 0.7 * b * heads
    assert_close(np.stack(clear_got), np.stack(clear_ref), TOL, what=f"top-k attention L={length}")
