"""Pins of the oracle's layer math against facts that do not come from it:
pure-Python brute force on tiny inputs (math.exp / math.erf loops), closed
forms and invariants the equations imply (causality, sequence independence,
prefill/decode agreement, softmax special cases), and the sizes the pages
print (parameter count, per-layer bytes, peak KV bytes).

Equations: "FlexGen: High-Throughput Generative Inference ..." walk-through,
section "P/D阶段计算"; multi-head form: survey notes eqs. (1)-(3); sizes:
section "内存占用分析" (parameter count l(12h^2+13h)+Vh, per-layer fp16 bytes
8h1^2 + 4h1h2, peak KV 4blh(s+n)).
"""
import dataclasses
import math
import os

import numpy as np
import pytest

import synth
from oracle import opt, q64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_cfg(**kw):
    base = dict(layers=1, h=128, heads=2, ffn=512, vocab=96, w_bits=4, kv_bits=4)
    base.update(kw)
    return opt.Config(**base)


def rand_layer(cfg, seed=7, layer=0):
    return opt.effective_layer(cfg, opt.raw_layer(cfg, seed, layer))


# ---------------------------------------------------------------------------
# Brute force on tiny inputs
# ---------------------------------------------------------------------------
def bf_softmax(xs):
    m = max(xs)
    e = [math.exp(x - m) for x in xs]
    t = sum(e)
    return [v / t for v in e]


def bf_attention(q, k, v, causal):
    """q, k, v nested lists [s][d] for one head."""
    s, d = len(q), len(q[0])
    out = []
    for i in range(s):
        keys = range(i + 1) if causal else range(len(k))
        sc = [sum(q[i][e] * k[j][e] for e in range(d)) / math.sqrt(d) for j in keys]
        p = bf_softmax(sc)
        out.append([sum(p[jj] * v[j][e] for jj, j in enumerate(keys)) for e in range(d)])
    return out


def test_causal_attention_brute_force(rng):
    b, a, s, d = 2, 2, 6, 8
    q, k, v = (rng.standard_normal((b, a, s, d)) for _ in range(3))
    got = opt.attention_causal(q, k, v)
    for bi in range(b):
        for ai in range(a):
            ref = bf_attention(q[bi, ai].tolist(), k[bi, ai].tolist(), v[bi, ai].tolist(), True)
            assert np.allclose(got[bi, ai], ref, rtol=1e-12, atol=1e-12)


def test_single_query_attention_brute_force(rng):
    b, a, L, d = 2, 3, 9, 8
    q = rng.standard_normal((b, a, d))
    k, v = rng.standard_normal((b, a, L, d)), rng.standard_normal((b, a, L, d))
    got = opt.attention_single(q, k, v)
    for bi in range(b):
        for ai in range(a):
            ref = bf_attention([q[bi, ai].tolist()], k[bi, ai].tolist(), v[bi, ai].tolist(), False)
            assert np.allclose(got[bi, ai], ref[0], rtol=1e-12, atol=1e-12)


def test_attention_special_cases(rng):
    d = 16
    v = rng.standard_normal((1, 1, 1, d))
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, 1, d))
    assert np.allclose(opt.attention_single(q, k, v)[0, 0], v[0, 0, 0])  # one key -> v
    V = rng.standard_normal((1, 1, 7, d))
    K = rng.standard_normal((1, 1, 7, d))
    zero_q = np.zeros((1, 1, d))  # equal scores -> mean of V
    assert np.allclose(opt.attention_single(zero_q, K, V)[0, 0], V[0, 0].mean(axis=0))
    sc = rng.standard_normal((3, 11))
    assert np.allclose(opt.softmax(sc).sum(axis=-1), 1.0)


def test_linear_orientation_brute_force(rng):
    x = rng.standard_normal((3, 5))
    w = rng.standard_normal((4, 5))   # [N_out][K_in]
    b = rng.standard_normal(4)
    y = opt.linear(x, w, b)
    for i in range(3):
        for n in range(4):
            assert math.isclose(y[i, n], sum(x[i, k] * w[n, k] for k in range(5)) + b[n],
                                rel_tol=1e-12, abs_tol=1e-12)


def test_layernorm_brute_force_and_moments(rng):
    x = rng.standard_normal((4, 32)) * 3 + 1
    g, b = rng.standard_normal(32), rng.standard_normal(32)
    y = opt.layernorm(x, g, b, 1e-5)
    for r in range(4):
        row = x[r].tolist()
        mu = sum(row) / 32
        var = sum((t - mu) ** 2 for t in row) / 32
        ref = [(t - mu) / math.sqrt(var + 1e-5) * g[i] + b[i] for i, t in enumerate(row)]
        assert np.allclose(y[r], ref, rtol=1e-12, atol=1e-12)
    z = opt.layernorm(x, np.ones(32), np.zeros(32), 1e-5)
    assert np.allclose(z.mean(axis=-1), 0, atol=1e-12)
    assert np.allclose(z.var(axis=-1), 1, atol=1e-4)


def test_gelu_brute_force_and_limits():
    zs = np.linspace(-8, 8, 161)
    got = opt.gelu(zs)
    ref = [z * 0.5 * (1 + math.erf(z / math.sqrt(2))) for z in zs]
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-15)
    assert opt.gelu(np.array([0.0]))[0] == 0.0
    assert abs(opt.gelu(np.array([8.0]))[0] - 8.0) < 1e-12
    assert abs(opt.gelu(np.array([-8.0]))[0]) < 1e-12
    assert abs(opt.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-12  # Phi(1)


def test_layer_prefill_brute_force():
    """The whole pre-LN layer, written out as loops, on a 1-sequence, 3-token,
    h=64, 2-head, ffn=128 case."""
    rng = np.random.default_rng(3)
    h, a, ffn, s = 64, 2, 128, 3
    cfg = opt.Config(layers=1, h=h, heads=a, ffn=ffn, vocab=8, w_bits=16, kv_bits=16)
    W = {"w_qkv": rng.standard_normal((3 * h, h)) * 0.1, "b_qkv": rng.standard_normal(3 * h) * 0.1,
         "w_o": rng.standard_normal((h, h)) * 0.1, "b_o": rng.standard_normal(h) * 0.1,
         "w_fc1": rng.standard_normal((ffn, h)) * 0.1, "b_fc1": rng.standard_normal(ffn) * 0.1,
         "w_fc2": rng.standard_normal((h, ffn)) * 0.1, "b_fc2": rng.standard_normal(h) * 0.1,
         "ln1_g": 1 + rng.standard_normal(h) * 0.1, "ln1_b": rng.standard_normal(h) * 0.1,
         "ln2_g": 1 + rng.standard_normal(h) * 0.1, "ln2_b": rng.standard_normal(h) * 0.1}
    x = rng.standard_normal((1, s, h))
    y, _, _ = opt.layer_prefill(cfg, W, x)

    def ln(row, g, b):
        mu = sum(row) / len(row)
        var = sum((t - mu) ** 2 for t in row) / len(row)
        return [(t - mu) / math.sqrt(var + 1e-5) * g[i] + b[i] for i, t in enumerate(row)]

    def lin(row, w, b):
        return [sum(row[k] * w[n][k] for k in range(len(row))) + b[n] for n in range(len(w))]

    d = h // a
    X = x[0].tolist()
    U = [ln(r, W["ln1_g"], W["ln1_b"]) for r in X]
    QKV = [lin(u, W["w_qkv"].tolist(), W["b_qkv"]) for u in U]
    O = [[0.0] * h for _ in range(s)]
    for hd in range(a):
        q = [r[hd * d:(hd + 1) * d] for r in QKV]
        k = [r[h + hd * d:h + (hd + 1) * d] for r in QKV]
        v = [r[2 * h + hd * d:2 * h + (hd + 1) * d] for r in QKV]
        z = bf_attention(q, k, v, True)
        for i in range(s):
            O[i][hd * d:(hd + 1) * d] = z[i]
    XO = [[p + r for p, r in zip(lin(O[i], W["w_o"].tolist(), W["b_o"]), X[i])] for i in range(s)]
    for i in range(s):
        v2 = ln(XO[i], W["ln2_g"], W["ln2_b"])
        f1 = [t * 0.5 * (1 + math.erf(t / math.sqrt(2))) for t in lin(v2, W["w_fc1"].tolist(), W["b_fc1"])]
        ref = [p + r for p, r in zip(lin(f1, W["w_fc2"].tolist(), W["b_fc2"]), XO[i])]
        assert np.allclose(y[0, i], ref, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------------------
# Invariants of the layer equations
# ---------------------------------------------------------------------------
def test_prefill_is_causal():
    cfg = tiny_cfg()
    W = rand_layer(cfg)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 10, cfg.h))
    y1, _, _ = opt.layer_prefill(cfg, W, x)
    x2 = x.copy()
    x2[0, 7:] += 1.0
    y2, _, _ = opt.layer_prefill(cfg, W, x2)
    assert np.array_equal(y1[0, :7], y2[0, :7])
    assert not np.allclose(y1[0, 7:], y2[0, 7:])


def test_sequences_are_independent():
    cfg = tiny_cfg()
    W = rand_layer(cfg)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 5, cfg.h))
    y, k, v = opt.layer_prefill(cfg, W, x)
    y1, k1, v1 = opt.layer_prefill(cfg, W, x[1:2])
    assert np.allclose(y[1], y1[0], rtol=1e-13, atol=1e-13)
    assert np.array_equal(k[1], k1[0]) or np.abs(k[1].astype(float) - k1[0].astype(float)).max() <= 2e-3


@pytest.mark.parametrize("kv_bits", [16, 4])
def test_prefill_and_decode_agree(kv_bits):
    """Prefill on s+1 tokens and prefill on s tokens followed by one decode of
    token s give the same last row (the decode reads K/V back from the cache:
    fp16 in 16-bit mode, 4-bit codes otherwise, hence the tolerances)."""
    cfg = tiny_cfg(kv_bits=kv_bits)
    W = rand_layer(cfg)
    rng = np.random.default_rng(4)
    s = 9
    x = rng.standard_normal((2, s + 1, cfg.h))
    y_full, _, _ = opt.layer_prefill(cfg, W, x)
    cache = opt.KVCache(cfg, 2, s + 1, kv_bits)
    y_s, K, V = opt.layer_prefill(cfg, W, x[:, :s])
    cache.write("k", K, 0)
    cache.write("v", V, 0)
    t = opt.layer_decode(cfg, W, x[:, s], cache, s)
    # fp16 rounding of the cached K/V in 16-bit mode; in 4-bit mode each cached
    # element moves by up to scale/2 = range/30 of its group, a few percent.
    tol = 2e-3 if kv_bits == 16 else 6e-2
    dy = t - x[:, s]
    assert np.linalg.norm(dy - (y_full[:, s] - x[:, s])) <= tol * np.linalg.norm(dy)
    assert np.allclose(y_s, y_full[:, :s], rtol=1e-12, atol=1e-12)


def test_decode_reads_only_slots_up_to_pos():
    cfg = tiny_cfg(kv_bits=16)
    W = rand_layer(cfg)
    rng = np.random.default_rng(5)
    c1 = opt.KVCache(cfg, 2, 12, 16)
    c2 = opt.KVCache(cfg, 2, 12, 16)
    hist = rng.standard_normal((2, 6, cfg.h)).astype(np.float16)
    for c in (c1, c2):
        c.write("k", hist, 0)
        c.write("v", hist, 0)
    junk = rng.standard_normal((2, 5, cfg.h)).astype(np.float16) * 100
    c2.write("k", junk, 7)
    c2.write("v", junk, 7)
    t = rng.standard_normal((2, cfg.h))
    assert np.array_equal(opt.layer_decode(cfg, W, t, c1, 6), opt.layer_decode(cfg, W, t, c2, 6))


def test_decode_appends_quantized_row():
    cfg = tiny_cfg(kv_bits=4)
    W = rand_layer(cfg)
    rng = np.random.default_rng(6)
    cache = opt.KVCache(cfg, 1, 4, 4)
    t = rng.standard_normal((1, cfg.h))
    opt.layer_decode(cfg, W, t, cache, 2)
    u = opt.layernorm(t, W["ln1_g"], W["ln1_b"])
    K = opt.linear(u, W["w_qkv"], W["b_qkv"])[:, cfg.h:2 * cfg.h].astype(np.float16)
    c, m, s = q64.quantize(K.reshape(-1))
    d = cfg.d
    for j in range(cfg.heads):
        assert np.array_equal(cache.t["k_codes"][0, j, 2], c[j * d // 2:(j + 1) * d // 2])
        assert cache.t["k_min"][0, j, 2, 0] == m[j * d // 64]
    assert np.all(cache.t["k_codes"][0, :, 3] == 0)


# ---------------------------------------------------------------------------
# Sizes printed on the pages
# ---------------------------------------------------------------------------
def _golden_param_rows():
    rows = []
    with open(os.path.join(GOLDEN, "opt_param_counts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                name, billions = line.split()
                rows.append((name, float(billions)))
    return rows


@pytest.mark.parametrize("name,billions", _golden_param_rows())
def test_parameter_count(name, billions):
    p = synth.CONFIGS[name]
    cfg = opt.Config.from_preset(p)
    census = opt.param_census(cfg)
    l, h, V = cfg.layers, cfg.h, cfg.vocab
    assert census["layers"] + census["embedding"] == l * (12 * h * h + 13 * h) + V * h
    total = census["layers"] + census["embedding"]
    assert abs(total / 1e9 - billions) / billions < 0.02


def test_fp16_layer_weight_bytes():
    for name in ("opt-1.3b", "opt-6.7b", "opt-30b", "opt-175b"):
        cfg = opt.Config.from_preset(synth.CONFIGS[name])
        lin = 0
        for w in opt.LINEAR:
            shape, _, _ = synth.layer_tensor_spec(w, cfg.h, cfg.ffn)
            lin += shape[0] * shape[1]
        h1, h2 = cfg.h, cfg.ffn
        assert 2 * lin == 8 * h1 * h1 + 4 * h1 * h2


@pytest.mark.parametrize("bits", [16, 4])
def test_peak_kv_bytes(bits):
    b, l, h, s, n = 3, 2, 128, 20, 6
    cfg = opt.Config(layers=l, h=h, heads=2, ffn=4 * h, vocab=8, w_bits=bits, kv_bits=bits)
    caches = [opt.KVCache(cfg, b, s + n, bits) for _ in range(l)]
    total = sum(c.nbytes() for c in caches)
    if bits == 16:
        assert total == 4 * b * l * h * (s + n)
    else:
        assert total == b * l * h * (s + n) * 9 // 8
    assert total == opt.kv_bytes_closed_form(b, l, h, s, n, bits)


# ---------------------------------------------------------------------------
# Generation
# ---------------------------------------------------------------------------
def test_generate_prefill_token_and_teacher_forcing():
    p = dict(synth.CONFIGS["tiny"])
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=512, vocab=64, w_bits=4, kv_bits=4)
    m = opt.build_model(cfg, 1000, 16)
    prompts = synth.tokens(1000, synth.TID_PROMPT, 2 * 6, cfg.vocab).reshape(2, 6)
    toks, logits = opt.generate(m, prompts, 4)
    assert toks.shape == (2, 4) and logits.shape == (4, 2, cfg.vocab)
    # token 1 comes from the prefill's last row
    x = opt.embed(m, prompts, np.arange(6)[None, :])
    x, _, _ = opt.layer_prefill(cfg, m.layers[0], x)
    assert np.array_equal(toks[:, 0], opt.greedy(opt.lm_logits(m, x[:, -1])))
    # forcing the oracle's own tokens changes nothing; n=2 is a prefix of n=4
    t2, l2 = opt.generate(m, prompts, 4, forced=toks)
    assert np.array_equal(t2, toks) and np.allclose(l2, logits)
    t3, _ = opt.generate(m, prompts, 2)
    assert np.array_equal(t3, toks[:, :2])
    assert p["n"] == 8


def test_greedy_lowest_index_on_ties():
    lg = np.array([[1.0, 3.0, 3.0, 2.0], [5.0, 5.0, 5.0, 5.0]])
    assert opt.greedy(lg).tolist() == [1, 0]


# ---------------------------------------------------------------------------
# Embedding, tied LM head, group axis and the fp16-LN1 reading, by brute force
# ---------------------------------------------------------------------------
def _bf_ln(row, g, b, eps=1e-5):
    mu = sum(row) / len(row)
    var = sum((t - mu) ** 2 for t in row) / len(row)
    return [(t - mu) / math.sqrt(var + eps) * float(g[i]) + float(b[i]) for i, t in enumerate(row)]


def _bf_lin(row, w, b):
    return [sum(row[k] * float(w[n][k]) for k in range(len(row))) + float(b[n]) for n in range(len(w))]


def test_embed_brute_force():
    """x0[i][t] = E[tok[i][t]] + P[t] element by element from the fp16 tables
    (survey notes: word embedding plus positional embedding)."""
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=256, vocab=40, w_bits=4, kv_bits=4)
    m = opt.build_model(cfg, 77, 9)
    tok = np.array([[3, 0, 39, 3], [12, 12, 7, 38]])
    pos = np.arange(4)[None, :] + np.array([[0], [5]])
    got = opt.embed(m, tok, pos)
    for i in range(2):
        for t in range(4):
            for e in range(cfg.h):
                want = float(m.E[tok[i, t]][e]) + float(m.P[pos[i, t]][e])
                assert got[i, t, e] == want
    # the word and the position rows are distinct tables, not swapped
    assert not np.array_equal(opt.embed(m, tok[:, :1], pos[:, 1:2]), opt.embed(m, tok[:, 1:2], pos[:, :1]))


def test_lm_logits_brute_force():
    """logits[i][v] = sum_e LN_f(x_i)[e] * E[v][e]: final LayerNorm, then the
    word-embedding matrix as the LM head ("内存占用分析": tied embedding)."""
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=256, vocab=24, w_bits=4, kv_bits=4)
    m = opt.build_model(cfg, 78, 4)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, cfg.h)) * 2 + 0.3
    got = opt.lm_logits(m, x)
    for i in range(2):
        u = _bf_ln(x[i].tolist(), m.lnf_g, m.lnf_b)
        for v in range(cfg.vocab):
            want = sum(u[e] * float(m.E[v][e]) for e in range(cfg.h))
            assert math.isclose(got[i, v], want, rel_tol=1e-11, abs_tol=1e-11)


def test_effective_layer_groups_run_along_k_in():
    """A weight that is constant over every 64-wide span of K_in inside a row
    (and varies across rows) is reproduced exactly: each group is constant, so
    scale 0 and x_hat = min.  Groups taken along N_out (the transposed memory
    order) would mix 64 different rows and could not be exact."""
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=256, vocab=8, w_bits=4, kv_bits=4)
    rng = np.random.default_rng(9)
    raw = opt.raw_layer(cfg, 5, 0)
    for name in opt.LINEAR:
        n, k = raw[name].shape
        c = rng.standard_normal((n, k // 64)).astype(np.float16)
        raw[name] = np.repeat(c, 64, axis=1)
    eff = opt.effective_layer(cfg, raw)
    for name in opt.LINEAR:
        assert np.array_equal(eff[name], raw[name].astype(np.float64)), name
        assert not np.array_equal(q64.roundtrip(raw[name].T.copy()).T, raw[name])


def _bf_decode(cfg, W, t, keys, values, ln1_f16):
    """One decode step for one sequence written out as loops: keys/values are
    the cached rows [L][h] of slots 0..pos-1 (float values as read back); the
    new token's K/V (fp16-rounded) is appended last.  Returns (t', K_new)."""
    h, a, d = cfg.h, cfg.heads, cfg.d
    u = _bf_ln(t, W["ln1_g"], W["ln1_b"])
    if ln1_f16:
        u = [float(np.float16(v)) for v in u]
    qkv = _bf_lin(u, W["w_qkv"], W["b_qkv"])
    q = qkv[:h]
    k_new = [float(np.float16(v)) for v in qkv[h:2 * h]]
    v_new = [float(np.float16(v)) for v in qkv[2 * h:]]
    K, V = keys + [k_new], values + [v_new]
    o = [0.0] * h
    for j in range(a):
        sl = slice(j * d, (j + 1) * d)
        z = bf_attention([q[sl]], [r[sl] for r in K], [r[sl] for r in V], False)[0]
        o[j * d:(j + 1) * d] = z
    xo = [p + r for p, r in zip(_bf_lin(o, W["w_o"], W["b_o"]), t)]
    v2 = _bf_ln(xo, W["ln2_g"], W["ln2_b"])
    f1 = [z * 0.5 * (1 + math.erf(z / math.sqrt(2))) for z in _bf_lin(v2, W["w_fc1"], W["b_fc1"])]
    return [p + r for p, r in zip(_bf_lin(f1, W["w_fc2"], W["b_fc2"]), xo)], k_new


@pytest.mark.parametrize("ln1_f16", [False, True])
def test_decode_brute_force_fp16_kv(ln1_f16):
    """16-bit KV decode (append fp16(K), attend over slots 0..pos) against
    loops, with and without the fp16 rounding of the LN1 output; the two
    readings are different functions (the option is not a no-op)."""
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=128, vocab=8, w_bits=16, kv_bits=16, ln1_f16=ln1_f16)
    W = rand_layer(cfg, seed=11)
    rng = np.random.default_rng(12)
    pos = 3
    hist = rng.standard_normal((1, pos, cfg.h)).astype(np.float16)
    cache = opt.KVCache(cfg, 1, pos + 1, 16)
    cache.write("k", hist, 0)
    cache.write("v", hist * np.float16(0.5), 0)
    t = rng.standard_normal((1, cfg.h))
    got = opt.layer_decode(cfg, W, t, cache, pos)
    keys = hist[0].astype(np.float64).tolist()
    vals = (hist[0] * np.float16(0.5)).astype(np.float64).tolist()
    want, k_new = _bf_decode(cfg, W, t[0].tolist(), keys, vals, ln1_f16)
    assert np.allclose(got[0], want, rtol=1e-10, atol=1e-10)
    assert cache.t["k"][0, :, pos].reshape(-1).astype(np.float64).tolist() == k_new
    other = opt.Config(**{**cfg.__dict__, "ln1_f16": not ln1_f16})
    cache2 = opt.KVCache(other, 1, pos + 1, 16)
    cache2.write("k", hist, 0)
    cache2.write("v", hist * np.float16(0.5), 0)
    assert not np.array_equal(opt.layer_decode(other, W, t, cache2, pos), got)


def _bf_dequant_slot(cache, kv, i, pos):
    """Slot `pos` of sequence i read back from the 4-bit cache by loops over
    the nibbles: x_hat = fp16(fp32(code * scale) + min), low nibble = even
    element, one (min, scale) pair per 64 elements of a head row."""
    cfg = cache.cfg
    row = []
    for j in range(cfg.heads):
        codes = cache.t[kv + "_codes"][i, j, pos]
        for e in range(cfg.d):
            byte = int(codes[e // 2])
            q = byte & 15 if e % 2 == 0 else byte >> 4
            g = e // 64
            s = np.float32(cache.t[kv + "_scale"][i, j, pos, g])
            m = np.float32(cache.t[kv + "_min"][i, j, pos, g])
            row.append(float(np.float16(np.float32(np.float32(q) * s) + m)))
    return row


@pytest.mark.parametrize("ln1_f16", [False, True])
def test_decode_brute_force_4bit_kv(ln1_f16):
    """4-bit KV decode against loops that read every cached element back from
    its nibble and its group's (min, scale): pins the dequantizing read path
    and the attention over slots 0..pos (including the appended slot) to
    1e-10, far tighter than a prefill/decode comparison can."""
    cfg = opt.Config(layers=1, h=128, heads=2, ffn=128, vocab=8, w_bits=4, kv_bits=4, ln1_f16=ln1_f16)
    W = rand_layer(cfg, seed=13)
    rng = np.random.default_rng(14)
    pos = 4
    cache = opt.KVCache(cfg, 1, pos + 2, 4)
    cache.write("k", rng.standard_normal((1, pos, cfg.h)).astype(np.float16), 0)
    cache.write("v", rng.standard_normal((1, pos, cfg.h)).astype(np.float16), 0)
    t = rng.standard_normal((1, cfg.h))
    got = opt.layer_decode(cfg, W, t, cache, pos)
    keys = [_bf_dequant_slot(cache, "k", 0, p) for p in range(pos + 1)]
    vals = [_bf_dequant_slot(cache, "v", 0, p) for p in range(pos + 1)]
    # the brute force appends its own fp16 K/V row; swap in the cached slot
    # (its codes are pinned by test_decode_appends_quantized_row) so that the
    # loop attends over exactly what the cache holds
    h, a, d = cfg.h, cfg.heads, cfg.d
    u = _bf_ln(t[0].tolist(), W["ln1_g"], W["ln1_b"])
    if ln1_f16:
        u = [float(np.float16(v)) for v in u]
    qkv = _bf_lin(u, W["w_qkv"], W["b_qkv"])
    o = [0.0] * h
    for j in range(a):
        sl = slice(j * d, (j + 1) * d)
        o[sl] = bf_attention([qkv[:h][sl]], [r[sl] for r in keys], [r[sl] for r in vals], False)[0]
    xo = [p + r for p, r in zip(_bf_lin(o, W["w_o"], W["b_o"]), t[0].tolist())]
    v2 = _bf_ln(xo, W["ln2_g"], W["ln2_b"])
    f1 = [z * 0.5 * (1 + math.erf(z / math.sqrt(2))) for z in _bf_lin(v2, W["w_fc1"], W["b_fc1"])]
    want = [p + r for p, r in zip(_bf_lin(f1, W["w_fc2"], W["b_fc2"]), xo)]
    assert np.allclose(got[0], want, rtol=1e-10, atol=1e-10)
    # the appended K codes are Q64 of fp16(K) from this step's projection input
    c, m, s = q64.quantize(np.array(qkv[h:2 * h], np.float64).astype(np.float16))
    assert np.array_equal(cache.t["k_codes"][0, :, pos].reshape(-1), c)


def test_ln1_f16_prefill_rounds_projection_input():
    """With the option on, the prefill's K rows are those of the projection
    of fp16(LN1(x)); with it off, of LN1(x) itself."""
    rng = np.random.default_rng(15)
    for flag in (False, True):
        cfg = tiny_cfg(ln1_f16=flag)
        W = rand_layer(cfg, seed=16)
        x = rng.standard_normal((1, 3, cfg.h))
        _, K, _ = opt.layer_prefill(cfg, W, x)
        for r in range(3):
            u = _bf_ln(x[0, r].tolist(), W["ln1_g"], W["ln1_b"])
            if flag:
                u = [float(np.float16(v)) for v in u]
            k = _bf_lin(u, W["w_qkv"][cfg.h:2 * cfg.h], W["b_qkv"][cfg.h:2 * cfg.h])
            assert np.array_equal(K[0, r], np.array(k).astype(np.float16))


# ---------------------------------------------------------------------------
# Top-k sparse attention ("FlexGen研究学术报告" section 三(C))
# ---------------------------------------------------------------------------
def test_topk_count_is_ten_percent_rounded_up():
    assert opt.topk_count(528, 100) == 53 and opt.topk_count(10, 100) == 1
    assert opt.topk_count(1, 100) == 1 and opt.topk_count(7, 1000) == 7 and opt.topk_count(11, 100) == 2


def test_topk_selection_brute_force_and_ties():
    """The kept set is the k largest scores; at a tie the lower index wins:
    checked against a selection by repeated arg-max in pure Python."""
    rng = np.random.default_rng(21)
    for trial in range(50):
        L = int(rng.integers(1, 40))
        sc = rng.integers(-4, 5, size=L).astype(float).tolist()  # many ties
        k = int(rng.integers(1, L + 1))
        left = list(range(L))
        want = []
        for _ in range(k):
            best = left[0]
            for t in left:
                if sc[t] > sc[best]:
                    best = t  # strict: the first (lowest) index of a tie stays
            want.append(best)
            left.remove(best)
        assert opt.topk_select(sc, k) == sorted(want), (sc, k)
    assert opt.topk_select([1.0, 3.0, 3.0, 2.0, 3.0], 2) == [1, 2]


def test_topk_attention_brute_force_and_limits(rng):
    b, a, L, d = 2, 2, 23, 16
    q = rng.standard_normal((b, a, d))
    k = rng.standard_normal((b, a, L, d))
    v = rng.standard_normal((b, a, L, d))
    kk = opt.topk_count(L, 100)
    got, sel = opt.attention_topk(q, k, v, kk)
    for i in range(b):
        for j in range(a):
            sc = [sum(q[i, j, e] * k[i, j, t, e] for e in range(d)) / math.sqrt(d) for t in range(L)]
            m = max(sc)
            z = sum(math.exp(x - m) for x in sc)
            keep = sorted(range(L), key=lambda t: (-sc[t], t))[:kk]
            assert sorted(keep) == sel[i, j].tolist()
            ref = [sum(math.exp(sc[t] - m) / z * v[i, j, t, e] for t in keep) for e in range(d)]
            assert np.allclose(got[i, j], ref, rtol=1e-12, atol=1e-12)
    # k = L is dense attention; k = 1 keeps the arg-max key with its full-softmax weight
    dense, _ = opt.attention_topk(q, k, v, L)
    assert np.allclose(dense, opt.attention_single(q, k, v), rtol=1e-13, atol=1e-13)
    one, sel1 = opt.attention_topk(q, k, v, 1)
    sc = np.einsum("bad,bald->bal", q, k) / math.sqrt(d)
    p = opt.softmax(sc)
    top = sc.argmax(axis=-1)
    assert np.array_equal(sel1[..., 0], top)
    for i in range(b):
        for j in range(a):
            assert np.allclose(one[i, j], p[i, j, top[i, j]] * v[i, j, top[i, j]], rtol=1e-13)


@pytest.mark.parametrize("kv_bits", [4, 16])
def test_prefill_reading_the_cache_equals_decode_steps(kv_bits):
    """With prefill_kv_cache the prefill's row t equals a decode step of token
    t over a cache holding rows 0..t-1: the decode path appends the token's
    K/V and reads every slot back through KVCache (quantize_rows /
    dequantize_rows in 4-bit mode), a different route from the prefill's
    cached_rows round trip."""
    cfg = dataclasses.replace(tiny_cfg(kv_bits=kv_bits), prefill_kv_cache=True)
    W = rand_layer(cfg)
    rng = np.random.default_rng(11)
    s = 7
    x = rng.standard_normal((2, s, cfg.h))
    y, _, _ = opt.layer_prefill(cfg, W, x)
    cache = opt.KVCache(cfg, 2, s, kv_bits)
    for t in range(s):
        yt = opt.layer_decode(cfg, W, x[:, t], cache, t)
        assert np.allclose(yt, y[:, t], rtol=1e-9, atol=1e-9), t
    # and the option matters in 4-bit mode (the pass's own K/V differ from the cache's)
    y_plain, _, _ = opt.layer_prefill(dataclasses.replace(cfg, prefill_kv_cache=False), W, x)
    if kv_bits == 4:
        assert not np.allclose(y_plain, y, rtol=1e-6, atol=1e-6)
