"""OPT-style decoder layer, KV cache and greedy generation (oracle, float64).

Sources (titles and sections of the FlexGen pages):

* "FlexGen: High-Throughput Generative Inference of Large Language Models
  with a Single GPU" walk-through (qingweiji.github.io), section "P/D阶段计算":
  prefill  x_K = x W_K, x_V = x W_V, x_Q = x W_Q,
           x_out = softmax(x_Q x_K^T / sqrt(.)) x_V W_O + x,
           x' = f_gelu(x_out W_1) W_2 + x_out;
  decode   x_K <- Concat(x_K, t W_K) (likewise V, along the sequence axis),
           t_out = softmax(t_Q x_K^T / sqrt(.)) x_V W_O + t,
           t' = f_gelu(t_out W_1) W_2 + t_out.
  Section "内存占用分析": Q, K, V, O and FC2 carry an [h] bias, FC1 an [ih] bias,
  each block has a LayerNorm (gamma, beta), the LM head is tied to the word
  embedding; the multi-head K is [b, s, a, h/a].
* Survey notes (gumorming.cn), eqs. (1)-(3): per-head Q_i, K_i, V_i,
  softmax(Q_i K_i^T / sqrt(d_k)) V_i, heads concatenated before W^O; word plus
  positional embedding before the first block; prefill emits the first output
  token and decoding emits one token per step.
* "FlexGen研究学术报告", section 三(C): weights and KV cache in the group-wise
  4-bit format, dequantized before compute.

Readings where the pages are silent or disagree (each is listed with its
reason in the design notes):
* the attention scale is 1/sqrt(d) with d = h / a (the single-head page's
  sqrt(h) is its a = 1 special case);
* pre-LN blocks: LN1 feeds Q/K/V, LN2 feeds FC1, residuals add the block
  input; LayerNorm uses the biased variance and eps = 1e-5; a final LayerNorm
  precedes the tied LM head;
* GELU is the exact erf form;
* prefill attends over the K/V of the pass before they are stored; decode
  first appends the new token's K/V (rounded to fp16, then quantized in 4-bit
  mode) and attends over the cached slots 0..pos read back (dequantized);
* greedy decoding takes the lowest index among equal maxima;
* ``Config.ln1_f16`` (off by default): the LN1 output is rounded to fp16
  before the Q/K/V projection.  The pages have the layer compute on FP16
  tensors ("FlexGen研究学术报告" section 三(C): dequantized to FP16 before
  compute), so the projection's input is an fp16 row there; with the option
  on, the K/V rows whose 4-bit codes the cache decides come from that same
  fp16 input.  Every other step stays float64.  A quantization decision is a
  step function of its input, so where a layer output hangs on those codes the
  oracle must take them from the input a fp16 layer sees; the GPU parity tests
  therefore turn the option on for every shape;
* ``Config.prefill_kv_cache`` (off by default): prefill attention reads the
  pass's K/V back from the cache as stored (4-bit: quantized and dequantized,
  fp16 mode: rounded to fp16) instead of using them as computed, i.e. it
  consumes the compressed cache like the decode steps do ("FlexGen研究学术报告"
  section 三(C): the KV cache is stored compressed and dequantized before
  compute).
Linear weights are stored [N_out][K_in], so a linear layer is y = x W^T + b.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
from scipy.special import erf

import synth
from . import q64


@dataclass
class Config:
    layers: int
    h: int
    heads: int
    ffn: int
    vocab: int
    w_bits: int = 4
    kv_bits: int = 4
    eps: float = 1e-5
    ln1_f16: bool = False
    topk_permille: int = 0  # decode attention keeps the top ceil(L * permille / 1000) keys (0: dense)
    embed_bits: int = 16    # 4: the tied embedding E is stored group-wise 4-bit (groups along h)
    prefill_kv_cache: bool = False  # prefill attention reads K/V back from the cache as stored

    @property
    def d(self) -> int:
        return self.h // self.heads

    @staticmethod
    def from_preset(p: dict, ln1_f16: bool = False) -> "Config":
        return Config(layers=p["layers"], h=p["h"], heads=p["heads"], ffn=p["ffn"],
                      vocab=p["vocab"], w_bits=p["w_bits"], kv_bits=p["kv_bits"],
                      ln1_f16=ln1_f16, topk_permille=p.get("topk_permille", 0),
                      embed_bits=p.get("embed_bits", 16),
                      prefill_kv_cache=bool(p.get("prefill_kv_cache", False)))


# ---------------------------------------------------------------------------
# Elementary operations (float64)
# ---------------------------------------------------------------------------
def layernorm(x, g, b, eps=1e-5):
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def gelu(z):
    return z * 0.5 * (1.0 + erf(z / math.sqrt(2.0)))


def linear(x, w, b):
    """y = x W^T + b with W stored [N_out][K_in]."""
    return x @ w.T + b


def softmax(s, axis=-1):
    m = s.max(axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=axis, keepdims=True)


def f16(x):
    """Round to fp16 (round to nearest even) and return float64 values."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# Weights
# ---------------------------------------------------------------------------
def raw_layer(cfg: Config, seed: int, layer: int) -> dict:
    """The fp16 tensors of one layer as drawn by the synthetic generator."""
    out = {}
    for name in synth.LAYER_TENSORS:
        shape, sigma, mean = synth.layer_tensor_spec(name, cfg.h, cfg.ffn)
        n = int(np.prod(shape))
        out[name] = synth.normal_f16(seed, synth.layer_tensor_id(layer, name), n,
                                     sigma, mean).reshape(shape)
    return out


LINEAR = ("w_qkv", "w_o", "w_fc1", "w_fc2")


def effective_layer(cfg: Config, raw: dict) -> dict:
    """float64 weights the layer computes with: the dequantized values of the
    stored 4-bit codes (groups of 64 along K_in) or the fp16 values."""
    eff = {}
    for k, v in raw.items():
        if k in LINEAR and cfg.w_bits == 4:
            eff[k] = q64.roundtrip(v).astype(np.float64)
        else:
            eff[k] = np.asarray(v, dtype=np.float16).astype(np.float64)
    return eff


def raw_globals(cfg: Config, seed: int, max_pos: int) -> dict:
    E = synth.normal_f16(seed, synth.TID_EMBED, cfg.vocab * cfg.h).reshape(cfg.vocab, cfg.h)
    P = synth.normal_f16(seed, synth.TID_POS, max_pos * cfg.h).reshape(max_pos, cfg.h)
    g = synth.normal_f16(seed, synth.TID_LNF_G, cfg.h, 0.02, 1.0)
    b = synth.normal_f16(seed, synth.TID_LNF_B, cfg.h)
    return {"E": E, "P": P, "lnf_g": g, "lnf_b": b}


def param_census(cfg: Config) -> dict:
    """Element counts of the tensors the model holds, by kind."""
    per_layer = 0
    for name in synth.LAYER_TENSORS:
        shape, _, _ = synth.layer_tensor_spec(name, cfg.h, cfg.ffn)
        per_layer += int(np.prod(shape))
    return {"layers": cfg.layers * per_layer, "embedding": cfg.vocab * cfg.h,
            "final_ln": 2 * cfg.h}


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------
@dataclass
class KVCache:
    """One layer's cache for b sequences and max_len slots, per head.
    4-bit: codes [b, a, L, d/2] u8 and min/scale [b, a, L, d/64] fp16 for each
    of K and V; 16-bit: values [b, a, L, d] fp16."""
    cfg: Config
    b: int
    max_len: int
    bits: int
    t: dict = field(default_factory=dict)

    def __post_init__(self):
        a, d, L, b = self.cfg.heads, self.cfg.d, self.max_len, self.b
        for kv in ("k", "v"):
            if self.bits == 4:
                self.t[kv + "_codes"] = np.zeros((b, a, L, d // 2), np.uint8)
                self.t[kv + "_min"] = np.zeros((b, a, L, d // 64), np.float16)
                self.t[kv + "_scale"] = np.zeros((b, a, L, d // 64), np.float16)
            else:
                self.t[kv] = np.zeros((b, a, L, d), np.float16)

    def nbytes(self) -> int:
        return sum(v.nbytes for v in self.t.values())

    def write(self, kv: str, rows16: np.ndarray, pos0: int):
        """rows16: fp16 [b, ntok, h] -> slots pos0 .. pos0+ntok-1 (concat along
        the sequence axis)."""
        b, ntok, _ = rows16.shape
        per_head = rows16.reshape(b, ntok, self.cfg.heads, self.cfg.d).transpose(0, 2, 1, 3)
        sl = slice(pos0, pos0 + ntok)
        if self.bits == 4:
            c, m, s = q64.quantize_rows(per_head)
            self.t[kv + "_codes"][:, :, sl] = c
            self.t[kv + "_min"][:, :, sl] = m
            self.t[kv + "_scale"][:, :, sl] = s
        else:
            self.t[kv][:, :, sl] = per_head

    def read(self, kv: str, length: int) -> np.ndarray:
        """float64 [b, a, length, d] of slots 0..length-1 as stored."""
        if self.bits == 4:
            c = self.t[kv + "_codes"][:, :, :length]
            m = self.t[kv + "_min"][:, :, :length]
            s = self.t[kv + "_scale"][:, :, :length]
            return q64.dequantize_rows(c, m, s).astype(np.float64)
        return self.t[kv][:, :, :length].astype(np.float64)


def kv_bytes_closed_form(b, layers, h, s, n, bits):
    """Peak KV size: 2 (K and V) * bytes/element * l * h * (s+n) * b; the
    fp16 case is the walk-through's 4blh(s+n).  In 4-bit form an element costs
    half a byte plus 4 bytes of min/scale per 64 elements."""
    per = 2.0 if bits == 16 else 0.5 + 4.0 / 64.0
    return int(round(2 * per * layers * h * (s + n) * b))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------
def heads_split(x, a):
    """[b, s, h] -> [b, a, s, d]."""
    b, s, h = x.shape
    return x.reshape(b, s, a, h // a).transpose(0, 2, 1, 3)


def heads_merge(x):
    """[b, a, s, d] -> [b, s, h] (Concat(Z_1..Z_a))."""
    b, a, s, d = x.shape
    return x.transpose(0, 2, 1, 3).reshape(b, s, a * d)


def attention_causal(q, k, v):
    """q, k, v: [b, a, s, d] -> [b, a, s, d]; key j is visible to query i
    when j <= i."""
    d = q.shape[-1]
    s = q.shape[2]
    sc = np.einsum("baid,bajd->baij", q, k) / math.sqrt(d)
    mask = np.triu(np.ones((s, s), dtype=bool), k=1)
    sc = np.where(mask, -np.inf, sc)
    return np.einsum("baij,bajd->baid", softmax(sc), v)


def attention_single(q, k, v):
    """q: [b, a, d]; k, v: [b, a, L, d] -> [b, a, d] (one query over all L keys)."""
    d = q.shape[-1]
    sc = np.einsum("bad,bald->bal", q, k) / math.sqrt(d)
    return np.einsum("bal,bald->bad", softmax(sc), v)


def topk_count(L: int, permille: int) -> int:
    """Keys kept by the top-k sparse attention: ceil(L * permille / 1000),
    at least 1 and at most L ("FlexGen研究学术报告" section 三(C): only the
    top 10 % of the cache by attention value is loaded; 10 % = 100 per mille)."""
    return max(1, min(L, -(-L * permille // 1000)))


def topk_select(scores, k):
    """Indices of the k largest scores in ascending index order; among equal
    scores the lower index is kept."""
    order = sorted(range(len(scores)), key=lambda t: (-scores[t], t))
    return sorted(order[:k])


def attention_topk(q, k, v, kk):
    """Top-k sparse decode attention.  q: [b, a, d]; k, v: [b, a, L, d];
    kk keys kept per (sequence, head).  Scores and their softmax p are formed
    over all L keys, exactly as dense attention; only the kk keys with the
    largest scores contribute their values, with their softmax weights as
    they are (no renormalisation over the kept keys): o = sum_{t in top-k}
    p_t v_t.  With kk = L this is attention_single.  Returns (o [b, a, d],
    selected indices [b, a, kk])."""
    d = q.shape[-1]
    sc = np.einsum("bad,bald->bal", q, k) / math.sqrt(d)
    p = softmax(sc)
    b, a, L = sc.shape
    out = np.zeros((b, a, d))
    sel = np.zeros((b, a, kk), dtype=np.int64)
    for i in range(b):
        for j in range(a):
            idx = topk_select(sc[i, j].tolist(), kk)
            sel[i, j] = idx
            out[i, j] = p[i, j, idx] @ v[i, j, idx]
    return out, sel


# ---------------------------------------------------------------------------
# Layer
# ---------------------------------------------------------------------------
def projection_input(cfg, W, x):
    """u = LN1(x), rounded to fp16 when cfg.ln1_f16 (the projection input of
    a layer that computes in fp16)."""
    u = layernorm(x, W["ln1_g"], W["ln1_b"], cfg.eps)
    return f16(u) if cfg.ln1_f16 else u


def _mlp(cfg, W, x_out):
    v = layernorm(x_out, W["ln2_g"], W["ln2_b"], cfg.eps)
    g = gelu(linear(v, W["w_fc1"], W["b_fc1"]))
    return linear(g, W["w_fc2"], W["b_fc2"]) + x_out


def cached_rows(cfg: Config, x: np.ndarray) -> np.ndarray:
    """The values the cache returns for rows x [..., h] once stored: fp16
    rounding, then (4-bit mode) the codec's round trip on 64-element groups
    along h, which are the per-head groups of the cache since d % 64 == 0."""
    x16 = np.asarray(x, dtype=np.float64).astype(np.float16)
    if cfg.kv_bits == 4:
        return q64.roundtrip(x16).astype(np.float64)
    return x16.astype(np.float64)


def layer_prefill(cfg: Config, W: dict, x: np.ndarray):
    """x: [b, s, h] -> (y [b, s, h], K16 [b, s, h], V16 [b, s, h]).  K16/V16
    are the fp16-rounded keys/values the cache stores for slots 0..s-1."""
    h = cfg.h
    u = projection_input(cfg, W, x)
    qkv = linear(u, W["w_qkv"], W["b_qkv"])
    Q, K, V = qkv[..., :h], qkv[..., h:2 * h], qkv[..., 2 * h:]
    a = cfg.heads
    Ka, Va = (cached_rows(cfg, K), cached_rows(cfg, V)) if cfg.prefill_kv_cache else (K, V)
    o = heads_merge(attention_causal(heads_split(Q, a), heads_split(Ka, a), heads_split(Va, a)))
    x_out = linear(o, W["w_o"], W["b_o"]) + x
    y = _mlp(cfg, W, x_out)
    return y, K.astype(np.float16), V.astype(np.float16)


def layer_decode(cfg: Config, W: dict, t: np.ndarray, cache: KVCache, pos: int):
    """t: [b, h] (the token at position pos) -> t' [b, h].  Appends this
    token's K/V to slot pos of the cache, then attends over slots 0..pos."""
    h, a = cfg.h, cfg.heads
    u = projection_input(cfg, W, t)
    qkv = linear(u, W["w_qkv"], W["b_qkv"])
    Q, K, V = qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:]
    cache.write("k", K.astype(np.float16)[:, None, :], pos)
    cache.write("v", V.astype(np.float16)[:, None, :], pos)
    b = t.shape[0]
    q = Q.reshape(b, a, cfg.d)
    if cfg.topk_permille > 0:
        kk = topk_count(pos + 1, cfg.topk_permille)
        o = attention_topk(q, cache.read("k", pos + 1), cache.read("v", pos + 1), kk)[0].reshape(b, h)
    else:
        o = attention_single(q, cache.read("k", pos + 1), cache.read("v", pos + 1)).reshape(b, h)
    t_out = linear(o, W["w_o"], W["b_o"]) + t
    return _mlp(cfg, W, t_out)


# ---------------------------------------------------------------------------
# Model and generation
# ---------------------------------------------------------------------------
@dataclass
class Model:
    cfg: Config
    layers: list          # effective (float64) layer weights
    E: np.ndarray         # fp16 [V, h]
    P: np.ndarray         # fp16 [max_pos, h]
    lnf_g: np.ndarray
    lnf_b: np.ndarray


def build_model(cfg: Config, seed: int, max_pos: int) -> Model:
    """The model as it computes: effective layer weights, and the tied
    embedding E as stored (its dequantized values when cfg.embed_bits == 4,
    groups of 64 along h; the lookups and the LM head then both use them)."""
    layers = [effective_layer(cfg, raw_layer(cfg, seed, i)) for i in range(cfg.layers)]
    g = raw_globals(cfg, seed, max_pos)
    E = q64.roundtrip(g["E"]) if cfg.embed_bits == 4 else g["E"]
    return Model(cfg, layers, E, g["P"], g["lnf_g"].astype(np.float64),
                 g["lnf_b"].astype(np.float64))


def embed(m: Model, tok: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """x0 = E[tok] + P[pos] (word plus positional embedding)."""
    return m.E[tok].astype(np.float64) + m.P[pos].astype(np.float64)


def lm_logits(m: Model, x_last: np.ndarray) -> np.ndarray:
    """logits = LN_f(x) E^T (LM head tied to the word embedding)."""
    return layernorm(x_last, m.lnf_g, m.lnf_b, m.cfg.eps) @ m.E.astype(np.float64).T


def greedy(logits: np.ndarray) -> np.ndarray:
    """argmax over the vocabulary; np.argmax returns the first (lowest) index
    among equal maxima."""
    return np.argmax(logits, axis=-1).astype(np.int32)


def generate(m: Model, prompts: np.ndarray, n: int, forced: np.ndarray | None = None):
    """prompts: int [b, s] -> (tokens int32 [b, n], logits float64 [n, b, V]).

    Prefill over the prompt yields token 1; each of the n-1 decode steps feeds
    the previous token at position s + j - 1 and yields the next one.  With
    ``forced`` [b, n] the next input is forced[:, j-1] instead of the oracle's
    own choice (teacher forcing, used to check another generator's choices)."""
    cfg = m.cfg
    b, s = prompts.shape
    caches = [KVCache(cfg, b, s + n, cfg.kv_bits) for _ in range(cfg.layers)]
    x = embed(m, prompts, np.arange(s)[None, :])
    for i, W in enumerate(m.layers):
        x, K16, V16 = layer_prefill(cfg, W, x)
        caches[i].write("k", K16, 0)
        caches[i].write("v", V16, 0)
    lg = lm_logits(m, x[:, -1])
    toks, all_logits = [greedy(lg)], [lg]
    for j in range(1, n):
        prev = toks[-1] if forced is None else forced[:, j - 1]
        pos = s + j - 1
        t = embed(m, prev, np.full(b, pos))
        for i, W in enumerate(m.layers):
            t = layer_decode(cfg, W, t, caches[i], pos)
        lg = lm_logits(m, t)
        toks.append(greedy(lg))
        all_logits.append(lg)
    return np.stack(toks, axis=1), np.stack(all_logits, axis=0)
