"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds no arithmetic of the method (no quantizer, no layer math).
It only turns (seed, tensor id, element index) into numbers:

* ``hash64``: the splitmix64 output function (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014) applied to a
  counter, so that every element is an independent function of its index.
  The CUDA library carries its own implementation of the same published
  definition (``flexq_synth_*``); a GPU test checks the two bit for bit.
* ``normal_f16``: an Irwin-Hall sum of the four 16-bit fields of one hash,
  centred and scaled to standard deviation ``sigma`` with one fp32
  round-to-nearest multiply and one fp32 add, then rounded to fp16.  The draw is
  bounded at about 3.46 sigma and needs no transcendental function, so host
  and device agree exactly.
* ``tokens``: ids uniform over ``[0, vocab)`` from the top 32 bits.

The workloads follow the FlexGen pages' setting (OPT-style shapes, prompt
length 512, 32 generated tokens; random weights ~N(0, 0.02)).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
IH_CENTER = 131070  # 4 * (65535 / 2)


def _mix_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    """64-bit key of one tensor's stream: mix(seed * GOLDEN + tensor_id)."""
    return _mix_int((seed * GOLDEN + tensor_id) & MASK64)


def hash64_scalar(key: int, idx: int) -> int:
    """Element ``idx`` of a stream: mix(key + GOLDEN * (idx + 1))."""
    return _mix_int((key + GOLDEN * (idx + 1)) & MASK64)


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
    return z ^ (z >> np.uint64(31))


def hash64(key: int, start: int, count: int) -> np.ndarray:
    """uint64 hashes of elements ``start .. start+count-1`` of stream ``key``."""
    idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = idx * np.uint64(GOLDEN) + np.uint64(key)
        return _mix_np(z)


def normal_scale(sigma: float) -> np.float32:
    """The fp32 constant sqrt(3)/65536*sigma that both sides multiply by."""
    return np.float32(math.sqrt(3.0) / 65536.0 * sigma)


def _normal_chunk(key, start, count, c32, mean32):
    h = hash64(key, start, count)
    m = np.uint64(0xFFFF)
    s = (h & m) + ((h >> np.uint64(16)) & m) + ((h >> np.uint64(32)) & m) + (h >> np.uint64(48))
    z = (s.astype(np.int64) - IH_CENTER).astype(np.float32)
    z = z * c32
    z = z + mean32
    return z.astype(np.float16)


def normal_f16(seed: int, tensor_id: int, n: int, sigma: float = 0.02, mean: float = 0.0,
               start: int = 0, threads: int = 0) -> np.ndarray:
    """fp16 draws ~N(mean, sigma^2) for elements ``start .. start+n-1``."""
    key = stream_key(seed, tensor_id)
    c32 = normal_scale(sigma)
    mean32 = np.float32(mean)
    chunk = 1 << 22
    if n <= chunk or threads == 1:
        return _normal_chunk(key, start, n, c32, mean32)
    out = np.empty(n, dtype=np.float16)
    spans = [(o, min(chunk, n - o)) for o in range(0, n, chunk)]

    def work(span):
        o, c = span
        out[o:o + c] = _normal_chunk(key, start + o, c, c32, mean32)

    with ThreadPoolExecutor(max_workers=threads or None) as ex:
        list(ex.map(work, spans))
    return out


def tokens(seed: int, tensor_id: int, n: int, vocab: int, start: int = 0) -> np.ndarray:
    """int32 ids uniform over [0, vocab): ((hash >> 32) * vocab) >> 32."""
    h = hash64(stream_key(seed, tensor_id), start, n)
    with np.errstate(over="ignore"):
        t = ((h >> np.uint64(32)) * np.uint64(vocab)) >> np.uint64(32)
    return t.astype(np.int32)


# ---------------------------------------------------------------------------
# Tensor ids and the synthetic model/workload recipe.
# ---------------------------------------------------------------------------
LAYER_TENSORS = ("w_qkv", "b_qkv", "w_o", "b_o", "w_fc1", "b_fc1", "w_fc2", "b_fc2",
                 "ln1_g", "ln1_b", "ln2_g", "ln2_b")
TID_EMBED, TID_POS, TID_LNF_G, TID_LNF_B, TID_PROMPT = 1, 2, 3, 4, 5
TID_TEST_BASE = 1 << 20  # ids for ad-hoc test tensors


def layer_tensor_id(layer: int, name: str) -> int:
    return (layer + 1) * 64 + LAYER_TENSORS.index(name)


def layer_tensor_spec(name: str, h: int, ffn: int):
    """(shape, sigma, mean) of one layer tensor.  Linear weights are stored
    [N_out][K_in]; LayerNorm gains are 1 + N(0, 0.02) so that the affine path
    is exercised, everything else is N(0, 0.02)."""
    shapes = {
        "w_qkv": (3 * h, h), "b_qkv": (3 * h,), "w_o": (h, h), "b_o": (h,),
        "w_fc1": (ffn, h), "b_fc1": (ffn,), "w_fc2": (h, ffn), "b_fc2": (h,),
        "ln1_g": (h,), "ln1_b": (h,), "ln2_g": (h,), "ln2_b": (h,),
    }
    mean = 1.0 if name.endswith("_g") else 0.0
    return shapes[name], 0.02, mean


CONFIGS = {
    # name: (layers, h, heads, ffn, vocab, b, s, n, w_bits, kv_bits, gpu_batch)
    "tiny": dict(layers=2, h=256, heads=4, ffn=1024, vocab=512, b=4, s=32, n=8,
                 w_bits=4, kv_bits=4, gpu_batch=4, index=0),
    "tiny16": dict(layers=2, h=256, heads=4, ffn=1024, vocab=512, b=4, s=32, n=8,
                   w_bits=16, kv_bits=16, gpu_batch=4, index=0),
    "opt-1.3b": dict(layers=24, h=2048, heads=32, ffn=8192, vocab=50272, b=64, s=512, n=32,
                     w_bits=16, kv_bits=16, gpu_batch=64, index=1),
    "opt-6.7b": dict(layers=32, h=4096, heads=32, ffn=16384, vocab=50272, b=256, s=512, n=32,
                     w_bits=4, kv_bits=4, gpu_batch=32, index=2),
    "opt-30b": dict(layers=48, h=7168, heads=56, ffn=28672, vocab=50272, b=144, s=512, n=32,
                    w_bits=4, kv_bits=4, gpu_batch=144, index=3),
    "opt-30b-s1024": dict(layers=48, h=7168, heads=56, ffn=28672, vocab=50272, b=144, s=1024,
                          n=32, w_bits=4, kv_bits=4, gpu_batch=144, index=3),
    "opt-175b": dict(layers=96, h=12288, heads=96, ffn=49152, vocab=50272, b=32, s=512, n=32,
                     w_bits=4, kv_bits=4, gpu_batch=32, index=4),
}


def config_seed(cfg: dict) -> int:
    return 1000 + cfg["index"]
