"""Group-wise asymmetric 4-bit codec (oracle).

Source: "FlexGen研究学术报告" (fmread.com), section 三(C): weights and the KV
cache are compressed to 4 bits with fine-grained group-wise asymmetric
quantization, groups of 64 contiguous elements, no retraining or calibration;
tensors are dequantized to FP16 before compute.

The pages leave the arithmetic open; this module fixes the plainest reading:

1. per group g: mn = min(x), mx = max(x) over the fp16 values (exact), with
   -0 canonicalised to +0 (x + 0.0);
2. scale s16 = fp16_rn((mx - mn) / 15) with fp32 round-to-nearest subtraction
   and division (15 = 2^4 - 1 levels above the minimum); min m16 = fp16(mn),
   which is exact;
3. code q = 0 if s == 0 else clamp(rint_half_even((x - m) / s), 0, 15), all in
   fp32 with s = float(s16), m = float(m16);
4. pack: byte j = q[2j] | (q[2j+1] << 4) (low nibble holds the even element);
5. dequantize: x_hat = fp16_rn(fp32(q * s) + m), two separately rounded fp32
   operations (no fused multiply-add).

Inputs must be finite fp16 with |x| <= 2^15 (a group reaching the fp16
maximum can round its scale up so that 15*scale + min overflows) and a length
that is a multiple of 64.
"""
from __future__ import annotations

import numpy as np

GROUP = 64
LEVELS = 15


def quantize(x16: np.ndarray):
    """fp16 array (any shape, size % 64 == 0, groups along the flattened
    memory order) -> (codes uint8 [n/2], min fp16 [n/64], scale fp16 [n/64])."""
    x16 = np.ascontiguousarray(x16, dtype=np.float16).reshape(-1)
    if x16.size % GROUP:
        raise ValueError("length must be a multiple of 64")
    g = x16.reshape(-1, GROUP).astype(np.float32)
    mn = g.min(axis=1) + np.float32(0.0)
    mx = g.max(axis=1) + np.float32(0.0)
    s16 = ((mx - mn) / np.float32(LEVELS)).astype(np.float16)
    m16 = mn.astype(np.float16)
    s = s16.astype(np.float32)[:, None]
    m = m16.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint((g - m) / s)
    q = np.where(s == 0, np.float32(0), np.clip(r, 0, LEVELS)).astype(np.uint8)
    return pack(q.reshape(-1)), m16, s16


def pack(q: np.ndarray) -> np.ndarray:
    q = np.asarray(q, dtype=np.uint8).reshape(-1, 2)
    return (q[:, 0] | (q[:, 1] << 4)).astype(np.uint8)


def unpack(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    q = np.empty(c.size * 2, dtype=np.uint8)
    q[0::2] = c & 0x0F
    q[1::2] = c >> 4
    return q


def dequantize(codes: np.ndarray, mn: np.ndarray, sc: np.ndarray) -> np.ndarray:
    """-> fp16 array of length 2 * codes.size."""
    q = unpack(codes).reshape(-1, GROUP).astype(np.float32)
    s = np.asarray(sc, dtype=np.float16).astype(np.float32).reshape(-1, 1)
    m = np.asarray(mn, dtype=np.float16).astype(np.float32).reshape(-1, 1)
    return ((q * s) + m).astype(np.float16).reshape(-1)


def roundtrip(x16: np.ndarray) -> np.ndarray:
    """fp16 tensor -> its dequantized fp16 values, same shape."""
    x16 = np.asarray(x16, dtype=np.float16)
    c, m, s = quantize(x16)
    return dequantize(c, m, s).reshape(x16.shape)


def quantize_rows(x16: np.ndarray):
    """Quantize each row of [..., d] (d % 64 == 0) independently; returns
    codes [..., d/2], min [..., d/64], scale [..., d/64]."""
    x16 = np.asarray(x16, dtype=np.float16)
    lead, d = x16.shape[:-1], x16.shape[-1]
    c, m, s = quantize(x16)
    return c.reshape(*lead, d // 2), m.reshape(*lead, d // GROUP), s.reshape(*lead, d // GROUP)


def dequantize_rows(codes, mn, sc) -> np.ndarray:
    lead, half = codes.shape[:-1], codes.shape[-1]
    return dequantize(codes, mn, sc).reshape(*lead, half * 2)
