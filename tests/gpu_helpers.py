"""Helpers shared by the GPU tests: host<->device copies and seeded inputs.
(Test infrastructure; the oracle side never sees anything the GPU computed.)"""
import numpy as np
import torch

from quantized_opt_decode_b200 import build

build.build()

from quantized_opt_decode_b200 import flexq as fq  # noqa: E402

DEV = "cuda"


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def to_host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


def f16_groups(rng, n_groups, extra=True):
    """fp16 test data: groups of 64 at magnitudes from 1e-6 to 1e4, plus the
    codec's special cases (constant, +-0, subnormal ramp, two-valued, the
    input-range boundary)."""
    mags = 10.0 ** rng.uniform(-6, 4, size=(n_groups, 1))
    x = (rng.standard_normal((n_groups, 64)) * mags + rng.standard_normal((n_groups, 1)) * mags)
    x = x.astype(np.float16)
    if extra and n_groups >= 8:
        x[0] = np.float16(0.75)
        x[1] = np.array([-0.0, 0.0] * 32, np.float16)
        x[2] = (np.arange(64) * 2.0 ** -24).astype(np.float16)
        x[3] = np.array([0.3, -1.7] * 32, np.float16)
        x[4] = np.linspace(-32768, 32768, 64).astype(np.float16)
        x[5] = np.float16(-0.0)
        x[6, :] = np.float16(1.0)
        x[6, 17] = np.float16(1.0009765625)
    return x.reshape(-1)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (d if d > 0 else 1.0))


def tiled_to_canonical(packed: np.ndarray, n_out: int, k_in: int):
    """Reads the GEMM's tiled 4-bit layout (as include/flexq.h documents it)
    back into canonical codes [n_out][k_in/2] and min/scale [n_out][k_in/64]."""
    kb = k_in // 64
    nt = (n_out + 127) // 128
    tiles = packed.reshape(nt, kb, 4608)
    codes = np.ascontiguousarray(tiles[:, :, :4096]).view(np.uint32).reshape(nt, kb, 128, 8)
    meta = np.ascontiguousarray(tiles[:, :, 4096:]).view(np.float16).reshape(nt, kb, 128, 2)
    q = np.zeros((nt, kb, 128, 8, 8), np.uint8)
    for e in range(8):
        pos = (e >> 1) + 4 * (e & 1)
        q[..., e] = (codes >> np.uint32(4 * pos)) & np.uint32(0xF)
    # q[nt, kb, row, word, e] -> element (word*8+e) of group kb of row nt*128+row
    q = q.transpose(0, 2, 1, 3, 4).reshape(nt * 128, kb * 64)[:n_out]
    can = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    meta = meta.transpose(0, 2, 1, 3).reshape(nt * 128, kb, 2)[:n_out]
    return can, meta[..., 0].copy(), meta[..., 1].copy()


def v_words_to_canonical(words: np.ndarray, b: int, heads: int, max_len: int, d: int):
    """Reads the token-interleaved 4-bit V layout (include/flexq.h: nibble k of
    word (block, e) = token 8*block + k at dimension e) back into canonical
    per-token rows [b][heads][max_len][d/2] (low nibble = even element)."""
    l8 = (max_len + 7) // 8 * 8
    w = np.ascontiguousarray(words).view(np.uint32).reshape(b, heads, l8 // 8, d)
    codes = np.zeros((b, heads, l8 // 8, 8, d), np.uint8)
    for k in range(8):
        codes[:, :, :, k, :] = (w >> np.uint32(4 * k)) & np.uint32(0xF)
    codes = codes.reshape(b, heads, l8, d)[:, :, :max_len]
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def ulp16(x):
    """Spacing of fp16 numbers at |x| (the subnormal spacing below 2^-14)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def assert_close(got, ref, tol=2e-3, c=10.0, what=""):
    """The parity bar of the GPU tests: relative Frobenius error below `tol`,
    and every element within one fp16 ulp of its reference plus c * tol times
    the reference's rms.  The second bound catches a single wrong element
    (an indexing slip in one tile) that a norm over 10^6 elements would
    average away."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    r = rel_fro(got, ref)
    assert r < tol, f"{what}: relative Frobenius error {r:.3e} >= {tol:.1e}"
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    bound = ulp16(ref) + c * tol * rms
    err = np.abs(got - ref)
    excess = err - bound
    k = int(np.argmax(excess)) if excess.size else 0
    assert excess.size == 0 or excess.flat[k] <= 0, (
        f"{what}: element {np.unravel_index(k, ref.shape)} off by {err.flat[k]:.3e} "
        f"(ref {ref.flat[k]:.4e}, bound {bound.flat[k]:.3e}, rms {rms:.3e})")
    return r
