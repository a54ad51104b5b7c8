"""GPU parity of the generator and the 4-bit codec: bit-exact against the
oracle (codes, fp16 min/scale, dequantized fp16)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import synth  # noqa: E402
from oracle import q64  # noqa: E402
from gpu_helpers import f16_groups, fq, tiled_to_canonical, to_dev, to_host  # noqa: E402


@pytest.mark.parametrize("n,start,sigma,mean", [(1000003, 0, 0.02, 0.0), (4097, 123456, 1.0, 1.0),
                                                (64, 5, 0.02, 1.0)])
def test_synth_normal_matches_host(n, start, sigma, mean):
    t = torch.empty(n, dtype=torch.float16, device="cuda")
    fq.flexq_synth_normal_f16(t, n, 1003, 77, start, sigma, mean)
    host = synth.normal_f16(1003, 77, n, sigma, mean, start=start)
    assert np.array_equal(to_host(t).view(np.uint16), host.view(np.uint16))


def test_synth_tokens_match_host():
    n = 100001
    t = torch.empty(n, dtype=torch.int32, device="cuda")
    fq.flexq_synth_tokens(t, n, 1003, 5, 50272, start=7)
    assert np.array_equal(to_host(t), synth.tokens(1003, 5, n, 50272, start=7))


@pytest.mark.parametrize("n_groups", [1, 3, 8, 1037, (1 << 16) + 5])
def test_quantize_bit_exact(n_groups):
    rng = np.random.default_rng(n_groups)
    x = f16_groups(rng, n_groups)
    n = x.size
    xd = to_dev(x)
    codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    mn = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    sc = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    fq.flexq_quantize(xd, n, codes, mn, sc)
    c_ref, m_ref, s_ref = q64.quantize(x)
    assert np.array_equal(to_host(codes), c_ref)
    assert np.array_equal(to_host(mn).view(np.uint16), m_ref.view(np.uint16))
    assert np.array_equal(to_host(sc).view(np.uint16), s_ref.view(np.uint16))
    out = torch.empty(n, dtype=torch.float16, device="cuda")
    fq.flexq_dequantize(codes, mn, sc, n, out)
    assert np.array_equal(to_host(out).view(np.uint16), q64.dequantize(c_ref, m_ref, s_ref).view(np.uint16))


def _boundary_groups(rng, n_groups):
    """Groups whose quotients (x - min) / scale sit on or one fp16 step beside
    the half-integers where rint changes its result: exact ties (half to even)
    and values a reciprocal multiply alone would round the other way."""
    x = np.empty((n_groups, 64), dtype=np.float16)
    for g in range(n_groups):
        s = np.float16(rng.choice([3, 5, 7, 11, 13, 0.75, 1 / 3, 0.1, 0.7]) if g % 2 == 0
                       else np.exp(rng.uniform(-7, 2)))
        m = np.float16(rng.choice([0.0, -1.5, 2.25, -7.0]) if g % 3 else rng.standard_normal())
        vals = [m, np.float16(np.float32(m) + 15 * np.float32(s))]
        while len(vals) < 64:
            v = np.float16(np.float32(m) + (rng.integers(0, 15) + 0.5) * np.float32(s))
            vals += [v, np.nextafter(v, np.float16(np.inf)), np.nextafter(v, np.float16(-np.inf))]
        x[g] = np.array(vals[:64], dtype=np.float16)
    return x.reshape(-1)


@pytest.mark.parametrize("kind", ["boundaries", "subnormal"])
def test_quantize_rounding_boundaries_bit_exact(kind):
    """Codes at and next to the rounding boundaries of rint((x - min) / scale),
    where the quotient must be the correctly rounded fp32 one (in the boundary
    set, rounding a * (1/scale) instead changes about 0.5 % of the codes), and
    groups of fp16 subnormals (coarse grids, many exact ties)."""
    rng = np.random.default_rng(11 if kind == "boundaries" else 12)
    if kind == "boundaries":
        x = _boundary_groups(rng, 2048)
    else:
        x = (rng.standard_normal(64 * 4096) * 1e-6).astype(np.float16)
    n = x.size
    codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    mn = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    sc = torch.empty(n // 64, dtype=torch.float16, device="cuda")
    fq.flexq_quantize(to_dev(x), n, codes, mn, sc)
    c_ref, m_ref, s_ref = q64.quantize(x)
    assert np.array_equal(to_host(codes), c_ref)
    assert np.array_equal(to_host(mn).view(np.uint16), m_ref.view(np.uint16))
    assert np.array_equal(to_host(sc).view(np.uint16), s_ref.view(np.uint16))


def test_dequantize_every_code_and_byte():
    """All 256 byte values under random (min, scale) pairs."""
    rng = np.random.default_rng(9)
    groups = 512
    codes = np.tile(np.arange(256, dtype=np.uint8), groups * 32 // 256)
    mn = (rng.standard_normal(groups) * 3).astype(np.float16)
    sc = np.abs(rng.standard_normal(groups) * 0.1).astype(np.float16)
    out = torch.empty(groups * 64, dtype=torch.float16, device="cuda")
    fq.flexq_dequantize(to_dev(codes), to_dev(mn), to_dev(sc), groups * 64, out)
    assert np.array_equal(to_host(out).view(np.uint16), q64.dequantize(codes, mn, sc).view(np.uint16))


@pytest.mark.parametrize("n_out,k_in", [(128, 64), (200, 192), (384, 1024), (1000, 320)])
def test_weight_tiling_is_a_permutation_of_the_codec(n_out, k_in):
    rng = np.random.default_rng(n_out + k_in)
    w = (rng.standard_normal((n_out, k_in)) * 0.02).astype(np.float16)
    wd = to_dev(w)
    nbytes = fq.flexq_packed_weight_bytes(n_out, k_in)
    p1 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    p2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    fq.flexq_quantize_weight_q4(wd, n_out, k_in, p1)
    codes = torch.empty(w.size // 2, dtype=torch.uint8, device="cuda")
    mn = torch.empty(w.size // 64, dtype=torch.float16, device="cuda")
    sc = torch.empty(w.size // 64, dtype=torch.float16, device="cuda")
    fq.flexq_quantize(wd, w.size, codes, mn, sc)
    fq.flexq_pack_weight_q4(codes, mn, sc, n_out, k_in, p2)
    a, b = to_host(p1), to_host(p2)
    assert np.array_equal(a, b)
    can, m, s = tiled_to_canonical(a, n_out, k_in)
    c_ref, m_ref, s_ref = q64.quantize(w)
    assert np.array_equal(can.reshape(-1), c_ref)
    assert np.array_equal(m.reshape(-1).view(np.uint16), m_ref.view(np.uint16))
    assert np.array_equal(s.reshape(-1).view(np.uint16), s_ref.view(np.uint16))
