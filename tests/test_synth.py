"""The seeded generator: the splitmix64 output function reproduces the
published sequence for state 0 (Steele, Lea and Flood 2014; the reference
C implementation's first three outputs), and the derived draws have the
stated ranges and moments."""
import numpy as np

import synth


def test_splitmix64_published_vectors():
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [synth.hash64_scalar(0, i) for i in range(3)] == want
    assert [int(v) for v in synth.hash64(0, 0, 3)] == want


def test_vectorised_matches_scalar():
    key = synth.stream_key(1003, 77)
    v = synth.hash64(key, 1000, 50)
    assert [int(x) for x in v] == [synth.hash64_scalar(key, 1000 + i) for i in range(50)]


def test_normal_draw_moments_and_bound():
    x = synth.normal_f16(1000, 9, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 1e-4 and abs(x.std() - 0.02) < 2e-4
    assert np.abs(x).max() <= 0.02 * 3.4642
    g = synth.normal_f16(1000, 10, 1 << 16, 0.02, 1.0).astype(np.float64)
    assert abs(g.mean() - 1.0) < 1e-3


def test_chunked_threads_match_single_pass():
    a = synth.normal_f16(1001, 11, (1 << 22) + 12345, threads=4)
    b = synth.normal_f16(1001, 11, (1 << 22) + 12345, threads=1)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    c = synth.normal_f16(1001, 11, 100, start=(1 << 22))
    assert np.array_equal(a[1 << 22:(1 << 22) + 100].view(np.uint16), c.view(np.uint16))


def test_tokens_range():
    t = synth.tokens(1000, synth.TID_PROMPT, 200000, 50272)
    assert t.min() >= 0 and t.max() < 50272
    assert abs(t.mean() - 50271 / 2) < 300
