"""The GPU group quantizer avoids most divisions: it rounds r = a * fl(1/s)
and takes rint(fl(a / s)) only where r lies within |r| * 2^-20 (+ 2^-40) of a
rounding boundary.  These CPU tests restate that decision rule in fp32 numpy
and check that it reproduces rint of the correctly rounded quotient (the
oracle's codes) on random groups, on groups built around the boundaries, on
fp16 subnormals and on the extremes of the fp16 range; and that without the
fallback the boundary set does round differently (so the rule is doing work)."""
import numpy as np

from oracle import q64

F = np.float32


def _codes_rule(x, mn, sc, fallback=True):
    G = x.size // 64
    m = np.repeat(mn.astype(F), 64).reshape(G, 64)
    s = np.repeat(sc.astype(F), 64).reshape(G, 64)
    a = (x.reshape(G, 64).astype(F) - m).astype(F)
    safe = np.where(s != 0, s, F(1))
    inv = (F(1) / safe).astype(F)
    r = (a * inv).astype(F)
    k = np.rint(r).astype(F)
    if fallback:
        margin = (np.abs(r) * F(2.0 ** -20) + F(2.0 ** -40)).astype(F)
        near = np.abs((F(0.5) - np.abs((r - k).astype(F))).astype(F)) <= margin
        k = np.where(near, np.rint((a / safe).astype(F)), k)
    return np.where(s != 0, np.clip(k, 0, 15), 0).astype(np.uint8).reshape(-1)


def _oracle_codes(x):
    c, mn, sc = q64.quantize(x)
    q = np.empty(c.size * 2, dtype=np.uint8)
    q[0::2], q[1::2] = c & 15, c >> 4
    return q, mn, sc


def _boundary_groups(rng, n_groups):
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


def _check(x):
    want, mn, sc = _oracle_codes(x)
    got = _codes_rule(x, mn, sc)
    assert np.array_equal(got, want)


def test_rule_matches_division_on_random_groups():
    rng = np.random.default_rng(1)
    for sigma in (0.02, 1.0, 300.0, 1e-4):
        _check((rng.standard_normal(64 * 8000) * sigma).astype(np.float16))


def test_rule_matches_division_at_rounding_boundaries():
    x = _boundary_groups(np.random.default_rng(11), 2048)
    _check(x)
    want, mn, sc = _oracle_codes(x)
    assert not np.array_equal(_codes_rule(x, mn, sc, fallback=False), want)


def test_rule_matches_division_on_subnormals_and_extremes():
    rng = np.random.default_rng(3)
    _check((rng.standard_normal(64 * 4000) * 1e-6).astype(np.float16))
    big = rng.uniform(-1, 1, 64 * 2000) * 30000.0
    _check(big.astype(np.float16))
