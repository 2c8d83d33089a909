"""The tensor-core epilogue rounds Q8_1(h) with a shortcut: q = round-half-away(v * RN(1/d)),
falling back to the IEEE quotient RN(v / d) when the product is within 2^-15 of a half-integer
or d is subnormal.  These CPU checks restate that rule in numpy float32 (IEEE binary32 with
round-to-nearest, as on the GPU) and confirm it picks the same integer as the plain
definition, round-half-away(RN(v / d)), on random blocks and on inputs built to sit on or next
to rounding ties."""
import numpy as np

F32 = np.float32


def _round_half_away(x):
    x = x.astype(np.float64)
    return np.where(x >= 0, np.floor(x + 0.5), np.ceil(x - 0.5))


def _shortcut(v, d):
    fast = d >= F32(2.0 ** -125)
    inv = F32(1.0) / d                          # RN(1/d)
    r = (v * inv).astype(F32)                   # RN(v * inv)
    a = np.abs(r)
    near = (~fast) | (np.abs(a - np.floor(a) - F32(0.5)) < F32(2.0 ** -15))
    rq = np.where(near, (v / d).astype(F32), r)
    return np.clip(_round_half_away(rq), -127, 127).astype(np.int32)


def _exact(v, d):
    return np.clip(_round_half_away((v / d).astype(F32)), -127, 127).astype(np.int32)


def _check(v):
    v = v.astype(F32)
    am = np.abs(v).max()
    d = (am / F32(127.0)).astype(F32)
    if d == 0:
        return 0
    ex = _exact(v, d)
    sc = _shortcut(v, d)
    assert np.array_equal(ex, sc), (v[ex != sc], d)
    return int(np.count_nonzero(np.abs((v * (F32(1) / d)).astype(F32)) % 1 == 0.5))


@np.errstate(over="ignore", invalid="ignore", under="ignore")
def test_random_blocks_agree():
    rng = np.random.default_rng(3)
    for _ in range(3000):
        scale = F32(10.0) ** F32(rng.uniform(-30, 30))
        _check((rng.standard_normal(32) * scale).astype(F32))


@np.errstate(over="ignore", invalid="ignore", under="ignore")
def test_ties_and_neighbours_agree():
    rng = np.random.default_rng(4)
    for _ in range(2000):
        d = F32(rng.uniform(0.5, 2.0)) * F32(2.0) ** F32(rng.integers(-60, 60))
        k = rng.integers(-127, 127, size=31).astype(F32)
        # values at k + 1/2 quanta and one or two ulp either side
        v = ((k + F32(0.5)) * d).astype(F32)
        v = np.nextafter(v, v + rng.choice([-1, 0, 1], size=31) * np.abs(v) * 2 + 1).astype(F32)
        v = np.concatenate([v, [F32(127.0) * d]]).astype(F32)   # fixes amax / 127 = d
        _check(v)


@np.errstate(over="ignore", invalid="ignore", under="ignore")
def test_subnormal_scales_take_the_division():
    rng = np.random.default_rng(5)
    for _ in range(500):
        v = (rng.standard_normal(32) * F32(2.0 ** -130)).astype(F32)
        _check(v)
