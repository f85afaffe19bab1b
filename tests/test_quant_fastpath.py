"""The append kernel decides each code rne(x / s) (x / s the IEEE fp32 quotient) from
q = x * (1/s), both correctly rounded, and divides only where q lies within 2^-14 of a
half-integer.  This checks that argument in float32 numpy (IEEE division, reciprocal and
multiply, the same roundings the kernel's __fdiv_rn, __frcp_rn and __fmul_rn make) on
random tokens with the codec's scales and on elements placed at and next to ties."""
import numpy as np

F = np.float32


def codes_by_division(x, s, lo, hi):
    with np.errstate(all="ignore"):
        r = np.rint((x / s).astype(F))
    r = np.where(np.isnan(r), 0, np.clip(r, lo, hi))
    return np.where(s == 0, 0, r).astype(np.int64)


def codes_by_reciprocal(x, s, lo, hi):
    with np.errstate(all="ignore"):
        q = (x * (F(1) / s).astype(F)).astype(F)
        h = np.abs((q - np.floor(q)).astype(F) - F(0.5))
        near = ~(h > F(2.0 ** -14))
        q = np.where(near, (x / s).astype(F), q)
        r = np.rint(q)
    r = np.where(np.isnan(r), 0, np.clip(r, lo, hi))
    return np.where(s == 0, 0, r).astype(np.int64), near


def scales(x, group, div):
    a = np.abs(x.reshape(x.shape[0], -1, group)).max(-1, keepdims=True)
    with np.errstate(over="ignore"):
        return (a / F(div)).astype(F).astype(np.float16).astype(F)


def test_random_tokens_with_codec_scales():
    rng = np.random.default_rng(3)
    for trial in range(12):
        x = (rng.standard_normal((512, 256)) * 10.0 ** rng.uniform(-6, 4.8)).astype(F)
        x[rng.random(x.shape) < 0.01] *= F(30)
        for group, div, lo, hi in ((256, 127.0, -127, 127), (32, 7.0, -8, 7)):
            s = np.broadcast_to(scales(x, group, div), (512, 256 // group, group))
            xg = x.reshape(512, -1, group)
            got, _ = codes_by_reciprocal(xg, s, lo, hi)
            assert np.array_equal(got, codes_by_division(xg, s, lo, hi)), (trial, group)


def test_elements_at_and_next_to_ties():
    rng = np.random.default_rng(4)
    for trial in range(60):
        s = F(np.float16(10.0 ** rng.uniform(-7, 4.5)))
        n = rng.integers(-128, 128, 20000).astype(F)
        x = ((n + F(0.5)) * s).astype(F)
        k = rng.integers(-4, 5, x.size)
        for _ in range(4):
            x = np.where(k != 0, np.nextafter(x, np.where(k > 0, F(np.inf), F(-np.inf))), x).astype(F)
            k = k - np.sign(k)
        sb = np.full_like(x, s)
        for lo, hi in ((-127, 127), (-8, 7)):
            got, near = codes_by_reciprocal(x, sb, lo, hi)
            assert np.array_equal(got, codes_by_division(x, sb, lo, hi)), trial
            assert near.mean() > 0.5   # the ties themselves take the division


def test_special_scales_and_values():
    s = np.array([0.0, 2.0 ** -24, 2.0 ** -20, 1.0, 65504.0, np.inf], dtype=F)
    x = np.array([0.0, -0.0, 1.5, -2.5, 127.49, np.inf, -np.inf, np.nan, 3.0e38, 1e-40], dtype=F)
    X, S = np.meshgrid(x, s)
    for lo, hi in ((-127, 127), (-8, 7)):
        got, _ = codes_by_reciprocal(X, S, lo, hi)
        assert np.array_equal(got, codes_by_division(X, S, lo, hi))
