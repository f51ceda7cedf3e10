"""The arithmetic the 8-bit int4 path relies on, checked in exact integer arithmetic (numpy int64 / float64).

For a scale group of 128 bf16 activations with largest magnitude M, the path takes the exponent c that puts
M * 2^c in [2^21, 2^22), holds X = rint(x * 2^c) as three signed 8-bit digits X = 65536 d2 + 256 d1 + d0, forms
per digit the s32 sums A_i = sum(u * d_i) with u = q + 8 the stored nibble, and recombines
65536 A2 + 256 A1 + A0 - 8 sum(X) = sum(q * X).  The claims pinned here:

- the digits exist and are in [-128, 127] for every |X| < 2^22;
- each A_i fits s32 for any 128 nibbles and digits;
- the recombination equals sum(q * X) exactly;
- X = x * 2^c exactly for every element with |x| >= M * 2^-13, and |X - x * 2^c| <= M * 2^-22 * 2^c otherwise.

(This is the exactness reading the 8-bit path is built on; the kernel itself is compared with the oracle by the
GPU parity tests.)
"""
import numpy as np

from weight_only_bit_route_b200 import synthetic as syn


def _bf16(a):
    return syn.to_bf16_bits(np.asarray(a, np.float32)).astype(np.uint32) << 16


def _groups(rng, n):
    """n groups of 128 bf16 values: N(0, 1) with a spread of magnitudes (down to 2^-30) and exact zeros."""
    x = rng.standard_normal((n, 128)) * np.exp2(rng.integers(-30, 8, size=(n, 128)) * (rng.random((n, 128)) < 0.3))
    x[rng.random((n, 128)) < 0.02] = 0.0
    return _bf16(x).view(np.float32).astype(np.float64)


def _exponent(M):
    c = 21 - int(np.floor(np.log2(M)))
    while M * 2.0 ** c >= 2 ** 22:
        c -= 1
    while M * 2.0 ** c < 2 ** 21:
        c += 1
    return c


def _digits(X):
    d0 = ((X + 128) % 256) - 128
    r = (X - d0) // 256
    d1 = ((r + 128) % 256) - 128
    d2 = (r - d1) // 256
    return d2, d1, d0


def test_digits_cover_every_value_below_2_22():
    X = np.arange(-(2 ** 22) + 1, 2 ** 22, 4099, dtype=np.int64)
    X = np.concatenate([X, [-(2 ** 22) + 1, 2 ** 22 - 1, 0, -1, 1, 127, 128, -128, -129, 65535, -65536]])
    d2, d1, d0 = _digits(X)
    for d in (d2, d1, d0):
        assert d.min() >= -128 and d.max() <= 127
    assert np.array_equal(65536 * d2 + 256 * d1 + d0, X)


def test_digit_sums_fit_s32():
    # the largest |sum(u * d)| over 128 terms: u <= 15, |d| <= 128
    assert 128 * 15 * 128 < 2 ** 31


def test_recombination_and_exactness():
    rng = np.random.default_rng(3)
    x = _groups(rng, 400)
    q = rng.integers(-8, 8, size=(400, 128)).astype(np.int64)
    u = q + 8
    for g in range(x.shape[0]):
        M = np.max(np.abs(x[g]))
        if M == 0:
            continue
        c = _exponent(M)
        xs = x[g] * 2.0 ** c                     # exact in float64 (bf16 values times a power of two)
        X = np.rint(xs).astype(np.int64)
        assert np.max(np.abs(X)) < 2 ** 22 and np.max(np.abs(X)) >= 2 ** 21
        d2, d1, d0 = _digits(X)
        A = [int(np.sum(u[g] * d)) for d in (d2, d1, d0)]
        assert all(abs(a) < 2 ** 31 for a in A)
        assert 65536 * A[0] + 256 * A[1] + A[2] - 8 * int(X.sum()) == int(np.sum(q[g] * X))
        big = np.abs(x[g]) >= M * 2.0 ** -13
        assert np.array_equal(X[big].astype(np.float64), xs[big])
        assert np.all(np.abs(X - xs) <= M * 2.0 ** -22 * 2.0 ** c)
