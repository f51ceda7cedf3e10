"""The arithmetic the 16-bit tensor-core path relies on, checked exactly with numpy's IEEE float16.

Weights (int4 g128): each weight row takes the power of two 2^k that puts its largest group scale in
[2^11, 2^12); then q * s * 2^k is an f16 value exactly (q in [-8, 7], s a bf16 scale) for every group whose
scale is at least 2^-25 of the row's largest.  Activations: each row takes the power of two that puts its
largest |x| in [2^13, 2^14); then every bf16 element within 2^27 of that largest is an f16 value exactly after
the scaling.  The NVFP4 weights: an e2m1 value times an E4M3 block scale is an f16 value exactly (at most 5
significant bits, magnitudes from 2^-10 to 2688).

(These are the exactness readings the 16-bit path is built on; the kernel itself is compared with the oracle by
the GPU parity tests.)
"""
import numpy as np

from weight_only_bit_route_b200 import synthetic as syn


def _bf16_values(a):
    return (syn.to_bf16_bits(np.asarray(a, np.float32)).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _pow2_into(M, lo):
    """k with M * 2^k in [2^lo, 2^(lo + 1))."""
    k = lo - int(np.floor(np.log2(M)))
    while M * 2.0 ** k >= 2.0 ** (lo + 1):
        k -= 1
    while M * 2.0 ** k < 2.0 ** lo:
        k += 1
    return k


def _exact_f16(v):
    return np.array_equal(v.astype(np.float16).astype(np.float64), v)


def test_int4_weights_exact_in_f16():
    rng = np.random.default_rng(21)
    for _ in range(300):
        # one weight row: 32 group scales spread over 2^-25 .. 1 of the largest, q over the full int4 range
        smax = float(2.0 ** rng.uniform(-20, 4))
        s = _bf16_values(smax * 2.0 ** -rng.uniform(0, 25, size=32))
        s[0] = _bf16_values([smax])[0]
        k = _pow2_into(s.max(), 11)
        q = rng.integers(-8, 8, size=(32, 128)).astype(np.float64)
        keep = s >= s.max() * 2.0 ** -25
        w = q[keep] * (s[keep] * 2.0 ** k)[:, None]
        assert _exact_f16(w)
        assert np.max(np.abs(w)) < 65504


def test_activations_exact_in_f16():
    rng = np.random.default_rng(22)
    for _ in range(300):
        x = _bf16_values(rng.standard_normal(512) * np.exp2(rng.uniform(-40, 10, size=512)))
        M = np.max(np.abs(x))
        k = _pow2_into(M, 13)
        keep = np.abs(x) >= M * 2.0 ** -27
        assert _exact_f16(x[keep] * 2.0 ** k)


def test_nvfp4_products_exact_in_f16():
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e2m1 = np.concatenate([e2m1, -e2m1])
    # every finite positive E4M3 value: subnormals m/8 * 2^-6, normals (1 + m/8) * 2^(e - 7)
    e4m3 = [m / 8 * 2.0 ** -6 for m in range(1, 8)]
    e4m3 += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    e4m3 = np.array(e4m3)
    assert e4m3.max() == 448.0 and len(e4m3) == 126
    assert _exact_f16(np.outer(e2m1, e4m3).ravel())
