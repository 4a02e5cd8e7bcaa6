"""Host checks of the per-element bound the GPU parity tests apply (tests/parity.py):
2e-2 wherever the bf16 rounding of the output leaves room for it (|ref| < 8),
half a bf16 ulp plus the same 4.4e-3 of pre-rounding error above that."""
import numpy as np

from parity import DELTA, MAX_ABS, bound, compare, half_ulp_bf16


def test_half_ulp_of_bf16():
    x = np.array([1.0, 1.5, 3.99, 4.0, 7.99, 8.0, 15.9, 16.0, -5.0])
    want = np.array([2 ** -8, 2 ** -8, 2 ** -7, 2 ** -6, 2 ** -6, 2 ** -5, 2 ** -5, 2 ** -4, 2 ** -6])
    assert np.array_equal(half_ulp_bf16(x), want)


def test_bound_is_the_plain_bound_below_eight():
    r = np.linspace(-7.999, 7.999, 10001)
    assert np.all(bound(r) == MAX_ABS)
    assert abs(DELTA - (0.02 - 2 ** -6)) < 1e-15


def test_bound_widens_only_by_the_rounding_above_eight():
    r = np.array([8.0, -9.5, 15.99, 16.0, 31.0])
    assert np.allclose(bound(r), half_ulp_bf16(r) + DELTA)
    assert np.all(bound(r) > MAX_ABS)


def test_compare_uses_the_plain_bound():
    ref = np.full(100, 5.0)
    ok, st = compare(ref + 0.019, ref)
    assert ok and abs(st["max_abs"] - 0.019) < 1e-12
    ok, _ = compare(ref + 0.021, ref)     # 2.1e-2 at |ref| = 5 fails, whatever the rounding there
    assert not ok
    big = np.full(100, 12.0)
    ok, st = compare(big + 0.035, big)   # 2^-5 + 3.5e-3 at |ref| = 12: within the widened bound
    assert ok and st["n_above_8"] == 100
    ok, _ = compare(big + 0.037, big)
    assert not ok
