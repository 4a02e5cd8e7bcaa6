"""Error bound of the FMA-pipe 2^x used for a quarter of the softmax
exponentials (csrc/ptx.cuh, exp2_fma_x2): round-to-nearest range reduction
with the 1.5 * 2^23 constant, a cubic for 2^f on [-1/2, 1/2], and the exponent
add.  The float32 steps are replayed in numpy (each fused multiply-add rounded
once to float32) and compared with 2^x in float64."""
import numpy as np

C = [np.float32(0.999928057), np.float32(0.693260968), np.float32(0.242611125), np.float32(0.0551716648)]
MAGIC = np.float32(12582912.0)


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_emulated(x):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    j = (t - MAGIC).astype(np.float32)
    f = fma32(j, np.full_like(j, -1.0), x)
    p = fma32(np.full_like(f, C[3]), f, np.full_like(f, C[2]))
    p = fma32(p, f, np.full_like(f, C[1]))
    p = fma32(p, f, np.full_like(f, C[0]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.random.default_rng(0).uniform(-40, 8, 1_000_000).astype(np.float32)])
    got = exp2_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.0e-4, rel.max()       # the cubic's 7.5e-5, far below bf16's 2^-9 step
    assert np.all(np.isfinite(got))
    # at the bottom of the range the result is subnormal and loses a little more
    edge = np.linspace(-126, -125, 10001, dtype=np.float32)
    rel = np.abs(exp2_emulated(edge).astype(np.float64) / np.exp2(edge.astype(np.float64)) - 1.0)
    assert rel.max() < 2.0e-4, rel.max()


def test_integers_and_underflow():
    x = np.arange(-125, 9, dtype=np.float32)
    got = exp2_emulated(x).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)
    # below the range (keys past N have score -inf): tiny, non-negative, never NaN
    tiny = exp2_emulated(np.array([-126.0, -126.5, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 1.2e-38), tiny
