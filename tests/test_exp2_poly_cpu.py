"""The FMA-pipe exponential of the FP8 attention kernel, checked on the CPU.

The E4M3 attention kernel computes some of its probabilities 2^x without the
MUFU unit: x = n + f with n = round(x) (by adding and subtracting 1.5 * 2^23 in
float32), 2^f from a degree-2 polynomial in fused multiply-adds, and n added
to the float32 exponent field; x is clamped below at -127 first. This test
models those float32 steps with NumPy (IEEE round-to-nearest-even adds, fused
multiply-adds evaluated exactly in float64 and rounded once) and checks them
against numpy.exp2 over the whole input range the softmax can produce: the
relative error stays within the stated 1.8e-3, far below E4M3's half unit of
2^-4; -inf (masked keys) and anything below -127 give at most 2^-126, which
rounds to zero in E4M3 at every block scale the kernel applies; and x = 0
gives 1 to within the bound. The GPU tests check the kernel's outputs against
the float64 oracle within the derived E4M3 bounds.
"""
import numpy as np

F32 = np.float32
C0, C1, C2 = F32(1.0004431), F32(0.70344603), F32(0.23842734)
MAGIC = F32(12582912.0)          # 1.5 * 2^23
BOUND = 1.8e-3


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def exp2_poly2(x):
    x = np.asarray(x, dtype=F32)
    xc = np.maximum(x, F32(-127.0))
    t = (xc + MAGIC).astype(F32)
    n = (t - MAGIC).astype(F32)
    f = (xc - n).astype(F32)
    p = _fma32(f, np.full_like(f, C2), np.full_like(f, C1))
    p = _fma32(p, f, np.full_like(f, C0))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(F32)


def test_relative_error_over_the_softmax_range():
    # x = s * c - m (+ the FP8 V-scale shift): at most 8 above the running max,
    # and down to -inf
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-126, 9, dtype=np.float64) + 0.5,
                        np.arange(-126, 9, dtype=np.float64)]).astype(F32)
    got = exp2_poly2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= BOUND, float(rel.max())
    assert rel.max() >= 1e-3          # the bound is tight, not vacuous


def test_masked_and_tiny_inputs_vanish():
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.5, -127.0], dtype=F32)
    got = exp2_poly2(x)
    assert np.all(got >= 0) and np.all(got <= 2.0 ** -126)
    assert np.all(np.isfinite(got))


def test_exact_points():
    got = exp2_poly2(np.array([0.0, 1.0, -1.0, 8.0, -20.0], dtype=F32)).astype(np.float64)
    want = np.array([1.0, 2.0, 0.5, 256.0, 2.0 ** -20])
    assert np.all(np.abs(got / want - 1.0) <= BOUND)
