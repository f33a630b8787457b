"""The FMA-pipe exponentials of the attention kernel, checked on the CPU.

The tensor-core attention kernel computes some of its probabilities 2^x
without the MUFU unit (which does 16 exponentials per clock per SM): x = n + f
with n = round(x) (by adding and subtracting 1.5 * 2^23 in float32), 2^f from
a polynomial in fused multiply-adds, and n added to the float32 exponent
field; x is clamped below at -126 first (with n >= -126 the exponent field
cannot borrow into the sign bit, even where 2^f < 1). The E4M3 instance uses
degree 2, the bf16 instance degree 3.

This test models those float32 steps with NumPy (IEEE round-to-nearest-even
adds, fused multiply-adds evaluated exactly in float64 and rounded once) and
checks them against numpy.exp2 over the whole input range the softmax can
produce (at most 8 above the running maximum, down to -inf):
  * degree 2: relative error within 1.8e-3, far below E4M3's unit roundoff 2^-4;
  * degree 3: relative error within 8e-5, far below bf16's unit roundoff 2^-8;
  * -inf (masked keys) and anything below -126 give a finite non-negative
    value below 2^-125, which is zero after rounding to E4M3 at every block
    scale the kernel applies, and nothing next to a row sum of at least 1.
Below about 2^-125 the exponent field reaches 0 and the result is read as a
subnormal, so the relative-error range starts at -125.
The GPU tests check the kernel's outputs against the float64 oracle.
"""
import numpy as np
import pytest

F32 = np.float32
MAGIC = F32(12582912.0)          # 1.5 * 2^23
COEFFS = {   # highest degree first, as the kernel evaluates them (Horner)
    2: (F32(0.23842734), F32(0.70344603), F32(1.0004431)),
    3: (F32(0.0551715), F32(0.24261096), F32(0.69326097), F32(0.99992806)),
}
BOUNDS = {2: 1.8e-3, 3: 8e-5}


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def exp2_poly(x, degree):
    x = np.asarray(x, dtype=F32)
    xc = np.maximum(x, F32(-126.0))
    t = (xc + MAGIC).astype(F32)
    n = (t - MAGIC).astype(F32)
    f = (xc - n).astype(F32)
    c = COEFFS[degree]
    p = _fma32(f, np.full_like(f, c[0]), np.full_like(f, c[1]))
    for ck in c[2:]:
        p = _fma32(p, f, np.full_like(f, ck))
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(F32)


@pytest.mark.parametrize("degree", [2, 3])
def test_relative_error_over_the_softmax_range(degree):
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 8, dtype=np.float64) + 0.5,
                        np.arange(-125, 9, dtype=np.float64)]).astype(F32)
    got = exp2_poly(x, degree).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= BOUNDS[degree], float(rel.max())
    assert rel.max() >= BOUNDS[degree] / 3          # the bound is tight, not vacuous


@pytest.mark.parametrize("degree", [2, 3])
def test_masked_and_tiny_inputs_vanish(degree):
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.5, -127.0, -126.7, -126.2, -126.0],
                 dtype=F32)
    got = exp2_poly(x, degree)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -125)
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("degree", [2, 3])
def test_exact_points(degree):
    got = exp2_poly(np.array([0.0, 1.0, -1.0, 8.0, -20.0], dtype=F32), degree).astype(np.float64)
    want = np.array([1.0, 2.0, 0.5, 256.0, 2.0 ** -20])
    assert np.all(np.abs(got / want - 1.0) <= BOUNDS[degree])
