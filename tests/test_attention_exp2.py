"""The attention softmax's FMA-pipe 2^t (a third of its exponentials): its arithmetic restated in
float32 with fused multiply-adds (a product of two float32 values is exact in float64, so rounding
a*b + c once to float32 is the fused operation) and checked against 2^t over the range the softmax
uses, t in [-125, 8]: relative error at most 2.7e-6, powers of two at integers to that bound, and
2^-125 for -inf.  The coefficients and the rounding / exponent steps are those of exp2_fma_pipe in the
attention kernel's source."""
import numpy as np

C = [np.float32(0.99999928), np.float32(0.69312179), np.float32(0.24024744), np.float32(0.055918001),
     np.float32(0.0095701320)]


def _fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_pipe(t):
    t = np.asarray(t, dtype=np.float32)
    tc = np.maximum(t, np.float32(-125.0))
    big = np.float32(12582912.0)
    r = (tc + big).astype(np.float32)
    n = (r - big).astype(np.float32)
    f = _fma(n, np.full_like(n, -1.0), tc)
    q = _fma(np.full_like(f, C[4]), f, np.full_like(f, C[3]))
    q = _fma(q, f, np.full_like(f, C[2]))
    q = _fma(q, f, np.full_like(f, C[1]))
    q = _fma(q, f, np.full_like(f, C[0]))
    bits = (q.view(np.uint32).astype(np.uint64) + (r.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(1)
    t = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-30.0, 8.0, 200000)]).astype(np.float32)
    got = exp2_fma_pipe(t).astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) <= 2.7e-6


def test_integers_and_masked_scores():
    t = np.arange(-125, 9, dtype=np.float32)
    got = exp2_fma_pipe(t).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(t.astype(np.float64)) - 1.0)) <= 2.7e-6
    masked = exp2_fma_pipe(np.array([-np.inf, -1e30, -200.0], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(masked / 2.0 ** -125 - 1.0) <= 2.7e-6)
