"""The kernels compute the log bucket of a distance x (reading r10) without
branches: for x >= 2^S they convert x to float rounding toward zero and read
(e - S + 1) 2^S + (top S bits below the leading one) off the float's bits as
(bits >> (23 - S)) - (126 + S) 2^S.  This checks that identity against the
oracle's bucket (host only; numpy stands in for the conversion: truncate x to
24 significant bits, then an exact float32 conversion)."""
import numpy as np

from oracle import hstu_oracle as F


def _float_rz_bits(x):
    x = np.asarray(x, np.int64)
    e = np.zeros_like(x)
    nz = x > 0
    e[nz] = np.frexp(x[nz].astype(np.float64))[1] - 1  # floor(log2 x), exact for x < 2^53
    sh = np.maximum(e - 23, 0)
    xt = (x >> sh) << sh
    return xt.astype(np.float32).view(np.uint32).astype(np.int64)


def _bucket_from_float(x, S, N):
    x = np.asarray(x, np.int64)
    big = (_float_rz_bits(x) >> (23 - S)) - ((126 + S) << S)
    return np.minimum(np.where(x < (1 << S), x, big), N - 1)


def test_float_exponent_bucket_equals_the_oracle_bucket():
    rng = np.random.default_rng(7)
    p2 = 1 << np.arange(31, dtype=np.int64)
    xs = np.unique(np.concatenate([np.arange(0, 1 << 14), rng.integers(0, (1 << 31) - 1, 200_000),
                                   p2 - 1, p2[:-1], p2[:-1] + 1, [(1 << 31) - 1]]))
    for S in range(0, 21):
        for N in (1, 2, 32, 128, 256, 4096, 1 << 20):
            assert np.array_equal(_bucket_from_float(xs, S, N), F.log_bucket(xs, N, S)), (S, N)


def test_planted_mistake_is_caught():
    """An off-by-one in the subtracted constant must fail the identity."""
    xs = np.arange(0, 5000, dtype=np.int64)
    S, N = 4, 128
    wrong = np.minimum(np.where(xs < (1 << S), xs,
                                (_float_rz_bits(xs) >> (23 - S)) - ((127 + S) << S)), N - 1)
    assert not np.array_equal(wrong, F.log_bucket(xs, N, S))
