"""The survivor threshold of the screen-then-verify selection (the kernels'
survivor_threshold) must never fall below the exact threshold of the bound
it implements.  The kernel's formula -- the square-root term of the bound
bounded linearly, sqrt(z) <= (z/(g alpha) + g alpha)/2 with g = 2^-8, giving
D(z) <= a z + b and the threshold (M + 2b)/(1 - a)^2 widened by 2^-10 -- is
evaluated here in binary32 exactly as the kernels evaluate it (one fused
multiply-add for b, one for M + 2b, one product) and compared with the exact
threshold computed in fp64 from the bound itself:

  U   the root of U = M + u(K1 U + K2 alpha sqrt(U)) + K3 u^2 alpha^2 + tau
  T*  (U + b sqrt(U)/2 + K3 u^2 alpha^2 + tau) / (1 - u K1 - b / (2 sqrt(U))),
      b = u K2 alpha

over random minima M, norms alpha^2 and allowances tau spanning the ranges
the kernels meet (including M = 0, a block reproduced exactly)."""
import numpy as np

U_, K1, K2, K3 = 2.0 ** -24, 128.0, 16.0, 64.0
f = np.float32


def exact_threshold(M, a2, tau):
    al = np.sqrt(a2)
    b = U_ * K2 * al
    g = K3 * U_ * U_ * a2 + tau
    a1 = 1 - U_ * K1
    sU = (b + np.sqrt(b * b + 4 * a1 * (M + g))) / (2 * a1)
    den = 1 - U_ * K1 - b / (2 * sU)
    return (sU * sU + 0.5 * b * sU + g) / den


def _fma32(a, b, c):
    """binary32 fused multiply-add: the exact a*b + c rounded once (the product
    of two binary32 values is exact in fp64, the sum rounds at most once more
    there, far below binary32 resolution away from ties)."""
    return f(np.float64(f(a)) * np.float64(f(b)) + np.float64(f(c)))


def kernel_threshold(M, a2, tau):
    """The kernels' survivor_threshold in binary32."""
    g = 2.0 ** -8
    A = f(U_ * (K1 + K2 / (2.0 * g)))
    B = f(0.5 * U_ * K2 * g + K3 * U_ * U_)
    C = f(f(1.0 + 2.0 ** -10) / f(f(f(1.0) - A) * f(f(1.0) - A)))
    b = _fma32(a2, f(B * f(1.0 + 2.0 ** -16)), tau)
    return f(_fma32(2.0, b, M) * C)


def test_kernel_threshold_dominates_the_exact_one():
    rng = np.random.default_rng(0)
    for _ in range(20000):
        a2 = 10.0 ** rng.uniform(-30, 8)
        r = rng.random()
        M = 0.0 if r < 0.05 else a2 * 10.0 ** rng.uniform(-20, 0.5)
        tau = 2.0 ** -120 + (2.0 ** -70 * 10.0 ** rng.uniform(-5, 5)) ** 2
        assert float(kernel_threshold(M, a2, tau)) >= exact_threshold(M, a2, tau), (M, a2, tau)


def test_kernel_threshold_on_binary32_boundaries():
    # minima and norms at binary32 extremes: zero, the smallest normal, values
    # whose products round, and the largest norms the range check admits
    for a2 in (2.0 ** -126, 1.0, 3.0, 16 * 1536.0 ** 2, 2.0 ** 100):
        for M in (0.0, 2.0 ** -149, 2.0 ** -126, 1e-30 * a2, 1e-4 * a2, a2):
            for tau in (2.0 ** -120, 2.0 ** -100):
                assert float(kernel_threshold(M, a2, tau)) >= exact_threshold(M, a2, tau), (M, a2, tau)


def test_threshold_is_tight_on_typical_blocks():
    # a block whose best loss is 1% of its energy: the threshold admits only
    # candidates within about 0.1% of the minimum (the 2^-10 widening)
    a2 = 16 * 300.0 ** 2
    M = 0.01 * a2
    T = float(kernel_threshold(M, a2, 2.0 ** -120))
    assert 1.0 < T / M < 1.0 + 2.0e-3
