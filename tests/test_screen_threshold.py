"""The survivor threshold of the screen-then-verify selection (the kernels'
survivor_threshold) must never fall below the exact threshold of the bound
it implements.  The kernel's formula is evaluated here in binary32 with every
approximate operation (square root, reciprocal square root, reciprocal)
pushed 2^-20 the wrong way -- far beyond their documented error -- and
compared with the exact threshold computed in fp64:

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


def kernel_threshold(M, a2, tau, e=-2.0 ** -20):
    M, a2, tau = f(M), f(a2), f(tau)
    alpha = f(f(f(np.sqrt(np.float64(max(a2, f(2.0 ** -126))))) * f(1 + e)) * f(1 + 2.0 ** -16))
    hb = f(f(0.5 * U_ * K2) * alpha)
    k3 = f(f(K3 * U_ * U_) * a2)
    c = f(f(f(M + k3) + tau) * f(1 + 2.0 ** -16))
    rho = f(f(f(1 / np.sqrt(np.float64(c))) * f(1 + e)) * f(1 + 2.0 ** -16))
    s = f(f(f(2 * hb) + f(c * rho)) * f(1 + 2.0 ** -15))
    den = f(f(1 - U_ * K1) - min(f(hb * rho), f(0.5)))
    assert den > 0.25
    num = f(f(f(f(s * s) + f(hb * s)) + k3) + tau)
    return f(f(num * f(f(1 / np.float64(den)) * f(1 + e))) * f(1 + 2.0 ** -10))


def test_kernel_threshold_dominates_the_exact_one():
    rng = np.random.default_rng(0)
    for _ in range(20000):
        a2 = 10.0 ** rng.uniform(-30, 8)
        r = rng.random()
        M = 0.0 if r < 0.05 else a2 * 10.0 ** rng.uniform(-20, 0.5)
        tau = 2.0 ** -120 + (2.0 ** -70 * 10.0 ** rng.uniform(-5, 5)) ** 2
        assert float(kernel_threshold(M, a2, tau)) >= exact_threshold(M, a2, tau), (M, a2, tau)


def test_threshold_is_tight_on_typical_blocks():
    # a block whose best loss is 1% of its energy: the threshold admits only
    # candidates within about 0.1% of the minimum (the 2^-10 widening)
    a2 = 16 * 300.0 ** 2
    M = 0.01 * a2
    T = float(kernel_threshold(M, a2, 2.0 ** -120, e=0.0))
    assert 1.0 < T / M < 1.0 + 2.0e-3
