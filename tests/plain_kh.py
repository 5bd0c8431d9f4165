"""Independent plain-loop Kernel Halving for tiny inputs (pure Python floats, no numpy).

Written from the same definitions as the oracle but without Gram or pair-difference
matrices: alpha is evaluated as psi(x) - psi(y) with psi = sum over kept points of
kappa(p, .) minus the sum over discarded points, recomputed from the points at
every step.  Used only by the oracle pin tests.
"""
import math


def _dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def plain_kernel_halving(K, V, scale, u):
    """K, V: lists of n rows; u: list of m uniforms.  Returns (keep_first list, margins, kernel scale)."""
    n = len(K)
    m = n // 2
    c2 = max(abs(x) for row in V for x in row) ** 2

    def kap(a, b):
        return math.exp(scale * _dot(K[a], K[b])) * (_dot(V[a], V[b]) + c2)

    kscale = max(kap(i, i) for i in range(n))
    kept, disc = [], []
    sigma2 = 0.0
    C = math.sqrt(2.0 * math.log(4.0 * m))       # sqrt(2 ln(2/delta_i)), delta_i = 1/(2m)
    keep, margins = [], []
    for i in range(m):
        x, y = 2 * i, 2 * i + 1

        def psi(z):
            return sum(kap(p, z) for p in kept) - sum(kap(p, z) for p in disc)

        alpha = psi(x) - psi(y)
        b2 = kap(x, x) + kap(y, y) - 2.0 * kap(x, y)
        if b2 <= 0.0:
            keep.append(True)
            margins.append(math.inf)
            kept.append(x)
            disc.append(y)
            continue
        a = max(math.sqrt(b2) * math.sqrt(sigma2) * C, b2)
        p = min(1.0, max(0.0, 0.5 * (1.0 - alpha / a)))
        kx = u[i] < p
        keep.append(kx)
        margins.append(abs(alpha - a * (1.0 - 2.0 * u[i])))
        if kx:
            kept.append(x)
            disc.append(y)
        else:
            kept.append(y)
            disc.append(x)
        sigma2 = sigma2 + b2 * max(0.0, 1.0 + (b2 - 2.0 * a) * sigma2 / (a * a))
    return keep, margins, kscale
