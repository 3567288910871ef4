"""Coefficients of the polynomial 2^f ~ c0 + c1 f + ... + c5 f^5 on [-1/2, 1/2] used by the
fused attention kernel for part of its exponentials (the rest use the hardware ex2).

Method: 2^t = 2^j * 2^f with j = rint(t) and f = t - j in [-1/2, 1/2]; c0 = 1 exactly (so
that t = 0, the row maximum, gives exactly 1), and c1..c5 are a weighted least-squares fit of
2^f - 1 in relative error of 2^f on 2000 Chebyshev nodes of [-1/2, 1/2] (close to the minimax
polynomial of that degree), then rounded to float32. `check()` evaluates
the polynomial the way the kernel does (float32 Horner steps with fused multiply-adds, each
rounded once) and returns the largest relative error against 2^f in float64.

Run as a script to print the float32 coefficients and the error bound.
"""
import numpy as np

DEGREE = 5


def fit(degree=DEGREE, nodes=2000):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))  # Chebyshev nodes of [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)[:, 1:] / y[:, None]  # relative-error weighting
    c, *_ = np.linalg.lstsq(V, (y - 1.0) / y, rcond=None)
    return np.float32(np.concatenate([[1.0], c]))


def fma32(a, b, c):
    """float32 fused multiply-add: exact product and sum in float64, one rounding to float32."""
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def horner32(c, f):
    acc = np.float32(c[-1])
    for ck in c[-2::-1]:
        acc = fma32(acc, f, np.float32(ck))
    return acc


def check(c, samples=200001):
    f = np.float32(np.linspace(-0.5, 0.5, samples))
    approx = np.array([horner32(c, x) for x in f], dtype=np.float64)
    return float(np.max(np.abs(approx / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, ci in enumerate(c):
        print(f"c{i} = {float(ci):.9e}f  (0x{np.float32(ci).view(np.uint32):08x})")
    print("max relative error (float32 evaluation):", check(c))
