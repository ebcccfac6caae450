"""Fits the polynomials behind the kernels' erf-form GeLU and prints them as C constants.

    python gated_linear_recurrence_conv1d_b200/csrc/gelu_tail_fit.py            (forward)
    python gated_linear_recurrence_conv1d_b200/csrc/gelu_tail_fit.py --precise  (backward)

GeLU(y) = y Phi(y) = max(y, 0) - s Q(s) with s = |y| and Q the upper tail of the standard normal
distribution.  Q(s) = exp(-s^2 / 2) R(s), where R(s) = Q(s) exp(s^2 / 2) is smooth and slowly
varying on [0, inf) (R(0) = 1/2, R(s) ~ 1 / (s sqrt(2 pi)) for large s).  The kernels evaluate
exp(-s^2 / 2) with one hardware exp2 and R by this polynomial in s, clamped to s <= S_MAX (for
larger s, s exp(-s^2 / 2) R(s) < 2e-7).  A Chebyshev least-squares fit of degree DEG on
[0, S_MAX], converted to powers of s, keeps the GeLU's absolute error below 2e-6 in fp32 Horner
form (printed below together with the constants).
"""
import numpy as np
from scipy.special import erfc

S_MAX = 5.5
DEG = 10


def fit():
    s = np.linspace(0.0, S_MAX, 20001)
    r = 0.5 * erfc(s / np.sqrt(2.0)) * np.exp(s * s / 2.0)
    cheb = np.polynomial.chebyshev.Chebyshev.fit(s, r, DEG, domain=[0.0, S_MAX])
    return cheb.convert(kind=np.polynomial.Polynomial).coef.astype(np.float32)


def gelu_error(coef):
    y = np.linspace(-12.0, 12.0, 400001)
    s = np.abs(y)
    sc = np.minimum(s, S_MAX).astype(np.float32)
    acc = np.full_like(sc, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        acc = acc * sc + coef[k]
    approx = np.maximum(y, 0.0) - s * np.exp(-s * s / 2.0) * acc.astype(np.float64)
    exact = y * 0.5 * erfc(-y / np.sqrt(2.0))
    return float(np.max(np.abs(approx - exact)))


# The backward needs Phi itself (GeLU' = Phi + v phi) to about 1e-7: R of degree PDEG in the
# centred variable t = (s - P_SMAX / 2) / (P_SMAX / 2), whose power-basis coefficients stay small,
# so that fp32 Horner keeps the fit's accuracy.
PDEG = 14
P_SMAX = 5.5


def fit_precise():
    s = np.linspace(0.0, P_SMAX, 200001)
    r = 0.5 * erfc(s / np.sqrt(2.0)) * np.exp(s * s / 2.0)
    t = (s - P_SMAX / 2) / (P_SMAX / 2)
    cheb = np.polynomial.chebyshev.Chebyshev.fit(t, r, PDEG, domain=[-1.0, 1.0])
    return cheb.convert(kind=np.polynomial.Polynomial).coef.astype(np.float32)


def phi_error(coef):
    s = np.linspace(0.0, P_SMAX, 200001)
    t = ((s - P_SMAX / 2) / (P_SMAX / 2)).astype(np.float32)
    acc = np.full_like(t, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        acc = (acc * t + coef[k]).astype(np.float32)
    q = np.exp(-s * s / 2.0) * acc.astype(np.float64)
    return float(np.max(np.abs(q - 0.5 * erfc(s / np.sqrt(2.0)))))


if __name__ == "__main__":
    import sys
    if "--precise" in sys.argv:
        c = fit_precise()
        print(f"// degree {PDEG} in t = (s - {P_SMAX / 2}) / {P_SMAX / 2}, max |Phi error| {phi_error(c):.2e} (fp32 Horner)")
        for k, v in enumerate(c):
            print(f"constexpr float kPhiR{k} = {float(v):.9e}f;")
    else:
        c = fit()
        print(f"// degree {DEG} on [0, {S_MAX}], max |GeLU error| {gelu_error(c):.2e}")
        for k, v in enumerate(c):
            print(f"constexpr float kGeluR{k} = {float(v):.9e}f;")
