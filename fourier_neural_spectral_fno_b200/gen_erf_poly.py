"""Generate the erf polynomial the CUDA kernels use for the exact-form GELU.

    python -m fourier_neural_spectral_fno_b200.gen_erf_poly

Method: a Chebyshev least-squares fit of erf(t) on [0, T] (T = 3.9, where
1 - erf(T) = 3.5e-8, below float32 resolution at 1), converted to the monomial
basis of the centred, scaled variable x = (t - T/2) / (T/2) in [-1, 1] and
evaluated in float32 by Horner's rule; erf(t) = 1 for t > T and erf is odd.
The scaled variable keeps the monomial coefficients O(1), so the float32
evaluation stays accurate (a fit in t itself does not).  The kernels use the
printed coefficients; tests/test_gelu_poly.py re-derives them and checks the
float32 evaluation against the double-precision erf.
"""

from __future__ import annotations

import numpy as np

T = 3.9
DEGREE = 18


def fit(t_max: float = T, degree: int = DEGREE):
    """Monomial coefficients (lowest first) of erf(m + h x), m = h = t_max / 2."""
    from numpy.polynomial import chebyshev as C
    from scipy.special import erf

    m = h = 0.5 * t_max
    x = np.cos(np.linspace(0.0, np.pi, 20000))
    cheb = C.chebfit(x, erf(m + h * x), degree)
    return np.asarray(C.cheb2poly(cheb), dtype=np.float64)


def eval_f32(coef, t):
    """float32 Horner evaluation as the kernels do it (t >= 0)."""
    c32 = np.asarray(coef, dtype=np.float64).astype(np.float32)
    m = np.float32(0.5 * T)
    inv_h = np.float32(1.0 / (0.5 * T))
    tc = np.minimum(np.asarray(t, np.float32), np.float32(T))
    x = ((tc - m) * inv_h).astype(np.float32)
    acc = np.full_like(x, c32[-1])
    for c in c32[-2::-1]:
        acc = (acc * x + c).astype(np.float32)
    return np.where(np.asarray(t) > T, np.float32(1.0), acc)


def main() -> None:
    coef = fit()
    print(f"// erf(t) ~= P((t - {0.5 * T}) / {0.5 * T}), t in [0, {T}], degree {DEGREE}, highest first")
    print(", ".join(f"{np.float32(c)!r}f".replace("np.float32(", "").replace(")", "")
                    for c in coef[::-1]))


if __name__ == "__main__":
    main()
