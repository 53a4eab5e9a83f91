"""Coefficients of the degree-3 polynomial p(f) ~ 2^f on f in [-1/2, 1/2] used
by the attention kernel's FMA-pipe exponential (exp2 split as
2^x = 2^round(x) * 2^(x - round(x))).

Method: relative-error minimax by iteratively reweighted least squares
(Lawson's algorithm) on a dense grid, starting from a Chebyshev-node
least-squares fit.  Run it to reprint the constants and their error bound:

    python -m block_sparse_attention_psa_b200.csrc.gen_exp2_poly
"""

import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5          # dense Chebyshev-spaced grid on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        A = V * (w / y)[:, None]
        c, *_ = np.linalg.lstsq(A, w, rcond=None)          # minimise sum w^2 (p/y - 1)^2
        r = np.abs(V @ c / y - 1.0)
        w = w * (r / r.max() + 1e-12) ** 0.5               # Lawson reweighting towards minimax
        w /= w.max()
    err = np.abs(V @ c / y - 1.0).max()
    return c, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{x:.9e}" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
