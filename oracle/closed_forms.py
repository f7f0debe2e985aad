"""Analytic quantities of the P-cast analysis (test infrastructure only).

Source: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
Optimality of S=2^8", technical summary, section 2 ("Theoretical framework",
"Optimisation 2: the optimality of S = 256") and section 3 (item 1, the
threshold Delta_c); the Italian summary "Riepilogo Tecnico: Precisione P-Cast
in FP8 Attention" gives the same formulas in its sections 2 and 3.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import integrate
from scipy.stats import norm

#: 10 ln 2: the E4M3 round-to-zero threshold 2^-10 in natural-log units, the
#: "6.93" of the closed form (section 2 of the summary names it so).
LN2_TEN = 10.0 * math.log(2.0)


def delta_k(k: int) -> float:
    """Expected maximum of k independent standard normals (section 2: the
    sink block's expected maximum, "about 1.0 for k = 4").

    E[max] = integral of x * k * phi(x) * Phi(x)^(k-1) over the real line,
    evaluated by adaptive quadrature.
    """
    if k < 1:
        raise ValueError("k >= 1")
    f = lambda x: x * k * norm.pdf(x) * norm.cdf(x) ** (k - 1)
    val, _ = integrate.quad(f, -12.0, 12.0, epsabs=1e-12, epsrel=1e-12, limit=200)
    return float(val)


def f_forward(delta, S, k: int = 4):
    """Fraction of non-sink P values that round to zero under forward KV order
    with static scale S (section 2): F(Delta, S) = Phi(Delta + delta_k - 10 ln 2 - ln S).

    The plug-in form: the running maximum is the sink block's expected
    maximum Delta + delta_k, and the non-sink logits are standard normal.
    """
    return norm.cdf(np.asarray(delta, dtype=np.float64) + delta_k(k) - LN2_TEN
                    - np.log(np.asarray(S, dtype=np.float64)))


def delta_c(S, k: int = 4):
    """Collapse threshold Delta_c = 10 ln 2 + ln S - delta_k (section 3, item 1):
    the sink strength at which F(Delta, S) = 1/2."""
    return LN2_TEN + np.log(np.asarray(S, dtype=np.float64)) - delta_k(k)


def f_row(row_max, row_sigma, S) -> float:
    """The same underflow probability conditioned on each row's realised running
    maximum m_i and non-sink logit standard deviation sigma_i, averaged over
    rows: mean_i Phi((m_i - 10 ln 2 - ln S) / sigma_i).

    A key j of row i underflows when P*S = exp(s_ij - m_i) * S <= 2^-10,
    i.e. s_ij <= m_i - 10 ln 2 - ln S; with s_ij ~ N(0, sigma_i^2) that has
    probability Phi((m_i - 10 ln 2 - ln S) / sigma_i).  Averaging over rows
    (instead of plugging in E[m]) removes the Jensen gap of the plug-in form
    in the tails.
    """
    m = np.asarray(row_max, dtype=np.float64)
    s = np.asarray(row_sigma, dtype=np.float64)
    return float(np.mean(norm.cdf((m - LN2_TEN - math.log(S)) / s)))


def dp_closed_form(S: float) -> float:
    """Maximal normalised quantisation step d_p(S) (section 2, condition 2).

    For P in (0, 1], P*S lies in (0, S]; the widest E4M3 step met there is the
    one just below S, whose spacing is 2^(floor(log2 S-) - 3) (three mantissa
    bits); dividing by S puts it back in units of P.  For S = 2^k this is
    2^-4 exactly; between powers of two it rises towards 2^-3 (the sawtooth).
    Valid for 2^-6 < S <= 448 (normal range, no saturation).
    """
    if not (2.0 ** -6 < S <= 448.0):
        raise ValueError("d_p(S) is defined here for 2^-6 < S <= 448")
    e = math.floor(math.log2(S))
    if 2.0 ** e == S:
        e -= 1  # S is itself a power of two: the binade just below it
    return 2.0 ** (e - 3) / S


def dp_from_grid(S: float, positive_grid) -> float:
    """d_p(S) by brute force over the E4M3 grid: the gap of the grid interval
    that holds values just below S, divided by S.  ``positive_grid`` is the
    sorted list of non-negative finite E4M3 values (from the codec)."""
    g = np.asarray(sorted(set(float(x) for x in positive_grid)))
    if not (g[0] == 0.0 and g[-1] >= S):
        raise ValueError("grid must start at 0 and reach S")
    idx = int(np.searchsorted(g, S, side="left"))  # g[idx-1] < S <= g[idx]
    return float((g[idx] - g[idx - 1]) / S)
