"""Coordinate law of a random unit vector and its Lloyd-Max codebook (float64).

Test infrastructure (see ``oracle/__init__``).

Source: zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5
bits per channel", paragraph 2 -- after a random rotation the coordinates of
a vector follow a Beta distribution, which makes an optimal per-coordinate
scalar quantizer applicable. The pages do not print the density; the reading
used here is the exact law of one coordinate y of a point drawn uniformly on
the unit sphere S^{d-1}:

    f_d(y) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - y^2)^((d-3)/2),
    y in [-1, 1],

i.e. (y + 1)/2 ~ Beta((d-1)/2, (d-1)/2). "Optimal" is read as minimum mean
squared error for a fixed number of levels L = 2**bits, which is the
Lloyd-Max fixed point: thresholds at midpoints of adjacent centroids,
centroids at the conditional mean of each cell.

Plain steps, no acceleration:
  * CDF through the regularized incomplete beta function (library routine).
  * First moment of a cell in closed form:
        int_a^b y f_d(y) dy = C_d/(d-1) * ((1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)).
  * Lloyd iteration from Gaussian-quantile starting points until the largest
    centroid move is below 1e-15 (or 100000 sweeps).
  * Exact symmetry c[L-1-j] = -c[j] imposed at the end (the law is even).
  * Centroids rounded to float32 (the type both the oracle and the GPU get);
    thresholds recomputed in float64 as midpoints of the float32 centroids.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import betainc, gammaln
from scipy.stats import norm as _std_normal


def density_const(d: int) -> float:
    """C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)), the normaliser of f_d."""
    if d < 2:
        raise ValueError("d must be >= 2")
    return math.exp(gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0))


def coord_pdf(y, d: int):
    """f_d(y): density of one coordinate of a uniform point on S^{d-1}."""
    y = np.asarray(y, dtype=np.float64)
    out = np.zeros_like(y)
    inside = np.abs(y) < 1.0
    out[inside] = density_const(d) * (1.0 - y[inside] ** 2) ** ((d - 3) / 2.0)
    return out


def coord_cdf(y, d: int):
    """P(Y <= y) = I_{(y+1)/2}((d-1)/2, (d-1)/2) (regularized incomplete beta)."""
    y = np.clip(np.asarray(y, dtype=np.float64), -1.0, 1.0)
    a = (d - 1) / 2.0
    return betainc(a, a, (y + 1.0) / 2.0)


def coord_first_moment(a, b, d: int):
    """int_a^b y f_d(y) dy, in closed form (antiderivative of y(1-y^2)^k)."""
    a = np.clip(np.asarray(a, dtype=np.float64), -1.0, 1.0)
    b = np.clip(np.asarray(b, dtype=np.float64), -1.0, 1.0)
    e = (d - 1) / 2.0
    return density_const(d) / (d - 1) * ((1.0 - a * a) ** e - (1.0 - b * b) ** e)


def cell_edges(centroids) -> np.ndarray:
    """[-1, t_0, ..., t_{L-2}, 1] with t_j the midpoint of c_j and c_{j+1}."""
    c = np.asarray(centroids, dtype=np.float64)
    return np.concatenate(([-1.0], (c[:-1] + c[1:]) / 2.0, [1.0]))


def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_sweeps: int = 100000) -> np.ndarray:
    """Float64 Lloyd-Max centroids (ascending, exactly symmetric) for f_d."""
    if bits < 1 or bits > 8:
        raise ValueError("bits must be in 1..8")
    L = 1 << bits
    # Starting points: quantiles of N(0, 1/d), the large-d limit of f_d.
    c = _std_normal.ppf((np.arange(L) + 0.5) / L) / math.sqrt(d)
    c = np.clip(c, -0.999, 0.999)
    for _ in range(max_sweeps):
        edges = cell_edges(c)
        mass = np.diff(coord_cdf(edges, d))
        moment = coord_first_moment(edges[:-1], edges[1:], d)
        c_new = moment / mass
        step = np.max(np.abs(c_new - c))
        c = c_new
        if step < tol:
            break
    c = (c - c[::-1]) / 2.0
    return c


def fit_codebook(d: int, bits: int):
    """(centroids_f32, thresholds_f64) used by both quantizer implementations.

    The float32 centroids are what the CUDA library receives; the thresholds
    are midpoints of those float32 values, exact in float64.
    """
    c32 = lloyd_max(d, bits).astype(np.float32)
    c64 = c32.astype(np.float64)
    thresholds = (c64[:-1] + c64[1:]) / 2.0
    return c32, thresholds


def mse_per_vector(d: int, centroids) -> float:
    """E || u - Pi^T c[idx(Pi u)] ||^2 for u uniform on S^{d-1} (MSE-only stage).

    By rotation invariance each coordinate of y = Pi u has law f_d, and the
    quantizer acts coordinate-wise, so the per-vector error is d times the
    per-coordinate error, integrated cell by cell with nearest-centroid cells:
        d * sum_j int_cell_j (y - c_j)^2 f_d(y) dy
      = d * (E[y^2] - 2 sum_j c_j M1_j + sum_j c_j^2 P_j),  E[y^2] = 1/d.
    """
    c = np.asarray(centroids, dtype=np.float64)
    edges = cell_edges(c)
    mass = np.diff(coord_cdf(edges, d))
    moment = coord_first_moment(edges[:-1], edges[1:], d)
    return float(d * (1.0 / d - 2.0 * np.sum(c * moment) + np.sum(c * c * mass)))

