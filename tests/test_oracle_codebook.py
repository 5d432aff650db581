"""Pins for the oracle's Lloyd-Max codebook (CPU only): Max's published table,
the closed-form distortion, and the centroid / midpoint optimality conditions
checked by independent numerical integration."""
import math
import os

import numpy as np
import scipy.integrate
import scipy.stats

from oracle import codebook as CB

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "max1960_gaussian_16level.txt")


def _max_table():
    xs, ys, dist = [], [], None
    for line in open(GOLDEN):
        if line.startswith("# distortion"):
            dist = float(line.split()[-1])
        if line.startswith("#") or not line.strip():
            continue
        _, x, y = line.split()
        xs.append(math.inf if x == "inf" else float(x))
        ys.append(float(y))
    return np.array(xs), np.array(ys), dist


def test_matches_max_1960_table():
    xs, ys, dist = _max_table()
    c, t, _ = CB.lloyd_max_gaussian(16, 1.0)
    # printed to 4 significant digits, a few off by one unit in the last place:
    # allow 1.5 units of the 4th significant digit of each printed value
    def unit(v):
        return 10.0 ** (np.floor(np.log10(np.abs(v))) - 3)
    assert (np.abs(c[8:] - ys) <= 1.5 * unit(ys)).all(), (c[8:], ys)
    assert (np.abs(t[8:] - xs[:-1]) <= 1.5 * unit(xs[:-1])).all(), (t[8:], xs)
    assert abs(CB.gaussian_mse(c) - dist) < 1e-5


def test_symmetric_and_sorted():
    c, t, _ = CB.lloyd_max_gaussian(16, 0.3)
    assert (np.diff(c) > 0).all()
    assert (c == -c[::-1]).all()
    cb16 = CB.lloyd_max_f16(16, 1 / math.sqrt(128))
    assert (cb16 == -cb16[::-1]).all()


def test_optimality_conditions_by_quadrature():
    sigma = 1 / math.sqrt(128)
    c, t, _ = CB.lloyd_max_gaussian(16, sigma)
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    pdf = scipy.stats.norm(scale=sigma).pdf
    for i in range(16):
        a, b = edges[i], edges[i + 1]
        mass = scipy.integrate.quad(pdf, a, b)[0]
        mean = scipy.integrate.quad(lambda z: z * pdf(z), a, b)[0] / mass
        assert abs(mean - c[i]) < 1e-9 * max(1.0, abs(c[i]) / sigma)
    # thresholds are midpoints
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-15)


def test_mse_closed_form_matches_quadrature():
    c, _, _ = CB.lloyd_max_gaussian(16, 1.0)
    edges = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    pdf = scipy.stats.norm.pdf
    q = sum(scipy.integrate.quad(lambda z, ci=ci: (z - ci) ** 2 * pdf(z), edges[i], edges[i + 1])[0]
            for i, ci in enumerate(c))
    assert abs(q - CB.gaussian_mse(c)) < 1e-10
