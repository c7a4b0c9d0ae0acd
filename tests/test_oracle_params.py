"""Pins of the oracle's parameter generation (random streams, rotation, QJL
matrix, Lloyd-Max codebooks) against things fixed outside the oracle:
closed forms, library routines (numpy QR, scipy's incomplete beta and
quadrature, KS tests), published Gaussian Lloyd-Max levels and Monte Carlo."""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special, stats


def test_uniform_and_normal_streams(O):
    u = O.uniforms(123, 200_000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    z = O.normals(7, 200_000)
    assert abs(z.mean()) < 4 / math.sqrt(len(z))
    assert abs(z.var() - 1.0) < 0.02
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # Box-Muller pairs are independent: no correlation between neighbours
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 0.01
    # different seeds give different streams; same seed is reproducible
    assert not np.array_equal(O.normals(7, 16), O.normals(8, 16))
    assert np.array_equal(O.normals(7, 16), z[:16])


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_orthogonal_and_norm_preserving(O, d):
    pi = O.rotation(d, 5)
    assert np.abs(pi.T @ pi - np.eye(d)).max() <= 1e-12
    assert abs(abs(np.linalg.det(pi)) - 1.0) < 1e-10
    # fp32 table, fp32 arithmetic: |Pi x| / |x| - 1 within 1e-6
    pi32 = pi.astype(np.float32)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((1000, d)).astype(np.float32)
    ratio = np.linalg.norm(x @ pi32.T, axis=1) / np.linalg.norm(x, axis=1)
    assert np.abs(ratio - 1.0).max() <= 1e-6


@pytest.mark.parametrize("d,seed", [(64, 0), (128, 3)])
def test_rotation_equals_library_qr(O, d, seed):
    """Pi = Q diag(sign R_ii) of the Gaussian matrix from stream 2*seed; the
    sign-fixed Q factor is unique, so LAPACK's QR must give the same matrix."""
    g = O.normals(2 * seed, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    ref = q * np.sign(np.diag(r))[None, :]
    assert np.abs(O.rotation(d, seed) - ref).max() <= 1e-12


def test_rotation_entries_look_haar(O):
    # entries of a Haar matrix scaled by sqrt(d) are close to N(0, 1)
    vals = np.concatenate([O.rotation(64, s).ravel() * 8.0 for s in range(8)])
    assert abs(vals.mean()) < 0.02
    assert abs(vals.var() - 1.0) < 0.03


def test_qjl_matrix_stream_and_rounding(O):
    m, d, seed = 64, 64, 9
    s = O.qjl_matrix(m, d, seed)
    raw = O.normals(2 * seed + 1, m * d).reshape(m, d)
    assert np.array_equal(s, raw.astype(np.float16).astype(np.float64))
    assert stats.kstest(s.ravel(), "norm").pvalue > 1e-4


@pytest.mark.parametrize("d", [16, 64, 128, 300])
def test_codebook_one_bit_closed_form(O, d):
    """1 bit: the centroid is E[X | X > 0] = Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2))."""
    c, t, mse, it = O.lloyd_max(d, 1)
    exact = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    assert abs(c[0] - exact) <= 1e-13
    assert abs(mse - (1.0 / d - exact ** 2)) <= 1e-13


def _max_gaussian_levels():
    """Lloyd-Max levels for the standard normal (J. Max, IRE Trans. IT-6, 1960)."""
    path = os.path.join(os.path.dirname(__file__), "golden", "gaussian_lloyd_max_levels.txt")
    out = {}
    for line in open(path):
        if line.startswith("bits="):
            head, *vals = line.split()
            out[int(head[5:])] = [float(v) for v in vals]
    return out


MAX_GAUSSIAN = _max_gaussian_levels()


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codebook_gaussian_limit(O, bits):
    """sqrt(d) X tends to N(0,1), so sqrt(d) c tends to Max's Gaussian levels."""
    d = 20_000
    c, t, mse, it = O.lloyd_max(d, bits, max_iter=20_000)
    assert np.abs(np.sqrt(d) * c - np.array(MAX_GAUSSIAN[bits])).max() < 2e-3


@pytest.mark.parametrize("d", [64, 128])
def test_codebook_structure(O, d):
    mses = []
    for bits in (1, 2, 3, 4):
        c, t, mse, it = O.lloyd_max(d, bits)
        assert it < 100000
        assert np.all(np.diff(c) > 0) and c[0] > 0 and c[-1] < 1
        assert np.allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=0)
        # centroid condition against library quadrature of x f(x) and f(x)
        edges = np.concatenate([[0.0], t, [1.0]])
        cd = math.exp(math.lgamma(d / 2) - math.lgamma((d - 1) / 2)) / math.sqrt(math.pi)
        f = lambda x: cd * (1 - x * x) ** ((d - 3) / 2)
        for k in range(len(c)):
            a, b = edges[k], edges[k + 1]
            num = integrate.quad(lambda x: x * f(x), a, b, epsabs=1e-16, epsrel=1e-13)[0]
            den = integrate.quad(f, a, b, epsabs=1e-16, epsrel=1e-13)[0]
            assert abs(c[k] - num / den) <= 1e-11 * max(1.0, c[k])
        mses.append(mse)
    assert all(b < a for a, b in zip(mses, mses[1:]))


@pytest.mark.parametrize("d", [64, 128])
def test_sphere_mass_matches_incomplete_beta(O, d):
    """X^2 ~ Beta(1/2, (d-1)/2) for a coordinate of a uniform unit vector."""
    for a, b in [(0.0, 0.05), (0.05, 0.2), (0.1, 1.0), (0.0, 1.0), (0.3, 0.31)]:
        ref = 0.5 * (special.betainc(0.5, (d - 1) / 2, b * b) - special.betainc(0.5, (d - 1) / 2, a * a))
        assert abs(O.sphere_mass(d, a, b) - ref) <= 1e-13
    assert abs(O.sphere_mass(d, -1.0, 1.0) - 1.0) <= 1e-12


@pytest.mark.parametrize("bits", [2, 4])
def test_codebook_monte_carlo(O, bits):
    """Cell means and distortion of uniform points on the sphere (d=64)."""
    d = 64
    c, t, mse, _ = O.lloyd_max(d, bits)
    rng = np.random.default_rng(11)
    g = rng.standard_normal((40_000, d))
    x = (g / np.linalg.norm(g, axis=1, keepdims=True)).ravel()
    ax = np.abs(x)
    idx = np.searchsorted(t, ax, side="right")
    for k in range(len(c)):
        sel = ax[idx == k]
        se = sel.std() / math.sqrt(len(sel))
        assert abs(sel.mean() - c[k]) < 5 * se
    err = (ax - c[idx]) ** 2
    assert abs(err.mean() - mse) < 5 * err.std() / math.sqrt(len(err))
