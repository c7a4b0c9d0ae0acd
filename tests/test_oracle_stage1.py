"""Pins of the oracle's stage-1 variants: PolarQuant (recursive polar
transform with quantised angles) and MSE-only b-bit codes.

- The exact transform inverts to the input (fp64) and its radius is |x|.
- Angle codebooks: symmetric about pi/4 (the density sin^(k-1)(2 phi) is),
  the two-level codebook for k = 2 in closed form (boundary pi/4, levels
  1/2 and pi/2 - 1/2), the centroid condition against scipy quadrature, and
  the angle density itself against block radii of Gaussian vectors (KS).
- The encoder's fp32 tangent comparisons pick the same bins as the nearest
  centroid of the exact fp64 angles, away from bin boundaries, and the bit
  layout decodes back to those centroids.
- MSE-only packing against a hand-worked bit pattern; MSE distortion equals
  d times the codebook's per-coordinate MSE.
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats


def test_exact_transform_inverts(O):
    rng = np.random.default_rng(0)
    for d in (8, 64, 128):
        x = rng.standard_normal(d)
        r, ang = O.polar_transform(x)
        assert abs(r - np.linalg.norm(x)) <= 1e-12 * r
        assert np.abs(O.polar_inverse(r, ang) - x).max() <= 1e-12 * r
        assert np.all(ang[: d // 2] >= 0) and np.all(ang[: d // 2] < 2 * math.pi)
        assert np.all(ang[d // 2:] >= 0) and np.all(ang[d // 2:] <= math.pi / 2)


def test_angle_codebook_closed_form_and_symmetry(O):
    c, t, _ = O.angle_lloyd_max(2, 1)
    assert abs(t[0] - math.pi / 4) < 1e-14
    assert abs(c[0] - 0.5) < 1e-13 and abs(c[1] - (math.pi / 2 - 0.5)) < 1e-13
    for k in (2, 4, 16, 64):
        for bits in (1, 2, 3):
            c, t, _ = O.angle_lloyd_max(k, bits)
            assert np.abs(c + c[::-1] - math.pi / 2).max() < 1e-12
            f = lambda x: math.sin(2 * x) ** (k - 1)
            edges = np.concatenate([[0.0], t, [math.pi / 2]])
            for j in range(len(c)):
                m0 = integrate.quad(f, edges[j], edges[j + 1], epsabs=0, epsrel=1e-13)[0]
                m1 = integrate.quad(lambda x: x * f(x), edges[j], edges[j + 1], epsabs=0,
                                    epsrel=1e-13)[0]
                assert abs(m1 / m0 - c[j]) < 1e-10


@pytest.mark.parametrize("k", [2, 8, 32])
def test_angle_density_matches_gaussian_blocks(O, k):
    rng = np.random.default_rng(k)
    g = rng.standard_normal((20000, 2, k))
    r = np.linalg.norm(g, axis=2)
    phi = np.arctan2(r[:, 1], r[:, 0])
    # cos^2 phi ~ Beta(k/2, k/2)
    p = stats.kstest(np.cos(phi) ** 2, stats.beta(k / 2, k / 2).cdf).pvalue
    assert p > 1e-3


@pytest.mark.parametrize("d,b1,b2", [(64, 4, 2), (128, 4, 2), (128, 3, 3)])
def test_encoder_bins_and_layout(O, d, b1, b2):
    rng = np.random.default_rng(d + b1)
    x = rng.standard_normal((300, d)).astype(np.float32)
    x[0, :4] = 0.0  # zero pairs
    x[1, 0], x[1, 1] = 0.0, 1.5  # on the axes
    x[1, 2], x[1, 3] = -2.0, 0.0
    codes, rad = O.polar_encode(x, b1, b2)
    assert codes.shape[1] == O.polar_code_bytes(d, b1, b2) == -(-(b1 * d // 2 + b2 * (d // 2 - 1)) // 8)
    M = 1 << b1
    nl = int(math.log2(d)) - 1
    books = [O.angle_lloyd_max(1 << (l + 1), b2)[:2] for l in range(nl)]
    xhat = O.polar_decode(codes, rad, d, b1, b2)
    near_any = 0
    for n in range(x.shape[0]):
        r, ang = O.polar_transform(x[n].astype(np.float64))
        assert abs(O.f16_value(int(rad[n])) - O.round_f16(r)) <= 2e-3 * r  # fp32 tree vs fp64
        # expected bins from the exact angles; skip angles within 1e-5 of a boundary
        want1 = np.floor(ang[: d // 2] / (2 * math.pi / M)).astype(int) % M
        edge1 = np.abs(ang[: d // 2] / (2 * math.pi / M) - np.round(ang[: d // 2] / (2 * math.pi / M)))
        rows = []
        off = d // 2
        cnt = d // 2
        for l in range(nl):
            cnt //= 2
            a = ang[off:off + cnt]
            c, t = books[l]
            wl = np.searchsorted(t, a, side="right")
            el = np.min(np.abs(a[:, None] - t[None, :]), axis=1) if len(t) else np.full(cnt, 1.0)
            rows.append((wl, el))
            off += cnt
        # decode the stored bins from the bit stream
        bits = np.unpackbits(codes[n], bitorder="little")
        got1 = np.array([int(sum(bits[b1 * i + k] << k for k in range(b1))) for i in range(d // 2)])
        ok1 = edge1 > 1e-5 / (2 * math.pi / M)
        zero = (x[n, 0::2] == 0) & (x[n, 1::2] == 0)
        assert np.array_equal(got1[ok1 & ~zero], want1[ok1 & ~zero])
        assert np.all(got1[zero] == 0)
        pos = b1 * (d // 2)
        for (wl, el) in rows:
            gl = np.array([int(sum(bits[pos + b2 * i + k] << k for k in range(b2)))
                           for i in range(len(wl))])
            ok = el > 1e-5
            assert np.array_equal(gl[ok], wl[ok])
            near_any += int((~ok).sum())
            pos += b2 * len(wl)
        # reconstruction = inverse transform of the decoded centroids, fp16 radius
        cent = [(got1 + 0.5) * 2 * math.pi / M]
        pos = b1 * (d // 2)
        for l, (wl, _) in enumerate(rows):
            gl = np.array([int(sum(bits[pos + b2 * i + k] << k for k in range(b2)))
                           for i in range(len(wl))])
            cent.append(books[l][0][gl])
            pos += b2 * len(wl)
        ref = O.polar_inverse(O.f16_value(int(rad[n])), np.concatenate(cent))
        assert np.abs(xhat[n] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    assert near_any < 0.01 * x.shape[0] * d


def test_mse_pack_hand_worked():
    import oracle
    sign = np.array([[0, 1, 1, 0]])
    mag = np.array([[1, 1, 3, 0]])  # codes 1, 5, 7, 0 at b = 3
    out = oracle.mse_pack(sign, mag, 3)
    # bits: 1 -> 0..2, 5 -> 3..5, 7 -> 6..8, 0 -> 9..11
    assert out.tolist() == [[1 | (5 << 3) | ((7 << 6) & 0xFF), 7 >> 2]]
    s2, m2 = oracle.mse_unpack(out, 4, 3)
    assert np.array_equal(s2, sign) and np.array_equal(m2, mag)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_distortion_matches_codebook(O, bits):
    d = 128
    P = O.Params(d, seed=0)
    rng = np.random.default_rng(bits)
    g = rng.standard_normal((4000, d))
    x = g / np.linalg.norm(g, axis=1, keepdims=True)  # uniform on the sphere
    packed, n, cpos = O.mse_encode(P, x, bits)
    xhat = O.mse_decode(packed, n, cpos, d, bits)
    rel = np.mean(np.sum((xhat - x) ** 2, axis=1))
    _, _, mse, _ = O.lloyd_max(d, bits)
    assert abs(rel - d * mse) < 0.05 * d * mse
