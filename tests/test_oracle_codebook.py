"""Pins of the oracle's Lloyd-Max codebooks and distortion: closed forms (d = 3 is uniform, the
1-bit Gaussian quantizer), Max's Gaussian table (the large-d limit), numerical quadrature of the
density written from its Gamma-function normaliser, Monte Carlo on uniform unit vectors, and the
rate-distortion bounds the pages quote."""
import json
import math
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle import tq_oracle as o
from _tqh import sphere_codebook

STORED = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "sphere_codebooks_b7_b8.json")))

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_d3_is_uniform_quantizer(bits):
    # On S^2 one coordinate is uniform on [-1, 1] (Archimedes), so Lloyd-Max is the uniform quantizer.
    c = o.sphere_codebook(3, bits)
    k = 1 << bits
    expect = -1.0 + (2.0 * np.arange(k) + 1.0) / k
    assert np.max(np.abs(c - expect)) < 1e-12
    w = 2.0 / k
    assert abs(o.sphere_distortion(3, c) - 3.0 * w * w / 12.0) < 1e-12


def test_gaussian_one_bit_closed_form():
    c, _ = o.lloyd_max(o.GaussianMarginal(), 1)
    assert abs(c[1] - math.sqrt(2.0 / math.pi)) < 1e-14
    assert abs(o.distortion(o.GaussianMarginal(), c) - (1.0 - 2.0 / math.pi)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_gaussian_levels_match_max_table(bits):
    ref = GOLDEN["gaussian_lloyd_max"]
    c, _ = o.lloyd_max(o.GaussianMarginal(), bits)
    pos = c[len(c) // 2:]
    printed = np.array(ref["levels_positive"][str(bits)])
    # printed to four significant digits
    assert np.all(np.abs(pos - printed) <= 5e-4 * np.maximum(1.0, printed))
    mse = o.distortion(o.GaussianMarginal(), c)
    assert abs(mse - ref["mse"][str(bits)]) <= 1e-3 * ref["mse"][str(bits)]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_large_d_limit_is_gaussian(bits):
    d = 1 << 16
    c = o.sphere_codebook(d, bits) * math.sqrt(d)
    g, _ = o.lloyd_max(o.GaussianMarginal(), bits)
    assert np.max(np.abs(c - g)) < 1e-3


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_codebook_invariants_and_bounds(d, bits):
    c = sphere_codebook(d, bits)
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(c, -c[::-1])
    dist = o.SphereMarginal(d)
    D = o.sphere_distortion(d, c)
    # centroid condition => D = 1 - d * sum_i c_i^2 P_i   (E x^2 = 1/d)
    t = np.concatenate(([0.0], 0.5 * (c[len(c) // 2:][:-1] + c[len(c) // 2:][1:]), [1.0]))
    p = dist.mass(t[:-1], t[1:])
    alt = 1.0 - d * 2.0 * np.sum(c[len(c) // 2:] ** 2 * p)
    assert abs(D - alt) < 1e-10
    lo, hi = o.distortion_bounds(bits)
    assert lo <= D <= hi


def test_bound_factor_is_the_pages_2_7():
    _, hi = o.distortion_bounds(1)
    lo, _ = o.distortion_bounds(1)
    assert round(hi / lo, 1) == GOLDEN["bound_constant_factor"]["value"]


@pytest.mark.parametrize("d,bits", [(8, 2), (64, 3), (128, 4), (256, 1)])
def test_distortion_by_quadrature_of_gamma_form_density(d, bits):
    # density written independently: Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2)
    lognorm = special.gammaln(d / 2.0) - 0.5 * math.log(math.pi) - special.gammaln((d - 1) / 2.0)

    def f(x):
        return math.exp(lognorm + (d - 3) / 2.0 * math.log1p(-x * x))

    c = o.sphere_codebook(d, bits)
    t = np.concatenate(([-1.0], o.boundaries_of(c), [1.0]))
    total = 0.0
    mass = 0.0
    for i, ci in enumerate(c):
        total += integrate.quad(lambda x: (x - ci) ** 2 * f(x), t[i], t[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)[0]
        mass += integrate.quad(f, t[i], t[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)[0]
        # centroid condition checked by quadrature too
        m1 = integrate.quad(lambda x: x * f(x), t[i], t[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)[0]
        m0 = integrate.quad(f, t[i], t[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)[0]
        assert abs(m1 / m0 - ci) < 1e-9 * max(1.0, abs(ci) * math.sqrt(d))
    assert abs(mass - 1.0) < 1e-9
    assert abs(d * total - o.sphere_distortion(d, c)) < 1e-9 * o.sphere_distortion(d, c)


@pytest.mark.parametrize("d", [8, 128])
def test_sphere_marginal_matches_uniform_unit_vectors(d):
    # Kolmogorov-Smirnov against coordinates of normalised Gaussian vectors (uniform on S^(d-1)).
    rng = np.random.default_rng(5)
    n = 40000
    v = rng.standard_normal((n, d))
    x = np.sort(v[:, 0] / np.linalg.norm(v, axis=1))
    cdf = o.SphereMarginal(d).cdf(x)
    ks = np.max(np.maximum(np.arange(1, n + 1) / n - cdf, cdf - np.arange(n) / n))
    assert ks < 1.95 / math.sqrt(n)      # 0.1% critical value


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_monte_carlo_distortion_of_unit_vectors(bits):
    # E ||y - Q(y)||^2 over uniform unit vectors y in R^128 equals D(b, 128).
    d, n = 128, 20000
    rng = np.random.default_rng(100 + bits)
    v = rng.standard_normal((n, d))
    y = v / np.linalg.norm(v, axis=1, keepdims=True)
    c = sphere_codebook(d, bits)
    q = c[o.nearest_index(y, o.boundaries_of(c))]
    err = np.sum((y - q) ** 2, axis=1)
    D = o.sphere_distortion(d, c)
    assert abs(err.mean() - D) < 4.0 * err.std() / math.sqrt(n)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_operational_codebook(d, bits):
    c = sphere_codebook(d, bits)
    c_op, t = o.operational_codebook(d, bits, levels=c)
    assert np.array_equal(c_op, c.astype(np.float16).astype(np.float64))
    assert np.array_equal(t.astype(np.float32).astype(np.float64), t)
    d_star = o.sphere_distortion(d, c)
    d_op = o.sphere_distortion(d, c_op, t)
    # fp16 rounding moves D only at second order
    assert 0.0 <= d_op - d_star < 1e-3 * d_star


@pytest.mark.parametrize("key", sorted(STORED["codebooks"]))
def test_stored_high_width_codebooks_are_fixed_points_of_the_lloyd_step(key):
    # the 7- and 8-bit levels the tests read: ascending, symmetric, and each level the conditional mean of its
    # nearest-neighbour cell under the sphere marginal (one step of the oracle's own iteration moves none of them)
    d, bits = (int(v) for v in key.split("/"))
    c = np.array([float.fromhex(h) for h in STORED["codebooks"][key]])
    assert len(c) == 1 << bits and np.all(np.diff(c) > 0) and np.array_equal(c, -c[::-1])
    dist = o.SphereMarginal(d)
    pos = c[len(c) // 2:]
    t = np.concatenate(([0.0], 0.5 * (pos[:-1] + pos[1:]), [1.0]))
    g = dist.first_moment(t[:-1], t[1:]) / dist.mass(t[:-1], t[1:])
    assert np.max(np.abs(g - pos)) <= 1e-13 * pos[-1]
    lo, hi = o.distortion_bounds(bits)
    assert lo <= o.sphere_distortion(d, c) <= hi


def test_a_stored_codebook_is_the_oracles_own():
    # the file is the oracle's output: recompute one of its entries (d = 64, 7 bits, about 15 s) and compare
    c = np.array([float.fromhex(h) for h in STORED["codebooks"]["64/7"]])
    assert np.array_equal(o.sphere_codebook(64, 7), c)


@pytest.mark.parametrize("bits", [5, 6, 7, 8])
def test_high_width_distortion_approaches_the_gaussian_limit(bits):
    # D(b, d) grows with d toward the Gaussian quantizer's distortion (d -> infinity); the ordering holds at
    # every width and the d = 256 value is within a few percent of the limit
    g, _ = o.lloyd_max(o.GaussianMarginal(), bits) if bits <= 6 else (None, None)
    ds = [o.sphere_distortion(d, sphere_codebook(d, bits)) for d in (64, 128, 256)]
    assert ds[0] < ds[1] < ds[2]
    if g is not None:
        dg = o.distortion(o.GaussianMarginal(), g)
        assert ds[2] < dg < ds[2] * 1.03
