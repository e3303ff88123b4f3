"""Pins of the oracle's random numbers and rotation against facts that do not come from the oracle:
SplitMix64's published outputs, the moments of a normal law, the definition of a QR factorisation
with positive R diagonal (and LAPACK's QR), and the Haar law of the first column."""
import math

import numpy as np
import pytest

from oracle import tq_oracle as o


def test_splitmix64_reference_outputs():
    # First three outputs of Vigna's reference splitmix64.c with the state seeded to 0.
    assert [int(v) for v in o.splitmix64(0, 3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_splitmix64_counter_form():
    # Output k of a stream is output 0 of the stream whose seed is advanced by k increments.
    seed = 123456789
    a = o.splitmix64(seed, 10)
    for k in range(10):
        b = o.splitmix64((seed + k * 0x9E3779B97F4A7C15) % 2 ** 64, 1)
        assert int(a[k]) == int(b[0])
    assert np.array_equal(o.splitmix64(seed, 5, start=5), a[5:])


def test_box_muller_moments():
    n = 1 << 20
    g = o.gaussian_stream(7, n)
    se = 1.0 / math.sqrt(n)
    assert abs(g.mean()) < 5 * se
    assert abs(g.var() - 1.0) < 5 * math.sqrt(2.0) * se
    assert abs(np.mean(g ** 4) - 3.0) < 5 * math.sqrt(96.0) * se
    # P(|Z| < 1) = erf(1/sqrt 2)
    p1 = math.erf(1.0 / math.sqrt(2.0))
    assert abs(np.mean(np.abs(g) < 1.0) - p1) < 5 * math.sqrt(p1 * (1 - p1)) * se
    # the two members of a pair are uncorrelated
    assert abs(np.mean(g[0::2] * g[1::2])) < 5 * math.sqrt(2.0) * se


@pytest.mark.parametrize("d", [3, 8, 64, 128, 256])
def test_rotation_is_qr_factor_with_positive_diagonal(d):
    seed = 11
    pi = o.haar_rotation(d, seed)
    g = o.gaussian_stream(seed, d * d).reshape(d, d)
    assert np.max(np.abs(pi.T @ pi - np.eye(d))) < 1e-12
    assert abs(abs(np.linalg.det(pi)) - 1.0) < 1e-10
    r = pi.T @ g
    assert np.max(np.abs(np.tril(r, -1))) < 1e-10 * np.max(np.abs(r))
    assert np.all(np.diag(r) > 0)
    # LAPACK's Householder QR with the page's sign fix gives the same matrix
    q, rr = np.linalg.qr(g)
    s = np.sign(np.diag(rr))
    s[s == 0] = 1.0
    assert np.max(np.abs(q * s[None, :] - pi)) < 1e-10


def test_rotation_first_column_is_haar():
    # Under the Haar law, Pi[0, 0] is one coordinate of a uniform unit vector: mean 0, variance 1/d.
    # A QR without the sign fix would give a mean near -sqrt(2/pi)/sqrt(d) * sqrt(d) ~ -0.8 here.
    d, seeds = 8, 2000
    v = np.array([o.haar_rotation(d, s)[0, 0] for s in range(seeds)]) * math.sqrt(d)
    se = 1.0 / math.sqrt(seeds)
    assert abs(v.mean()) < 5 * se
    # variance of sqrt(d) x under f_d is exactly 1
    assert abs(v.var() - 1.0) < 0.25


@pytest.mark.parametrize("d", [64, 128, 256])
def test_operational_rotation_deviation(d):
    pi = o.haar_rotation(d, 0)
    op = o.operational_rotation(d, 0)
    # every entry is the nearest fp16 value
    assert np.array_equal(op, pi.astype(np.float16).astype(np.float64))
    # entries are O(1/sqrt d); fp16 relative rounding is 2^-11, so Pi_op^T Pi_op stays within 2e-3 of I
    assert np.max(np.abs(op.T @ op - np.eye(d))) < 2e-3
    assert np.max(np.abs(op - pi)) <= 2.0 ** -11 * np.max(np.abs(pi))


# ---- randomized Walsh-Hadamard rotation ("turbo-attn", The codec, "Hadamard rotation")

@pytest.mark.parametrize("d", [2, 4, 64, 128, 256])
def test_sylvester_hadamard_is_the_library_hadamard(d):
    from scipy import linalg
    assert np.array_equal(o.sylvester_hadamard(d), linalg.hadamard(d).astype(np.float64))


def _fwht(v: np.ndarray) -> np.ndarray:
    """Fast Walsh-Hadamard transform by butterflies (pairs (a + b, a - b) at strides 1, 2, 4, ...), the
    O(d log d) algorithm, independent of the matrix construction."""
    v = np.array(v, dtype=np.float64)
    h = 1
    while h < v.shape[-1]:
        a = v.reshape(*v.shape[:-1], -1, 2, h)
        v = np.concatenate([a[..., 0, :] + a[..., 1, :], a[..., 0, :] - a[..., 1, :]], axis=-1).reshape(v.shape)
        h *= 2
    return v


@pytest.mark.parametrize("d", [64, 128, 256])
def test_hadamard_rotation_is_orthogonal_and_is_the_fast_transform(d):
    pi = o.hadamard_rotation(d, 5)
    assert np.abs(pi @ pi.T - np.eye(d)).max() < 1e-14
    x = np.random.default_rng(0).standard_normal((16, d))
    s = o.hadamard_signs(d, 5)
    assert np.abs(x @ pi.T - _fwht(x * s) / math.sqrt(d)).max() < 1e-12
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(int((s < 0).sum()) - d / 2) < 4 * math.sqrt(d)     # fair signs
    assert not np.array_equal(s, o.hadamard_signs(d, 6))


@pytest.mark.parametrize("bits", [2, 3])
def test_hadamard_rotation_keeps_the_codebook_distortion(bits):
    # an orthogonal map sends an isotropic Gaussian to an isotropic Gaussian, so the rotated unit vector is
    # uniform on the sphere and the measured distortion is the codebook's D(b, d)
    d, n = 128, 20000
    pi = o.operational_rotation(d, 9, "hadamard")
    c, t = o.operational_codebook(d, bits)
    x = o.to_fp16_values(np.random.default_rng(bits).standard_normal((n, d)))
    idx, nrm, y = o.encode_k(x, pi, t)
    measured = float(np.mean(np.sum((y - c[idx]) ** 2, axis=1)))
    assert abs(measured - o.sphere_distortion(d, c, t)) <= 0.02 * o.sphere_distortion(d, c, t)
