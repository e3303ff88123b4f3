"""Oracle for TurboQuant-style KV-cache compression -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct CPU restatement (numpy, fp64 unless a page fixes the precision)
of what the hot path computes.  It exists to check the CUDA library, not to serve it: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg may import
or call anything in this package.  The product path (the C-ABI library ``libtq`` and its Python
binding) never imports, links or executes it, and this module imports nothing from the product.

Pages this follows (cited by page title and section throughout):

* [P1] "aitherkvcache" -- the ``TurboQuant`` encode/decode call: fp16 vectors of head_dim 128 become
  64 uint8 codes (4 bits) plus one f32 norm per vector.
* [P2] "TurboQuant: A KV Cache Compression Technique ..." -- Haar rotation, data-independent
  Lloyd-Max codebooks, norm separation, distortion within a ~2.7x factor of the bound.
* [P3] "KV Cache API" (TurboQuant docs) -- ``compressors.py`` (``MSECompressor`` and
  ``TurboQuantCompressorMSE``: rotation construction, compress, decompress), ``values.py``
  (``quantize_values``, ``dequantize_values``, ``value_formula_nbytes``) and ``store.py``
  (``TurboQuantKVCache.attention_scores`` / ``attend``; the older ``quantize_value_chunk``).
* [P4] "turbo-attn" (PyPI) -- the ``TkvCodec`` demo (3.88x vs bf16, relative error 0.10) and the
  rotated-query scoring of its split-K decode kernel.
* [P5] "turboquant-pytorch" -- rotation makes every coordinate follow one predictable bell curve;
  quantize = normalise, rotate, round to the nearest centroid, store indices + norm.

Readings taken where the pages are silent or disagree are listed in the repository's design notes
and repeated beside the function that takes them.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special

# ----------------------------------------------------------------------------------------------
# Counter-based random numbers for the rotation (the pages draw G with torch's CPU generator,
# whose stream cannot and need not be reproduced; this build fixes SplitMix64 + Box-Muller, both
# published definitions, and the library implements the same two from the same definitions).
# ----------------------------------------------------------------------------------------------

_U64 = np.uint64
_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB


def splitmix64(seed: int, count: int, start: int = 0) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of SplitMix64 seeded with ``seed``.

    Definition (Steele, Lea & Flood, "Fast splittable pseudorandom number generators", 2014; the
    reference C by S. Vigna): the state advances by the golden-ratio increment and each output
    is the state passed through the two xor-shift-multiply rounds below.
    """
    i = np.arange(start + 1, start + count + 1, dtype=_U64)
    z = _U64(seed & 0xFFFFFFFFFFFFFFFF) + i * _U64(_GOLDEN)
    z = (z ^ (z >> _U64(30))) * _U64(_MIX1)
    z = (z ^ (z >> _U64(27))) * _U64(_MIX2)
    return z ^ (z >> _U64(31))


def gaussian_stream(seed: int, count: int) -> np.ndarray:
    """``count`` standard normal draws: Box-Muller (1958) on consecutive SplitMix64 pairs.

    Pair p uses outputs 2p and 2p+1: u1 = (top 53 bits + 1/2) * 2^-53 in (0, 1),
    u2 = top 53 bits * 2^-53 in [0, 1); r = sqrt(-2 ln u1); draws 2p, 2p+1 = r cos(2 pi u2),
    r sin(2 pi u2).
    """
    pairs = (count + 1) // 2
    z = splitmix64(seed, 2 * pairs)
    top = (z >> _U64(11)).astype(np.float64)
    u1 = (top[0::2] + 0.5) * 2.0 ** -53
    u2 = top[1::2] * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * math.pi * u2)
    out[1::2] = r * np.sin(2.0 * math.pi * u2)
    return out[:count]


# ----------------------------------------------------------------------------------------------
# Rotation  ([P3] compressors.py, MSECompressor.__init__: G = randn(d, d); Q, R = qr(G);
# Pi = Q * sign(diag R) with zero signs set to +1.  [P2] "Random Orthogonal Rotation": a
# Haar-distributed orthogonal matrix.)
# ----------------------------------------------------------------------------------------------


def haar_rotation(d: int, seed: int) -> np.ndarray:
    """The seeded Haar rotation Pi (d x d, fp64): rotated = Pi @ x.

    G[i][j] is Gaussian draw i*d + j.  Pi is the Q factor of the QR factorisation of G whose R has
    a positive diagonal -- exactly what the page's ``Q * sign(diag R)`` produces.  Q is formed by
    classical Gram-Schmidt over the columns of G, each column orthogonalised twice against the
    previous ones (re-orthogonalisation keeps Q orthogonal to ~1e-15); the norm taken as R_jj is
    positive, so no sign fix is needed afterwards.
    """
    g = gaussian_stream(seed, d * d).reshape(d, d)
    q = np.zeros((d, d), dtype=np.float64)
    for j in range(d):
        v = g[:, j].copy()
        for _ in range(2):
            v -= q[:, :j] @ (q[:, :j].T @ v)
        q[:, j] = v / np.linalg.norm(v)
    return q


def to_fp16_values(a: np.ndarray) -> np.ndarray:
    """Round to the nearest fp16 (ties to even) and return the values as fp64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def sylvester_hadamard(d: int) -> np.ndarray:
    """The d x d Walsh-Hadamard matrix of +-1 entries (d a power of two) by Sylvester's doubling:
    H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    if d < 1 or d & (d - 1):
        raise ValueError(f"d={d} is not a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_signs(d: int, seed: int) -> np.ndarray:
    """Seeded signs s_j = -1 if the top bit of SplitMix64(seed) output j is set, else +1."""
    top = (splitmix64(seed, d) >> _U64(63)).astype(np.int64)
    return 1.0 - 2.0 * top


def hadamard_rotation(d: int, seed: int) -> np.ndarray:
    """The randomized Walsh-Hadamard rotation Pi = H diag(s) / sqrt(d) (d x d, fp64): rotated = Pi @ x.

    [P4] "turbo-attn", The codec, "Hadamard rotation": a Walsh-Hadamard transform spreads outlier channels
    over the vector, and queries are rotated the same way.  Reading: the page fixes neither the signs nor
    the scale; this build takes the usual randomized, orthonormal form -- seeded signs (so the coordinates
    of a rotated isotropic vector follow the same marginal and the same data-independent codebook
    applies) and 1/sqrt(d) (so Pi is orthogonal and norms are kept).
    """
    return sylvester_hadamard(d) * hadamard_signs(d, seed)[None, :] / math.sqrt(d)


ROTATIONS = ("haar", "hadamard")


def operational_rotation(d: int, seed: int, kind: str = "haar") -> np.ndarray:
    """Pi_op = fp16(Pi): the rotation the tensor-core path multiplies by (values as fp64).

    Reading: the pages keep Pi in fp32; this build rounds it once to fp16 so that fp16 inputs times
    Pi_op are exact products in an fp32 accumulator, and states the deviation separately.
    """
    if kind == "haar":
        return to_fp16_values(haar_rotation(d, seed))
    if kind == "hadamard":
        return to_fp16_values(hadamard_rotation(d, seed))
    raise ValueError(f"unknown rotation {kind!r}")


# ----------------------------------------------------------------------------------------------
# Codebook  ([P3] compressors.py calls ``_solve_codebook(head_dim, bits)``, whose body is not on the
# page; [P2] "Lloyd-Max Scalar Quantization": optimal codebooks pre-computed from a mathematical
# derivation, data-independent; [P5] "How It Works": after the rotation every coordinate follows a
# predictable bell-curve distribution.)
#
# Reading: the distribution is the exact marginal of one coordinate of a uniform point on the unit
# sphere S^(d-1) (which a Haar-rotated unit vector is):
#     f_d(x) = (1 - x^2)^a / B(1/2, a + 1),  a = (d - 3) / 2,  x in [-1, 1].
# Its cell masses and moments are regularised incomplete beta functions, so each Lloyd step below
# is exact up to the library's betainc.
# ----------------------------------------------------------------------------------------------


class SphereMarginal:
    """Masses and moments of f_d over intervals [lo, hi] of [0, 1] (the density is even)."""

    def __init__(self, d: int):
        if d < 2:
            raise ValueError("d must be >= 2")
        self.d = d
        self.a = (d - 3) / 2.0
        self.log_b0 = special.betaln(0.5, self.a + 1.0)          # normaliser B(1/2, a+1)
        self.ratio2 = math.exp(special.betaln(1.5, self.a + 1.0) - self.log_b0)   # = 1/d

    def mass(self, lo, hi):
        """P(lo < x < hi) for 0 <= lo < hi <= 1: (I_{hi^2} - I_{lo^2}) / 2 with I the regularised
        incomplete beta of (1/2, a+1); the upper tail uses the complement for precision."""
        lo = np.asarray(lo, dtype=np.float64)
        hi = np.asarray(hi, dtype=np.float64)
        p, q = 0.5, self.a + 1.0
        upper = np.where(hi >= 1.0, 0.0, special.betaincc(p, q, np.minimum(hi, 1.0) ** 2))
        return 0.5 * (special.betaincc(p, q, lo * lo) - upper)

    def first_moment(self, lo, hi):
        """int_lo^hi x f(x) dx = ((1-lo^2)^(a+1) - (1-hi^2)^(a+1)) / (2 (a+1) B(1/2, a+1))."""
        lo = np.asarray(lo, dtype=np.float64)
        hi = np.asarray(hi, dtype=np.float64)
        e = self.a + 1.0
        hi_in = np.where(hi >= 1.0, 0.0, hi)          # (1 - 1^2)^(a+1) = 0 at the end of the support
        top = np.exp(e * np.log1p(-lo * lo)) - np.where(hi >= 1.0, 0.0, np.exp(e * np.log1p(-hi_in * hi_in)))
        return top / (2.0 * e * math.exp(self.log_b0))

    def second_moment(self, lo, hi):
        """int_lo^hi x^2 f(x) dx = (B(3/2, a+1) / B(1/2, a+1)) (J_{hi^2} - J_{lo^2}) / 2, J the
        regularised incomplete beta of (3/2, a+1)."""
        lo = np.asarray(lo, dtype=np.float64)
        hi = np.asarray(hi, dtype=np.float64)
        p, q = 1.5, self.a + 1.0
        upper = np.where(hi >= 1.0, 0.0, special.betaincc(p, q, np.minimum(hi, 1.0) ** 2))
        return self.ratio2 * 0.5 * (special.betaincc(p, q, lo * lo) - upper)

    def cdf(self, x):
        x = np.asarray(x, dtype=np.float64)
        return 0.5 + 0.5 * np.sign(x) * special.betainc(0.5, self.a + 1.0, np.minimum(x * x, 1.0))

    upper_end = 1.0


class GaussianMarginal:
    """Masses and moments of N(0, sigma^2) over [lo, hi] (lo >= 0); the d -> infinity limit of
    sqrt(d) * x under f_d when sigma = 1."""

    def __init__(self, sigma: float = 1.0):
        self.s = float(sigma)
        self.ratio2 = self.s ** 2

    def _phi(self, z):
        return np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)

    def mass(self, lo, hi):
        lo = np.asarray(lo, dtype=np.float64) / self.s
        hi = np.asarray(hi, dtype=np.float64) / self.s
        return special.ndtr(-lo) - np.where(np.isinf(hi), 0.0, special.ndtr(-np.where(np.isinf(hi), 0.0, hi)))

    def first_moment(self, lo, hi):
        lo = np.asarray(lo, dtype=np.float64) / self.s
        hi = np.asarray(hi, dtype=np.float64) / self.s
        return self.s * (self._phi(lo) - np.where(np.isinf(hi), 0.0, self._phi(np.where(np.isinf(hi), 0.0, hi))))

    def second_moment(self, lo, hi):
        # int z^2 phi = Phi - z phi
        lo_z = np.asarray(lo, dtype=np.float64) / self.s
        hi_z = np.asarray(hi, dtype=np.float64) / self.s
        fin = ~np.isinf(hi_z)
        hz = np.where(fin, hi_z, 0.0)
        m = self.mass(lo, hi)
        edge = lo_z * self._phi(lo_z) - np.where(fin, hz * self._phi(hz), 0.0)
        return self.s ** 2 * (m + edge)

    upper_end = math.inf


def _lloyd_positive_half(dist, levels_half: int, init: np.ndarray, tol: float, max_iter: int):
    """Lloyd-Max on the positive half of an even density.

    Levels c_1 < ... < c_L > 0 (L = 2^(b-1)); cells [t_{i-1}, t_i] with t_0 = 0, t_L = the end of the
    support and t_i = (c_i + c_{i+1}) / 2 (nearest-neighbour condition); each level is then moved to
    the conditional mean of its cell (centroid condition).  Repeat until no level moves by more
    than ``tol`` (relative to the largest level).
    """
    c = np.array(init, dtype=np.float64)
    for it in range(max_iter):
        t = np.concatenate(([0.0], 0.5 * (c[:-1] + c[1:]), [dist.upper_end]))
        new = dist.first_moment(t[:-1], t[1:]) / dist.mass(t[:-1], t[1:])
        step = np.max(np.abs(new - c))
        c = new
        if step <= tol * np.max(np.abs(c)):
            return c, it + 1
    return c, max_iter


def lloyd_max(dist, bits: int, tol: float = 1e-15, max_iter: int = 200000):
    """Symmetric 2^bits-level Lloyd-Max codebook for ``dist``: ascending levels, fp64.

    The density is even, so the optimal codebook is symmetric, c_i = -c_{2^b-1-i}, with a decision
    boundary at 0; only the positive half is iterated.  Start: the levels at the quantiles
    (i + 1/2) / L of the positive half-distribution.
    """
    if bits < 1 or bits > 8:
        raise ValueError("bits must be in [1, 8]")
    half = 1 << (bits - 1)
    # quantile initialisation by bisection on the positive-half mass
    total = dist.mass(0.0, dist.upper_end)
    init = []
    for i in range(half):
        target = (i + 0.5) / half * total
        lo, hi = 0.0, (1.0 if dist.upper_end == 1.0 else 40.0 * getattr(dist, "s", 1.0))
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if dist.mass(0.0, mid) < target:
                lo = mid
            else:
                hi = mid
        init.append(0.5 * (lo + hi))
    pos, iters = _lloyd_positive_half(dist, half, np.array(init), tol, max_iter)
    return np.concatenate((-pos[::-1], pos)), iters


def sphere_codebook(d: int, bits: int) -> np.ndarray:
    """c*: the Lloyd-Max levels of the sphere-coordinate marginal f_d at ``bits`` bits."""
    c, _ = lloyd_max(SphereMarginal(d), bits)
    return c


def boundaries_of(c: np.ndarray) -> np.ndarray:
    """Decision boundaries of a nearest-neighbour scalar quantizer: midpoints of adjacent levels."""
    c = np.asarray(c, dtype=np.float64)
    return 0.5 * (c[:-1] + c[1:])


def operational_codebook(d: int, bits: int, levels: np.ndarray | None = None):
    """(c_op, t): c_op = fp16(c*) as fp64 values; t = the midpoints of c_op, which are exact in fp32.

    Reading: the kernels compare rotated coordinates with fp32 boundaries and gather fp16 levels, so
    the operational codebook is c* rounded once to fp16; the oracle consumes the same values.
    ``levels`` may pass c* when it is already at hand (the 7- and 8-bit fixed points take minutes).
    """
    c_op = to_fp16_values(sphere_codebook(d, bits) if levels is None else np.asarray(levels, dtype=np.float64))
    t = boundaries_of(c_op)
    if not np.array_equal(t.astype(np.float32).astype(np.float64), t):
        raise AssertionError("boundary midpoints of fp16 levels are expected to be exact in fp32")
    return c_op, t


def distortion(dist, c: np.ndarray, t: np.ndarray | None = None, dim_scale: float = 1.0) -> float:
    """Mean squared error of the scalar quantizer (levels c, boundaries t) under ``dist``, times
    ``dim_scale``.  With dist = f_d and dim_scale = d this is D(b, d) = E||y - Q(y)||^2 for a unit
    vector y whose d coordinates each follow f_d -- the per-unit-vector distortion of the rotated
    quantizer.  Cell by cell: int (x - c_i)^2 f = S2_i - 2 c_i M_i + c_i^2 P_i (both halves).
    """
    c = np.asarray(c, dtype=np.float64)
    t = boundaries_of(c) if t is None else np.asarray(t, dtype=np.float64)
    end = dist.upper_end
    edges = np.concatenate(([-end], t, [end]))
    total = 0.0
    for i, ci in enumerate(c):
        lo, hi = edges[i], edges[i + 1]
        # split each cell at 0 and use evenness of the density
        parts = []
        if lo < 0.0:
            a, b = max(0.0, -hi), -lo          # mirrored to the positive half
            parts.append((a, b, -1.0))
        if hi > 0.0:
            parts.append((max(lo, 0.0), hi, 1.0))
        for a, b, sgn in parts:
            if b <= a:
                continue
            p = float(dist.mass(a, b))
            m = sgn * float(dist.first_moment(a, b))
            s2 = float(dist.second_moment(a, b))
            total += s2 - 2.0 * ci * m + ci * ci * p
    return dim_scale * total


def sphere_distortion(d: int, c: np.ndarray, t: np.ndarray | None = None) -> float:
    """D(b, d) of levels c (and boundaries t, default the midpoints) on the sphere marginal."""
    return distortion(SphereMarginal(d), c, t, dim_scale=float(d))


def distortion_bounds(bits: int):
    """The rate-distortion sandwich the pages quote: 4^-b <= D <= (sqrt(3) pi / 2) 4^-b
    ([P2] "within a ~2.7x constant factor" of the information-theoretic bound)."""
    lower = 4.0 ** (-bits)
    return lower, math.sqrt(3.0) * math.pi / 2.0 * lower


# ----------------------------------------------------------------------------------------------
# Bit packing.  Reading: one LSB-first bitstream per row for both K and V -- index j occupies bits
# [j*b, (j+1)*b) of the row read as little-endian bytes.  This is the order of [P3] store.py
# (``v0 | v1 << 2 | ...``) and gives the dense (d*b + 7) // 8 bytes of [P3] values.py for b = 3.
# ----------------------------------------------------------------------------------------------


def pack_lsb(idx: np.ndarray, bits: int) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    out = np.zeros((n, (d * bits + 7) // 8), dtype=np.uint8)
    for j in range(d):
        for k in range(bits):
            pos = j * bits + k
            out[:, pos // 8] |= (((idx[:, j] >> k) & 1) << (pos % 8)).astype(np.uint8)
    return out


def unpack_lsb(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    idx = np.zeros((n, d), dtype=np.int64)
    for j in range(d):
        for k in range(bits):
            pos = j * bits + k
            idx[:, j] |= ((packed[:, pos // 8].astype(np.int64) >> (pos % 8)) & 1) << k
    return idx


# ----------------------------------------------------------------------------------------------
# Key codec  ([P3] compressors.py, MSECompressor.compress / decompress; [P1] encode returns codes +
# f32 norms; [P5] "normalise, rotate, round each coordinate, store indices + norm".)
# ----------------------------------------------------------------------------------------------


def encode_k(x16: np.ndarray, pi_op: np.ndarray, t: np.ndarray):
    """Key encode of fp16 rows x [N][d].

    n = ||x||_2;  y = Pi_op x / (n + 1e-8)  (the page normalises then rotates; identical in exact
    arithmetic);  idx_j = #{i : t_i < y_j}, which is argmin_i |y_j - c_i| with ties to the lower
    index (the page's ``argmin``).  Returns (idx [N][d] int64, n [N] fp64, y [N][d] fp64).
    """
    x = np.asarray(x16).astype(np.float64)
    n = np.sqrt(np.sum(x * x, axis=-1))
    y = (x @ pi_op.T) / (n + 1e-8)[:, None]
    return nearest_index(y, t), n, y


def nearest_index(y: np.ndarray, t: np.ndarray) -> np.ndarray:
    """Index of the nearest level given the ascending boundaries t: #{i : t_i < y}.  A value exactly
    on a boundary goes to the lower level, as the first-occurrence ``argmin`` of the page does."""
    idx = np.zeros(np.shape(y), dtype=np.int64)
    for ti in t:
        idx += (np.asarray(y) > ti)
    return idx


def decode_k(idx: np.ndarray, norms: np.ndarray, pi_op: np.ndarray, c_op: np.ndarray) -> np.ndarray:
    """Key decode: x_hat = n * Pi_op^T c_op[idx]  (the page's ``centroids[idx] @ Pi * norm``)."""
    return np.asarray(norms, dtype=np.float64)[:, None] * (c_op[np.asarray(idx)] @ pi_op)


def k_row_bytes(d: int, bits: int) -> int:
    return (d * bits + 7) // 8


# ----------------------------------------------------------------------------------------------
# Value codec  ([P3] values.py, quantize_values / dequantize_values).  The page's fp32 operation
# sequence IS the format, so this part runs in IEEE float32, one rounding per operation, exactly
# in the page's order; fp16 metadata are round-to-nearest-even conversions.
# ----------------------------------------------------------------------------------------------

V_BITS = (2, 3, 4, 8)


def encode_v(x16: np.ndarray, bits: int, group_size: int = 32, scale_layout: str = "group"):
    """Grouped affine value quantizer.

    Per (row, group): vmin, vmax (padding lanes masked out); scale = max((vmax - vmin) / (2^b - 1),
    1e-12) in fp32; zero = vmin; q = clamp(round_half_even((x - zero) / scale), 0, 2^b - 1) using
    the fp32 scale; data = LSB-first packed q; scales, zeros stored as fp16.
    ``scale_layout="token"`` uses one group per row (group = d).
    Returns (data [N][(d_pad*b+7)//8] u8, scales [N][G] f16, zeros [N][G] f16, q [N][d_pad] int64).
    """
    if bits not in V_BITS:
        raise ValueError(f"value bits must be one of {V_BITS}")
    if scale_layout not in ("group", "token"):
        raise ValueError("scale_layout must be 'group' or 'token'")
    x = np.asarray(x16).astype(np.float32)
    n, d = x.shape
    g = d if scale_layout == "token" else group_size
    d_pad = -(-d // g) * g
    xp = np.zeros((n, d_pad), dtype=np.float32)
    xp[:, :d] = x
    valid = (np.arange(d_pad) < d).reshape(d_pad // g, g)
    grouped = xp.reshape(n, d_pad // g, g)
    vmin = np.where(valid, grouped, np.float32(np.inf)).min(axis=-1, keepdims=True)
    vmax = np.where(valid, grouped, np.float32(-np.inf)).max(axis=-1, keepdims=True)
    levels = np.float32((1 << bits) - 1)
    scales = np.maximum((vmax - vmin) / levels, np.float32(1e-12))
    zeros = vmin
    q = np.clip(np.rint((grouped - zeros) / scales), np.float32(0), levels).astype(np.int64)
    q = np.where(valid, q, 0).reshape(n, d_pad)
    data = pack_lsb(q, bits)
    return data, scales[..., 0].astype(np.float16), zeros[..., 0].astype(np.float16), q


def decode_v(data: np.ndarray, scales16: np.ndarray, zeros16: np.ndarray, bits: int, d: int,
             group_size: int = 32, scale_layout: str = "group") -> np.ndarray:
    """Value decode: q * float(scale16) + float(zero16), two fp32 operations, padding cropped.
    Returns float32 [N][d]."""
    g = d if scale_layout == "token" else group_size
    d_pad = -(-d // g) * g
    q = unpack_lsb(data, bits, d_pad).astype(np.float32)
    n = q.shape[0]
    grouped = q.reshape(n, d_pad // g, g)
    s = np.asarray(scales16).astype(np.float32)[..., None]
    z = np.asarray(zeros16).astype(np.float32)[..., None]
    out = (grouped * s) + z
    return out.reshape(n, d_pad)[:, :d]


def v_formula_nbytes(shape, bits: int, group_size: int, scale_layout: str = "group",
                     scale_dtype_bytes: int = 2, zero_dtype_bytes: int = 2) -> dict:
    """Byte counts of a value payload ([P3] values.py, value_formula_nbytes): payload
    outer * ((d_pad * b + 7) // 8), metadata outer * groups * (2 + 2)."""
    d = int(shape[-1])
    g = d if scale_layout == "token" else group_size
    d_pad = -(-d // g) * g
    outer = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    groups = d_pad // g
    return {"compressed_v_bytes": outer * ((d_pad * bits + 7) // 8),
            "scales_bytes": outer * groups * scale_dtype_bytes,
            "zeros_bytes": outer * groups * zero_dtype_bytes,
            "padded_dim": d_pad, "groups": groups}


def k_compression_ratio(d: int, bits: int, norm_bytes: int) -> float:
    """Bytes of a 16-bit vector over bytes of its code + norm."""
    return (2.0 * d) / (k_row_bytes(d, bits) + norm_bytes)


# ----------------------------------------------------------------------------------------------
# Decode-step attention over the compressed cache  ([P3] store.py, TurboQuantKVCache:
# attention_scores with scale 1/sqrt(head_dim) default, softmax by the caller, attend = weights @
# dequantised values; [P4] the decode kernel scores a rotated query against the codes.)
# Reading: GQA maps query head h_q to kv head floor(h_q / G); one query token per sequence; no mask.
# ----------------------------------------------------------------------------------------------


def attend_one(q16: np.ndarray, k_idx: np.ndarray, k_norms: np.ndarray, v_hat: np.ndarray,
               pi_op: np.ndarray, c_op: np.ndarray, scale: float):
    """Attention of one query vector over one kv head's compressed cache (T tokens).

    Path A (definition): k_hat_t = decode_k; s_t = scale * <q, k_hat_t>; p = softmax(s);
    o = sum_t p_t v_hat_t.  Path B (what the fused kernel computes): q_rot = Pi_op q,
    s_t = scale * n_t * <q_rot, c_op[idx_t]>.  Equal in exact arithmetic.
    Returns (o [d] fp64, scores_a [T], scores_b [T]).
    """
    q = np.asarray(q16).astype(np.float64)
    k_hat = decode_k(k_idx, k_norms, pi_op, c_op)
    s_a = scale * (k_hat @ q)
    q_rot = pi_op @ q
    s_b = scale * np.asarray(k_norms, dtype=np.float64) * (c_op[np.asarray(k_idx)] @ q_rot)
    m = np.max(s_a)
    p = np.exp(s_a - m)
    p /= p.sum()
    o = p @ np.asarray(v_hat, dtype=np.float64)
    return o, s_a, s_b


def attend(q16: np.ndarray, k_idx: np.ndarray, k_norms: np.ndarray, v_hat: np.ndarray,
           pi_op: np.ndarray, c_op: np.ndarray, scale: float | None = None,
           seq_lens: np.ndarray | None = None) -> np.ndarray:
    """Batched decode attention, contiguous cache.

    q16 [B][H_q][d]; k_idx [B][H_kv][T][d]; k_norms [B][H_kv][T]; v_hat [B][H_kv][T][d] (the value
    decode, fp32); optional seq_lens [B] (tokens 0..len-1 of each sequence are attended).
    Returns o [B][H_q][d] fp64.
    """
    bsz, hq, d = q16.shape
    hkv = k_idx.shape[1]
    if hq % hkv:
        raise ValueError("H_q must be a multiple of H_kv")
    grp = hq // hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((bsz, hq, d), dtype=np.float64)
    for b in range(bsz):
        tl = k_idx.shape[2] if seq_lens is None else int(seq_lens[b])
        for h in range(hq):
            kv = h // grp
            if tl == 0:
                continue
            out[b, h], _, _ = attend_one(q16[b, h], k_idx[b, kv, :tl], k_norms[b, kv, :tl],
                                         v_hat[b, kv, :tl], pi_op, c_op, scale)
    return out


def attend_window(q16: np.ndarray, k_idx: np.ndarray, k_norms: np.ndarray, v_hat: np.ndarray,
                  win_k16: np.ndarray, win_v16: np.ndarray, pi_op: np.ndarray, c_op: np.ndarray,
                  scale: float | None = None, seq_lens: np.ndarray | None = None,
                  win_lens: np.ndarray | None = None) -> np.ndarray:
    """Decode attention over the compressed cache plus a window of recent uncompressed tokens.

    [P3] store.py ``TurboQuantKVCache``: ``attention_scores`` concatenates scale * (the quantized part's
    scores) with scale * query @ key_buffer^T; the caller's softmax runs over all of them; ``attend`` adds
    the quantized part's weights times the dequantized values and the buffer's weights times the buffer's
    values, which are used as stored (fp16).  The compressed part's scores are those of ``attend_one``
    (path A, the decoded keys).

    q16 [B][H_q][d]; k_idx [B][H_kv][T][d]; k_norms [B][H_kv][T]; v_hat [B][H_kv][T][d];
    win_k16, win_v16 [B][H_kv][W][d] fp16; optional seq_lens / win_lens [B] (tokens 0..len-1 of each part).
    Returns o [B][H_q][d] fp64 (zeros where both parts are empty).
    """
    bsz, hq, d = q16.shape
    hkv = k_idx.shape[1]
    grp = hq // hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((bsz, hq, d), dtype=np.float64)
    for b in range(bsz):
        tl = k_idx.shape[2] if seq_lens is None else int(seq_lens[b])
        wl = win_k16.shape[2] if win_lens is None else int(win_lens[b])
        for h in range(hq):
            kv = h // grp
            q = np.asarray(q16[b, h]).astype(np.float64)
            k_all = np.concatenate([decode_k(k_idx[b, kv, :tl], k_norms[b, kv, :tl], pi_op, c_op),
                                    np.asarray(win_k16[b, kv, :wl]).astype(np.float64)], axis=0)
            v_all = np.concatenate([np.asarray(v_hat[b, kv, :tl], dtype=np.float64),
                                    np.asarray(win_v16[b, kv, :wl]).astype(np.float64)], axis=0)
            if k_all.shape[0] == 0:
                continue
            s = scale * (k_all @ q)
            p = np.exp(s - s.max())
            out[b, h] = (p / p.sum()) @ v_all
    return out


def paged_rows(block_table: np.ndarray, b: int, h: int, length: int, num_kv_heads: int,
               block_size: int) -> np.ndarray:
    """Pool rows of sequence b, kv head h, positions 0..length-1 in the paged layout.

    Reading (the pages name paged blocks without fixing a layout): position p lives in physical
    block block_table[b][p // block_size] at slot p % block_size, and each pool array is indexed
    by row (physical_block * H_kv + h) * block_size + slot.
    """
    p = np.arange(length)
    blocks = np.asarray(block_table)[b, p // block_size].astype(np.int64)
    return (blocks * num_kv_heads + h) * block_size + (p % block_size)


# ----------------------------------------------------------------------------------------------
# QJL residual keys  ([P3] compressors.py, TurboQuantCompressorV2: __init__, compress and
# asymmetric_attention_scores; store.py TurboQuantKVCache.attention_scores uses that estimator for
# the quantized part).  Stage 1 is the MSE key codec at bits - 1 (at least 1); stage 2 keeps one sign
# bit per coordinate of S r, r the residual in the original space, and ||r||.
# Readings: S is a d x d matrix of standard normal draws taken from this build's generator with seed
# + 10000 (the page's offset; its torch stream is not reproduced); the multiply uses S_op = fp16(S),
# as the rotation uses Pi_op; a sign bit is 1 for +1 (S r >= 0, zero included, as the page's
# ``projected >= 0``); ||r|| is stored in f32 like the key norm (the page keeps both in fp16).
# ----------------------------------------------------------------------------------------------

QJL_SEED_OFFSET = 10000


def qjl_mse_bits(bits: int) -> int:
    """Bits of the MSE stage of a ``bits``-bit QJL key: max(bits - 1, 1)."""
    return max(bits - 1, 1)


def qjl_matrix(d: int, seed: int) -> np.ndarray:
    """S (d x d, fp64): Gaussian draws i*d + j of the generator seeded with seed + 10000."""
    return gaussian_stream(seed + QJL_SEED_OFFSET, d * d).reshape(d, d)


def operational_qjl_matrix(d: int, seed: int) -> np.ndarray:
    """S_op = fp16(S) as fp64 values: the projection the tensor-core path multiplies by."""
    return to_fp16_values(qjl_matrix(d, seed))


def encode_k_qjl(x16: np.ndarray, pi_op: np.ndarray, c_op: np.ndarray, t: np.ndarray, s_op: np.ndarray,
                 idx: np.ndarray | None = None):
    """QJL key encode of fp16 rows x [N][d], in the page's order.

    n = ||x||; y = Pi_op x / (n + 1e-8); idx = nearest level of the (bits-1)-bit codebook (c_op, t);
    k_mse = n * Pi_op^T c_op[idx] (the reconstruction in the original space); r = x - k_mse;
    rho = ||r||; proj = S_op r; sign bit = (proj >= 0).
    ``idx`` may be given (e.g. another implementation's indices) to take r from those.
    Returns (idx [N][d], n [N], y [N][d], bits [N][d] bool, rho [N], proj [N][d]).
    """
    x = np.asarray(x16).astype(np.float64)
    n = np.sqrt(np.sum(x * x, axis=-1))
    y = (x @ pi_op.T) / (n + 1e-8)[:, None]
    if idx is None:
        idx = nearest_index(y, t)
    k_mse = n[:, None] * (c_op[np.asarray(idx)] @ pi_op)
    r = x - k_mse
    rho = np.sqrt(np.sum(r * r, axis=-1))
    proj = r @ s_op.T
    return np.asarray(idx), n, y, proj >= 0, rho, proj


def qjl_inner_products(q: np.ndarray, idx: np.ndarray, norms: np.ndarray, sign_bits: np.ndarray, rho: np.ndarray,
                       pi_op: np.ndarray, c_op: np.ndarray, s_op: np.ndarray) -> np.ndarray:
    """The asymmetric estimate of <q, k_t> for one query q [d] and T keys:
    <q, k_mse_t> + rho_t * sqrt(pi / 2) / m * <S_op q, signs_t>, signs in {-1, +1}, m = rows of S."""
    q = np.asarray(q, dtype=np.float64)
    term1 = decode_k(idx, norms, pi_op, c_op) @ q
    pm = np.where(np.asarray(sign_bits, dtype=bool), 1.0, -1.0)
    term2 = math.sqrt(math.pi / 2.0) / s_op.shape[0] * np.asarray(rho, dtype=np.float64) * (pm @ (s_op @ q))
    return term1 + term2


def attend_qjl(q16: np.ndarray, k_idx: np.ndarray, k_norms: np.ndarray, k_bits: np.ndarray, k_rho: np.ndarray,
               v_hat: np.ndarray, pi_op: np.ndarray, c_op: np.ndarray, s_op: np.ndarray,
               scale: float | None = None, seq_lens: np.ndarray | None = None, win_k16: np.ndarray | None = None,
               win_v16: np.ndarray | None = None, win_lens: np.ndarray | None = None) -> np.ndarray:
    """Decode attention whose compressed part is scored by the QJL estimator ([P3] store.py
    ``attention_scores``: scale * the asymmetric scores of the quantized part, then scale * q . key_buffer
    for the recent uncompressed window when there is one; softmax over both; weights @ values).

    q16 [B][H_q][d]; k_idx, k_bits [B][H_kv][T][d]; k_norms, k_rho [B][H_kv][T]; v_hat [B][H_kv][T][d];
    optional window win_k16, win_v16 [B][H_kv][W][d] fp16 with win_lens [B].  Returns o [B][H_q][d] fp64.
    """
    bsz, hq, d = q16.shape
    hkv = k_idx.shape[1]
    grp = hq // hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((bsz, hq, d), dtype=np.float64)
    for b in range(bsz):
        tl = k_idx.shape[2] if seq_lens is None else int(seq_lens[b])
        wl = 0 if win_k16 is None else (win_k16.shape[2] if win_lens is None else int(win_lens[b]))
        for h in range(hq):
            kv = h // grp
            q = np.asarray(q16[b, h]).astype(np.float64)
            s = scale * qjl_inner_products(q, k_idx[b, kv, :tl], k_norms[b, kv, :tl], k_bits[b, kv, :tl],
                                           k_rho[b, kv, :tl], pi_op, c_op, s_op)
            v_all = np.asarray(v_hat[b, kv, :tl], dtype=np.float64)
            if wl:
                s = np.concatenate([s, scale * (np.asarray(win_k16[b, kv, :wl]).astype(np.float64) @ q)])
                v_all = np.concatenate([v_all, np.asarray(win_v16[b, kv, :wl]).astype(np.float64)], axis=0)
            if s.shape[0] == 0:
                continue
            p = np.exp(s - s.max())
            out[b, h] = (p / p.sum()) @ v_all
    return out


def qjl_key_row_bytes(d: int, bits: int, norm_bytes: int = 4) -> int:
    """Bytes of one QJL key: (bits-1)-bit codes + d sign bits + the norm and the residual norm."""
    return k_row_bytes(d, qjl_mse_bits(bits)) + d // 8 + 2 * norm_bytes
