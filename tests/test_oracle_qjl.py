"""Pins of the oracle's QJL residual keys ("KV Cache API", compressors.py, TurboQuantCompressorV2) against
facts that do not come from the oracle itself:

* the estimator <q, k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)> is unbiased over the draw of S (the
  Gaussian identity E[z1 sign(z2)] = sqrt(2/pi) cov(z1, z2) / sd(z2)), and its variance over S is the
  closed form (pi/2 ||q||^2 ||r||^2 - <q, r>^2) / m -- checked by Monte Carlo over many seeds of S while the
  MSE term alone is visibly biased;
* the residual is the MSE stage's error in the original space: mean ||r||^2 / ||x||^2 equals the
  distortion D(b - 1, d) of the (b-1)-bit codebook;
* the bit budget reproduces the compression column the turboquant-pytorch page prints for V2 and V3;
* the degenerate zero key, and attention with zero residuals reducing to the (separately pinned) MSE-only
  and window attention.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import tq_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")


def _fp16(a):
    return np.asarray(a, dtype=np.float16)


def _params(d, bits, seed=0):
    pi = o.operational_rotation(d, seed)
    c, t = o.operational_codebook(d, o.qjl_mse_bits(bits))
    return pi, c, t


def _monte_carlo(d, bits, draws, rng_seed):
    rng = np.random.default_rng(rng_seed)
    x16 = _fp16(rng.standard_normal((1, d)))
    q = rng.standard_normal(d) + x16[0].astype(np.float64)      # correlated with the key: a large <q, r>
    pi, c, t = _params(d, bits)
    est, mse_term = [], []
    r_ref = None
    for s in range(1, draws + 1):
        s_op = o.operational_qjl_matrix(d, s)
        idx, n, _, sb, rho, proj = o.encode_k_qjl(x16, pi, c, t, s_op)
        est.append(o.qjl_inner_products(q, idx, n, sb, rho, pi, c, s_op)[0])
        if r_ref is None:
            r_ref = x16[0].astype(np.float64) - o.decode_k(idx, n, pi, c)[0]
            mse_term.append(float(o.decode_k(idx, n, pi, c)[0] @ q))
    return np.array(est), float(x16[0].astype(np.float64) @ q), mse_term[0], q, r_ref


def test_estimator_is_unbiased_and_has_the_closed_form_variance():
    d, bits, draws = 32, 2, 3000
    est, exact, mse_only, q, r = _monte_carlo(d, bits, draws, 7)
    se = est.std(ddof=1) / math.sqrt(draws)
    assert abs(est.mean() - exact) <= 4 * se, (est.mean(), exact, se)
    # the MSE stage alone is biased by <q, r>, many standard errors away: the test has power
    assert abs(mse_only - exact) > 20 * se
    var_closed = (math.pi / 2 * (q @ q) * (r @ r) - (q @ r) ** 2) / d
    assert abs(est.var(ddof=1) / var_closed - 1.0) <= 0.10, (est.var(ddof=1), var_closed)


def test_wrong_constant_or_projection_would_be_biased():
    # the same draws with sqrt(2/pi) in place of sqrt(pi/2), or S^T q in place of S q, miss <q, k> by many
    # standard errors -- the plausible slips the unbiasedness pin rules out
    d, bits, draws = 32, 2, 1500
    rng = np.random.default_rng(3)
    x16 = _fp16(rng.standard_normal((1, d)))
    q = rng.standard_normal(d) + x16[0].astype(np.float64)
    pi, c, t = _params(d, bits)
    good, const, trans = [], [], []
    for s in range(1, draws + 1):
        s_op = o.operational_qjl_matrix(d, s)
        idx, n, _, sb, rho, _ = o.encode_k_qjl(x16, pi, c, t, s_op)
        t1 = float(o.decode_k(idx, n, pi, c)[0] @ q)
        pm = np.where(sb[0], 1.0, -1.0)
        good.append(t1 + math.sqrt(math.pi / 2) / d * rho[0] * (pm @ (s_op @ q)))
        const.append(t1 + math.sqrt(2 / math.pi) / d * rho[0] * (pm @ (s_op @ q)))
        trans.append(t1 + math.sqrt(math.pi / 2) / d * rho[0] * (pm @ (s_op.T @ q)))
    exact = float(x16[0].astype(np.float64) @ q)
    for name, v in (("const", const), ("trans", trans)):
        v = np.array(v)
        se = v.std(ddof=1) / math.sqrt(draws)
        assert abs(v.mean() - exact) > 6 * se, name
    g = np.array(good)
    assert abs(g.mean() - exact) <= 4 * g.std(ddof=1) / math.sqrt(draws)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_residual_energy_is_the_mse_stage_distortion(bits):
    d, n = 128, 20000
    rng = np.random.default_rng(bits)
    x16 = _fp16(rng.standard_normal((n, d)))
    pi, c, t = _params(d, bits)
    s_op = o.operational_qjl_matrix(d, 0)
    _, nrm, _, _, rho, _ = o.encode_k_qjl(x16, pi, c, t, s_op)
    measured = float(np.mean((rho / nrm) ** 2))
    dist = o.sphere_distortion(d, c, t)
    assert abs(measured / dist - 1.0) <= 0.02, (bits, measured, dist)


def test_mse_bits_follow_the_page():
    assert [o.qjl_mse_bits(b) for b in (1, 2, 3, 4, 5)] == [1, 1, 2, 3, 4]


def test_bit_budget_reproduces_the_printed_compression():
    fig = json.load(open(GOLDEN))["v2_v3_compression"]
    d = fig["setting"]["head_dim"]
    nb = fig["setting"]["norm_bytes"]
    for row in fig["rows"]:
        kb, vb = row["key_bits"], row["value_bits"]
        k_bytes = o.qjl_key_row_bytes(d, kb, nb) if row["qjl"] else o.k_row_bytes(d, kb) + nb
        v_bytes = o.k_row_bytes(d, vb) + nb
        ratio = 2 * (2 * d) / (k_bytes + v_bytes)
        assert round(ratio, fig["printed_digits"]) == row["ratio"], (row, ratio)


def test_zero_key_keeps_positive_signs_and_no_residual():
    d, bits = 64, 3
    pi, c, t = _params(d, bits)
    s_op = o.operational_qjl_matrix(d, 1)
    idx, n, _, sb, rho, proj = o.encode_k_qjl(np.zeros((1, d), np.float16), pi, c, t, s_op)
    assert n[0] == 0 and rho[0] == 0 and np.all(proj == 0) and np.all(sb)
    q = np.random.default_rng(0).standard_normal(d)
    assert o.qjl_inner_products(q, idx, n, sb, rho, pi, c, s_op)[0] == 0.0


def test_projection_stream_is_its_own():
    d = 64
    s = o.qjl_matrix(d, 0)
    assert abs(s.mean()) < 0.1 and abs(s.var() - 1.0) < 0.1
    # the projection for seed s is not the rotation's draw for the same seed
    g = o.gaussian_stream(0, d * d).reshape(d, d)
    assert not np.allclose(s, g)
    assert np.array_equal(o.operational_qjl_matrix(d, 0), np.float16(s).astype(np.float64))


def test_attention_with_zero_residuals_is_the_mse_attention():
    rng = np.random.default_rng(5)
    b, hkv, hq, tl, d, w = 2, 2, 4, 40, 32, 6
    pi, c, _ = _params(d, 3)
    s_op = o.operational_qjl_matrix(d, 0)
    idx = rng.integers(0, len(c), (b, hkv, tl, d))
    nrm = rng.uniform(0.5, 3.0, (b, hkv, tl))
    sb = rng.integers(0, 2, (b, hkv, tl, d)).astype(bool)
    v = rng.standard_normal((b, hkv, tl, d))
    q16 = _fp16(rng.standard_normal((b, hq, d)))
    zero = np.zeros((b, hkv, tl))
    ref = o.attend(q16, idx, nrm, v, pi, c, seq_lens=np.array([40, 17]))
    got = o.attend_qjl(q16, idx, nrm, sb, zero, v, pi, c, s_op, seq_lens=np.array([40, 17]))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    wk = _fp16(rng.standard_normal((b, hkv, w, d)))
    wv = _fp16(rng.standard_normal((b, hkv, w, d)))
    ref_w = o.attend_window(q16, idx, nrm, v, wk, wv, pi, c, seq_lens=np.array([40, 0]), win_lens=np.array([3, 6]))
    got_w = o.attend_qjl(q16, idx, nrm, sb, zero, v, pi, c, s_op, seq_lens=np.array([40, 0]), win_k16=wk, win_v16=wv,
                         win_lens=np.array([3, 6]))
    assert np.allclose(got_w, ref_w, rtol=1e-12, atol=1e-12)


def test_attention_single_token_and_dominant_logit():
    rng = np.random.default_rng(9)
    d = 32
    pi, c, t = _params(d, 3)
    s_op = o.operational_qjl_matrix(d, 0)
    x16 = _fp16(rng.standard_normal((3, d)))
    idx, n, _, sb, rho, _ = o.encode_k_qjl(x16, pi, c, t, s_op)
    v = rng.standard_normal((1, 1, 3, d))
    q16 = _fp16(rng.standard_normal((1, 1, d)))
    one = o.attend_qjl(q16, idx[None, None, :1], n[None, None, :1], sb[None, None, :1], rho[None, None, :1],
                       v[:, :, :1], pi, c, s_op)
    assert np.allclose(one[0, 0], v[0, 0, 0], rtol=0, atol=1e-12)
    # a huge scale makes the softmax one-hot on the largest estimated score
    est = o.qjl_inner_products(q16[0, 0].astype(np.float64), idx, n, sb, rho, pi, c, s_op)
    big = o.attend_qjl(q16, idx[None, None], n[None, None], sb[None, None], rho[None, None], v, pi, c, s_op,
                       scale=1e6)
    assert np.allclose(big[0, 0], v[0, 0, int(np.argmax(est))], atol=1e-9)
