"""Pins of the oracle's decode-step attention: analytic cases (equal keys, one token, a dominant
logit), the identity between the decode-then-dot and rotate-the-query score paths, the GQA
mapping, a dense library softmax-attention on the decoded cache, and the paged layout."""
import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as o

D = 128


def _cache(rng, b, hkv, t, kb=3, vb=2):
    pi = o.operational_rotation(D, 1)
    c, tt = o.operational_codebook(D, kb)
    k16 = rng.standard_normal((b * hkv * t, D)).astype(np.float16)
    v16 = rng.standard_normal((b * hkv * t, D)).astype(np.float16)
    idx, norms, _ = o.encode_k(k16, pi, tt)
    data, s, z, _ = o.encode_v(v16, vb)
    vh = o.decode_v(data, s, z, vb, D)
    return (pi, c, idx.reshape(b, hkv, t, D), norms.astype(np.float32).astype(np.float64).reshape(b, hkv, t),
            vh.reshape(b, hkv, t, D))


def test_score_paths_agree_and_match_dense_attention():
    rng = np.random.default_rng(0)
    b, hkv, hq, t = 2, 2, 8, 300
    pi, c, idx, norms, vh = _cache(rng, b, hkv, t)
    q16 = rng.standard_normal((b, hq, D)).astype(np.float16)
    out = o.attend(q16, idx, norms, vh, pi, c)
    g = hq // hkv
    for bi in range(b):
        for h in range(hq):
            _, sa, sb = o.attend_one(q16[bi, h], idx[bi, h // g], norms[bi, h // g], vh[bi, h // g], pi, c, 1 / math.sqrt(D))
            assert np.max(np.abs(sa - sb)) < 1e-12 * np.max(np.abs(sa))
    # dense attention by the library on the decoded cache, GQA by repeating kv heads
    kh = np.stack([[o.decode_k(idx[bi, h], norms[bi, h], pi, c) for h in range(hkv)] for bi in range(b)])
    qt = torch.from_numpy(q16.astype(np.float64))[:, :, None, :]
    kt = torch.from_numpy(kh).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(vh.astype(np.float64)).repeat_interleave(g, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[:, :, 0, :].numpy()
    assert np.max(np.abs(ref - out)) < 1e-12 * np.max(np.abs(out))


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    pi, c, idx, norms, vh = _cache(rng, 1, 1, 50)
    idx[:] = idx[:, :, :1]
    norms[:] = norms[:, :, :1]
    q16 = rng.standard_normal((1, 1, D)).astype(np.float16)
    out = o.attend(q16, idx, norms, vh, pi, c)
    assert np.allclose(out[0, 0], vh[0, 0].astype(np.float64).mean(0), rtol=0, atol=1e-12)


def test_single_token_and_dominant_logit():
    rng = np.random.default_rng(2)
    pi, c, idx, norms, vh = _cache(rng, 1, 1, 40)
    q16 = rng.standard_normal((1, 1, D)).astype(np.float16)
    assert np.allclose(o.attend(q16, idx[:, :, :1], norms[:, :, :1], vh[:, :, :1], pi, c)[0, 0], vh[0, 0, 0], atol=1e-12)
    # make token 17's key a large multiple of the query direction
    s = np.array([np.dot(pi @ q16[0, 0].astype(np.float64), c[idx[0, 0, k]]) for k in range(40)])
    k_star = int(np.argmax(s))
    norms[0, 0, k_star] *= 1e4
    out = o.attend(q16, idx, norms, vh, pi, c)
    assert np.allclose(out[0, 0], vh[0, 0, k_star], atol=1e-9)


def test_gqa_mapping():
    rng = np.random.default_rng(3)
    pi, c, idx, norms, vh = _cache(rng, 1, 4, 20)
    for h in range(4):
        vh[0, h] = float(h + 1)
    q16 = rng.standard_normal((1, 16, D)).astype(np.float16)
    out = o.attend(q16, idx, norms, vh, pi, c)
    for hq in range(16):
        assert np.allclose(out[0, hq], hq // 4 + 1.0, atol=1e-12)


def test_seq_lens_and_paged_layout():
    rng = np.random.default_rng(4)
    b, hkv, hq, t, bs = 3, 2, 4, 64, 16
    pi, c, idx, norms, vh = _cache(rng, b, hkv, t)
    q16 = rng.standard_normal((b, hq, D)).astype(np.float16)
    lens = np.array([64, 17, 1])
    ref = o.attend(q16, idx, norms, vh, pi, c, seq_lens=lens)
    for bi in range(b):
        short = o.attend(q16[bi:bi + 1], idx[bi:bi + 1, :, :lens[bi]], norms[bi:bi + 1, :, :lens[bi]],
                         vh[bi:bi + 1, :, :lens[bi]], pi, c)
        assert np.array_equal(short[0], ref[bi])
    # scatter the contiguous cache into a paged pool through a random block table, read it back
    nblk = b * t // bs
    table = rng.permutation(nblk + 5)[:nblk].reshape(b, t // bs)
    pool_idx = np.zeros(((nblk + 5) * hkv * bs, D), np.int64)
    for bi in range(b):
        for h in range(hkv):
            pool_idx[o.paged_rows(table, bi, h, t, hkv, bs)] = idx[bi, h]
    for bi in range(b):
        for h in range(hkv):
            assert np.array_equal(pool_idx[o.paged_rows(table, bi, h, t, hkv, bs)], idx[bi, h])


# ---- recent uncompressed window ("KV Cache API", store.py TurboQuantKVCache: quantized part + fp16 buffer)

def _window_case(seed, tl, wl, d=64, kb=3, vb=2):
    rng = np.random.default_rng(seed)
    pi = o.operational_rotation(d, seed)
    c, t = o.operational_codebook(d, kb)
    q16 = rng.standard_normal((1, 4, d)).astype(np.float16)
    k16 = rng.standard_normal((1, 2, tl, d)).astype(np.float16)
    v16 = rng.standard_normal((1, 2, tl, d)).astype(np.float16)
    idx, nrm, _ = o.encode_k(k16.reshape(-1, d), pi, t)
    idx = idx.reshape(1, 2, tl, d)
    nrm = nrm.reshape(1, 2, tl)
    dat, sc, zr, _ = o.encode_v(v16.reshape(-1, d), vb)
    vh = o.decode_v(dat, sc, zr, vb, d).reshape(1, 2, tl, d)
    wk = rng.standard_normal((1, 2, wl, d)).astype(np.float16)
    wv = rng.standard_normal((1, 2, wl, d)).astype(np.float16)
    return q16, idx, nrm, vh, wk, wv, pi, c


def test_window_attention_is_softmax_over_the_concatenation():
    # pinned against the library's scaled-dot-product attention on the explicitly concatenated keys and values
    q16, idx, nrm, vh, wk, wv, pi, c = _window_case(1, 37, 21)
    got = o.attend_window(q16, idx, nrm, vh, wk, wv, pi, c)
    for h in range(4):
        kv = h // 2
        k_all = np.concatenate([o.decode_k(idx[0, kv], nrm[0, kv], pi, c), wk[0, kv].astype(np.float64)])
        v_all = np.concatenate([vh[0, kv].astype(np.float64), wv[0, kv].astype(np.float64)])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q16[0, h].astype(np.float64))[None, None, None],
            torch.from_numpy(k_all)[None, None], torch.from_numpy(v_all)[None, None])[0, 0, 0].numpy()
        assert np.abs(got[0, h] - ref).max() < 1e-12


def test_window_attention_reduces_to_its_parts():
    q16, idx, nrm, vh, wk, wv, pi, c = _window_case(2, 40, 16)
    # an empty window is the compressed attention; an empty compressed part is attention over the window alone
    assert np.abs(o.attend_window(q16, idx, nrm, vh, wk, wv, pi, c, win_lens=np.array([0]))
                  - o.attend(q16, idx, nrm, vh, pi, c)).max() < 1e-12
    only_w = o.attend_window(q16, idx, nrm, vh, wk, wv, pi, c, seq_lens=np.array([0]))
    for h in range(4):
        s = wk[0, h // 2].astype(np.float64) @ q16[0, h].astype(np.float64) / np.sqrt(64)
        p = np.exp(s - s.max())
        assert np.abs(only_w[0, h] - (p / p.sum()) @ wv[0, h // 2].astype(np.float64)).max() < 1e-12
    both_empty = o.attend_window(q16, idx, nrm, vh, wk, wv, pi, c, seq_lens=np.array([0]), win_lens=np.array([0]))
    assert np.all(both_empty == 0)
