"""GPU parity of decode attention with a window of recent uncompressed tokens (tq_attend_decode_window
through the C ABI) against the oracle's attend_window on the same compressed cache and window: relative L2
<= 1e-3 per output head vector.  "KV Cache API", store.py TurboQuantKVCache: the quantized part's scores and
the fp16 buffer's scores share one softmax; the buffer's values are used as stored."""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
STREAM_WK, STREAM_WV = 21, 22


def _cache(b, hkv, t, d, kb, vb, vg, seed=0):
    ks = synth.channel_scales(seed, hkv, d, "k")
    vs = synth.channel_scales(seed, hkv, d, "v")
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=ks).view(-1, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=DEV, scales=vs).view(-1, d)
    cd = tq.Codec(d, kb, seed)
    kp, kn = cd.encode_k(k)
    vd, vsc, vz = tq.encode_v(v, vb, vg)
    return cd, tq.Cache(kp, kn, vd, vsc, vz)


def _window(b, hkv, w, d, seed=0):
    wk = synth.kv_tensor(seed, STREAM_WK, b, hkv, w, d, device=DEV)
    wv = synth.kv_tensor(seed, STREAM_WV, b, hkv, w, d, device=DEV)
    return wk, wv


def _oracle(cd, cache, q16, wk, wv, bi, h, rows, wl, vb, vg, g):
    d, kb = cd.d, cd.bits
    pi, c, _ = params(d, kb, cd.seed)
    r = torch.as_tensor(rows, device=DEV, dtype=torch.int64)
    idx = o.unpack_lsb(to_np(cache.k_packed[r]), kb, d) if len(rows) else np.zeros((0, d), np.int64)
    nrm = to_np(cache.k_norms[r]).astype(np.float64)
    layout = "token" if vg == d else "group"
    vh = (o.decode_v(to_np(cache.v_data[r]), to_np(cache.v_scales[r]), to_np(cache.v_zeros[r]), vb, d, 32, layout)
          if len(rows) else np.zeros((0, d)))
    qs = q16[bi:bi + 1, h * g:(h + 1) * g]
    wkh = to_np(wk[bi:bi + 1, h:h + 1, :wl])
    wvh = to_np(wv[bi:bi + 1, h:h + 1, :wl])
    return o.attend_window(qs, idx[None, None], nrm[None, None], vh[None, None], wkh, wvh, pi, c)[0]


def _run(b, hkv, hq, t, d, kb, vb, vg, w, seq_lens, win_lens, seed=0):
    cd, cache = _cache(b, hkv, t, d, kb, vb, vg, seed)
    wk, wv = _window(b, hkv, w, d, seed)
    q16 = synth.normal_fp16(seed, synth.STREAM_Q, (b, hq, d))
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    wl = torch.tensor(win_lens, dtype=torch.int32, device=DEV) if win_lens is not None else None
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=t,
                                 seq_lens=sl, win_k=wk, win_v=wv, win_lens=wl))
    g = hq // hkv
    for bi in range(b):
        lw = w if win_lens is None else max(0, min(win_lens[bi], w))
        for h in range(hkv):
            rows = (bi * hkv + h) * t + np.arange(seq_lens[bi])
            ref = _oracle(cd, cache, q16.numpy(), wk, wv, bi, h, rows, lw, vb, vg, g)
            for gi in range(g):
                got = out[bi, h * g + gi]
                if seq_lens[bi] == 0 and lw == 0:
                    assert np.all(got == 0)
                else:
                    assert rel_l2(got, ref[gi]) <= L2_RTOL, (bi, h, gi, rel_l2(got, ref[gi]))
    assert tq.read_device_flag() == 0
    return cd, cache, q16, out


@pytest.mark.parametrize("d,kb,vb,vg", [(128, 3, 2, 32), (64, 4, 4, 64), (256, 2, 8, 32)])
def test_window_formats(d, kb, vb, vg):
    _run(3, 2, 8, 320, d, kb, vb, vg, w=128, seq_lens=[320, 157, 0], win_lens=[128, 37, 5])


def test_window_edges():
    # a full window and no compressed tokens, an empty window, both empty, lengths past the capacity
    _run(4, 2, 4, 160, 128, 4, 2, 32, w=64, seq_lens=[0, 160, 0, 33], win_lens=[64, 0, 0, 1000])
    _run(2, 1, 8, 64, 128, 3, 2, 32, w=256, seq_lens=[64, 17], win_lens=None)


def test_empty_window_equals_the_plain_call():
    cd, cache, q16, out = _run(2, 2, 8, 256, 128, 3, 2, 32, w=32, seq_lens=[256, 100], win_lens=[0, 0])
    plain = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=2, v_bits=2, v_group=32, max_seq_len=256,
                                   seq_lens=torch.tensor([256, 100], dtype=torch.int32, device=DEV)))
    # the same compressed partials merged with an empty one: equal up to the merge's rounding
    for bi in range(2):
        for hh in range(8):
            assert rel_l2(out[bi, hh], plain[bi, hh]) <= 1e-6


def test_window_70b_class_full_size_sampled():
    # batch 1, 8 kv heads, 64 query heads, 131072 compressed tokens + 128 recent fp16 tokens, K3 / V2 g32
    b, hkv, hq, t, d, w = 1, 8, 64, 131072, 128, 128
    cd, cache = _cache(b, hkv, t, d, 3, 2, 32)
    wk, wv = _window(b, hkv, w, d)
    q16 = synth.normal_fp16(0, synth.STREAM_Q, (b, hq, d))
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=2, v_group=32, max_seq_len=t,
                                 win_k=wk, win_v=wv))
    g = hq // hkv
    for h in (0, 6):
        rows = h * t + np.arange(t)
        ref = _oracle(cd, cache, q16.numpy(), wk, wv, 0, h, rows, w, 2, 32, g)
        for gi in range(g):
            assert rel_l2(out[0, h * g + gi], ref[gi]) <= L2_RTOL
    assert tq.read_device_flag() == 0
