"""GPU parity of the compressed path's attention logits (tq_attend_scores through the C ABI) with the oracle's
path-B scores (scale * n_t * <Pi_op q, c_op[idx_t]>, the form pinned equal to the decoded-key scores), and the
score-fidelity metrics of "turboquant-pytorch" (V3: Attention Score Accuracy) on a synthetic 8K cache.

Tolerance: the query's fp16 hi/lo halves carry ~2^-22 of the largest rotated coordinate, so a score's error is
bounded relative to the scores' scale, not to the score itself (a score near zero after cancellation keeps an
absolute error of the same size): max |s - s_ref| <= 1e-4 (1 + max |s_ref|)."""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import fidelity, synth, tq
from oracle import tq_oracle as o
from _tqh import params, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _close(got, ref):
    return float(np.abs(got - ref).max()) <= 1e-4 * (1.0 + float(np.abs(ref).max()))


def _scores_ref(cd, cache, q16, bi, h, rows, g):
    d, kb = cd.d, cd.bits
    pi, c, _ = params(d, kb, cd.seed)
    r = torch.as_tensor(rows, device=DEV, dtype=torch.int64)
    idx = o.unpack_lsb(to_np(cache.k_packed[r]), kb, d)
    nrm = to_np(cache.k_norms[r]).astype(np.float64)
    vh = np.zeros((len(rows), d))
    refs = []
    for gi in range(g):
        _, s_a, s_b = o.attend_one(q16[bi, h * g + gi], idx, nrm, vh, pi, c, 1.0 / np.sqrt(d))
        refs.append(s_b)
    return refs


@pytest.mark.parametrize("d,kb", [(128, 3), (64, 4), (256, 2)])
def test_scores_contiguous(d, kb):
    b, hkv, hq, t = 2, 2, 8, 304
    k = synth.kv_tensor(0, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=synth.channel_scales(0, hkv, d, "k"))
    cd = tq.Codec(d, kb, 0)
    kp, kn = cd.encode_k(k.view(-1, d))
    vd, vs, vz = tq.encode_v(k.view(-1, d), 2, 32)
    cache = tq.Cache(kp, kn, vd, vs, vz)
    q16 = synth.normal_fp16(0, synth.STREAM_Q, (b, hq, d))
    lens = [304, 150]
    s = to_np(tq.attend_scores(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=2, max_seq_len=t,
                               seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV)))
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            rows = (bi * hkv + h) * t + np.arange(lens[bi])
            refs = _scores_ref(cd, cache, q16.numpy(), bi, h, rows, g)
            for gi in range(g):
                got = s[bi, h * g + gi]
                assert _close(got[:lens[bi]], refs[gi])
                assert np.all(np.isneginf(got[lens[bi]:]))
    assert tq.read_device_flag() == 0


def test_scores_paged():
    b, hkv, hq, d, kb = 3, 2, 4, 128, 4
    lens = [40, 16, 1]
    max_blocks = 3
    nblocks = b * max_blocks + 2
    table = synth.block_table(8, b, max_blocks, nblocks)
    cd = tq.Codec(d, kb, 0)
    rows_total = nblocks * hkv * 16
    x = synth.normal_fp16(3, synth.STREAM_K, (rows_total, d)).to(DEV)
    kp, kn = cd.encode_k(x)
    vd, vs, vz = tq.encode_v(x, 4, 32)
    cache = tq.Cache(kp, kn, vd, vs, vz)
    q16 = synth.normal_fp16(5, synth.STREAM_Q, (b, hq, d))
    s = to_np(tq.attend_scores(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=4, block_table=table.to(DEV),
                               seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV)))
    assert s.shape == (b, hq, max_blocks * 16)
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            rows = o.paged_rows(table.numpy(), bi, h, lens[bi], hkv, 16)
            refs = _scores_ref(cd, cache, q16.numpy(), bi, h, rows, g)
            for gi in range(g):
                assert _close(s[bi, h * g + gi, :lens[bi]], refs[gi])
                assert np.all(np.isneginf(s[bi, h * g + gi, lens[bi]:]))


def test_score_fidelity_of_an_8k_cache():
    # Llama-3-8B-shaped layer at 8K: K 4-bit against the exact fp16 scores; the page's V3 K4 reports cosine
    # 0.9996 / top-1 94 % / top-5 97 % on real captured KV (context only: these caches are synthetic)
    b, hkv, hq, t, d = 2, 8, 32, 8192, 128
    k = synth.kv_tensor(0, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=synth.channel_scales(0, hkv, d, "k"))
    cd = tq.Codec(d, 4, 0)
    kp, kn = cd.encode_k(k.view(-1, d))
    vd, vs, vz = tq.encode_v(k.view(-1, d), 2, 32)
    q = synth.normal_fp16(0, synth.STREAM_Q, (b, hq, d), device=DEV)
    approx = tq.attend_scores(cd, q, tq.Cache(kp, kn, vd, vs, vz), num_kv_heads=hkv, v_bits=2, max_seq_len=t)
    m = fidelity.score_fidelity(approx, fidelity.exact_scores(q, k))
    assert m["pairs"] == b * hq
    assert m["cosine"] > 0.99 and m["top5"] >= m["top1"]
