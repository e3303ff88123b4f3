"""GPU parity of keys of 5..8 bits (for example the protected first and last layers of "turboquant-pytorch"
V3, kept at 8 bits) through the C ABI: the key codec (indices bit-exact except in-band flips, norms 1e-6,
decode rel-L2 1e-3), the fused attention and the score logits (rel-L2 1e-3) against the oracle.  Wide codes
use a single-code table (2^bits entries) and, in the encoder, a binary search over the boundaries; d = 64 and
128."""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, NORM_RTOL, check_key_indices, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
_CODECS = {}


def codec(d, bits):
    if (d, bits) not in _CODECS:
        _CODECS[(d, bits)] = tq.Codec(d, bits, 0)
    return _CODECS[(d, bits)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [5, 6, 7, 8])
def test_wide_key_codec_parity(d, bits):
    cd = codec(d, bits)
    pi, c, t = params(d, bits, 0)
    for n in (1, 129, 1000, 4100):
        x = synth.normal_fp16(n + 17 * bits, synth.STREAM_K, (n, d))
        x[0, 0] = 0.0 if n > 1 else x[0, 0]
        packed, norms = cd.encode_k(x.to(DEV))
        out = to_np(cd.decode_k(packed, norms, out_dtype=torch.float32))
        ref_idx, ref_n, y = o.encode_k(x.numpy(), pi, t)
        gidx = o.unpack_lsb(to_np(packed), bits, d)
        check_key_indices(gidx, ref_idx, y, t)
        gn = to_np(norms)
        assert np.all(np.abs(gn - ref_n) <= NORM_RTOL * ref_n)
        ref_dec = o.decode_k(gidx, gn.astype(np.float64), pi, c)
        assert rel_l2(out, ref_dec) <= L2_RTOL
        for r in range(0, n, max(1, n // 32)):
            assert rel_l2(out[r], ref_dec[r]) <= L2_RTOL


def test_wide_key_zero_vector_and_slot_mapping():
    d, bits = 128, 8
    cd = codec(d, bits)
    x = synth.normal_fp16(5, synth.STREAM_K, (200, d))
    x[3] = 0.0
    slots = torch.randperm(256, generator=torch.Generator().manual_seed(8))[:200]
    slots[::7] = -1
    packed = torch.full((256, cd.row_bytes), 0x33, dtype=torch.uint8, device=DEV)
    norms = torch.full((256,), -1.0, device=DEV)
    cd.encode_k(x.to(DEV), slot_mapping=slots.to(DEV), packed=packed, norms=norms)
    ref_p, ref_n = cd.encode_k(x.to(DEV))
    keep = slots >= 0
    assert torch.equal(packed[slots[keep].to(DEV)], ref_p[keep.to(DEV)])
    assert torch.equal(norms[slots[keep].to(DEV)], ref_n[keep.to(DEV)])
    zi = o.unpack_lsb(to_np(ref_p[3:4]), bits, d)
    assert np.all(zi == (1 << (bits - 1)) - 1) and float(ref_n[3]) == 0.0


def test_wide_keys_refused_at_head_dim_256():
    with pytest.raises(tq.TQError, match="d <= 128"):
        tq.Codec(256, 5, 0)


def _cache(b, hkv, t, d, kb, vb, seed=0):
    cd = codec(d, kb)
    ks = synth.channel_scales(seed, hkv, d, "k")
    vs = synth.channel_scales(seed, hkv, d, "v")
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=ks).view(-1, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=DEV, scales=vs).view(-1, d)
    kp, kn = cd.encode_k(k)
    vd, vsc, vz = tq.encode_v(v, vb, 32)
    return cd, tq.Cache(kp, kn, vd, vsc, vz)


@pytest.mark.parametrize("d,kb,vb", [(128, 5, 2), (64, 6, 4), (128, 7, 8), (128, 8, 4), (64, 8, 2)])
def test_wide_key_attention(d, kb, vb):
    b, hkv, hq, t = 2, 2, 8, 608
    lens = [608, 211]
    cd, cache = _cache(b, hkv, t, d, kb, vb)
    q16 = synth.normal_fp16(9, synth.STREAM_Q, (b, hq, d))
    kw = dict(num_kv_heads=hkv, v_bits=vb, v_group=32, max_seq_len=t,
              seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV))
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, **kw))
    scores = to_np(tq.attend_scores(cd, q16.to(DEV), cache, **kw))
    pi, c, _ = params(d, kb, 0)
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            rows = (bi * hkv + h) * t + np.arange(lens[bi])
            r = torch.as_tensor(rows, device=DEV)
            idx = o.unpack_lsb(to_np(cache.k_packed[r]), kb, d)
            nrm = to_np(cache.k_norms[r]).astype(np.float64)
            vh = o.decode_v(to_np(cache.v_data[r]), to_np(cache.v_scales[r]), to_np(cache.v_zeros[r]), vb, d, 32,
                            "group")
            qs = q16.numpy()[bi:bi + 1, h * g:(h + 1) * g]
            ref = o.attend(qs, idx[None, None], nrm[None, None], vh[None, None], pi, c)[0]
            kd = o.decode_k(idx, nrm, pi, c)
            for gi in range(g):
                assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL
                ref_s = kd @ qs[0, gi].astype(np.float64) / np.sqrt(d)
                assert rel_l2(scores[bi, h * g + gi, :lens[bi]], ref_s) <= L2_RTOL
    assert tq.read_device_flag() == 0


def test_wide_key_attention_long_split_sequence():
    # 8-bit keys over one 16384-token sequence split across many CTAs
    d, kb, vb = 128, 8, 2
    cd, cache = _cache(1, 1, 16384, d, kb, vb, seed=2)
    q16 = synth.normal_fp16(3, synth.STREAM_Q, (1, 8, d))
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=1, v_bits=vb, max_seq_len=16384))
    pi, c, _ = params(d, kb, 0)
    idx = o.unpack_lsb(to_np(cache.k_packed), kb, d)
    nrm = to_np(cache.k_norms).astype(np.float64)
    vh = o.decode_v(to_np(cache.v_data), to_np(cache.v_scales), to_np(cache.v_zeros), vb, d, 32, "group")
    ref = o.attend(q16.numpy(), idx[None, None], nrm[None, None], vh[None, None], pi, c)[0]
    for gi in range(8):
        assert rel_l2(out[0, gi], ref[gi]) <= L2_RTOL


def test_wide_key_attention_format_refusal():
    cd, cache = _cache(1, 1, 32, 128, 6, 2)
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device=DEV)
    with pytest.raises(tq.TQError, match="2, 4 or 8 bits"):
        tq.attend_decode(cd, q, cache, num_kv_heads=1, v_bits=3, max_seq_len=32)
