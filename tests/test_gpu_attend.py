"""GPU parity of the fused decode attention (tq_attend_decode through the C ABI) with the fp64 oracle
run on the same compressed cache (the GPU's indices, norms and value codes): relative L2 <= 1e-3 per
output head vector.  Covers contiguous and paged layouts, ragged and empty sequences, split-K and
single-split launches, GQA groups 1..8, head dims 64/128/256 and every value format."""
import math

import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
_CODECS = {}


def codec(d, bits, seed=0, rotation="haar"):
    if (d, bits, seed, rotation) not in _CODECS:
        _CODECS[(d, bits, seed, rotation)] = tq.Codec(d, bits, seed, rotation=rotation)
    return _CODECS[(d, bits, seed, rotation)]


def build_contiguous(b, hkv, t, d, kb, vb, vg, seed=0, scaled=True, rotation="haar"):
    ks = synth.channel_scales(seed, hkv, d, "k") if scaled else None
    vs = synth.channel_scales(seed, hkv, d, "v") if scaled else None
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=ks).view(-1, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=DEV, scales=vs).view(-1, d)
    cd = codec(d, kb, seed, rotation)
    kp, kn = cd.encode_k(k)
    vd, vsc, vz = tq.encode_v(v, vb, vg)
    return cd, tq.Cache(kp, kn, vd, vsc, vz)


def oracle_heads(cd, cache, q16, b, h, rows, vb, vg, hq_per_kv, scale=None):
    """Oracle outputs of the query heads of kv head h of sequence b over pool rows `rows`."""
    d, kb = cd.d, cd.bits
    pi, c, _ = params(d, kb, cd.seed, cd.rotation)
    r = torch.as_tensor(rows, device=DEV)
    idx = o.unpack_lsb(to_np(cache.k_packed[r]), kb, d)
    nrm = to_np(cache.k_norms[r]).astype(np.float64)
    layout = "token" if vg == d else "group"
    vh = o.decode_v(to_np(cache.v_data[r]), to_np(cache.v_scales[r]), to_np(cache.v_zeros[r]), vb, d, 32, layout)
    g = hq_per_kv
    qs = q16[b:b + 1, h * g:(h + 1) * g]
    if len(rows) == 0:
        return np.zeros((g, d))
    return o.attend(qs, idx[None, None], nrm[None, None], vh[None, None], pi, c, scale)[0]


def _run_contiguous(b, hkv, hq, t, d, kb, vb, vg, seq_lens=None, seed=0, check_bh=None, rotation="haar"):
    cd, cache = build_contiguous(b, hkv, t, d, kb, vb, vg, seed, rotation=rotation)
    q16 = synth.normal_fp16(seed, synth.STREAM_Q, (b, hq, d))
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=DEV) if seq_lens is not None else None
    out = tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=t,
                           seq_lens=sl)
    out = to_np(out)
    g = hq // hkv
    pairs = check_bh if check_bh is not None else [(bi, h) for bi in range(b) for h in range(hkv)]
    for bi, h in pairs:
        length = t if seq_lens is None else seq_lens[bi]
        rows = (bi * hkv + h) * t + np.arange(length)
        ref = oracle_heads(cd, cache, q16.numpy(), bi, h, rows, vb, vg, g)
        for gi in range(g):
            got = out[bi, h * g + gi]
            if length == 0:
                assert np.all(got == 0)
            else:
                assert rel_l2(got, ref[gi]) <= L2_RTOL, (bi, h, gi, rel_l2(got, ref[gi]))
    return out


@pytest.mark.parametrize("d,kb,vb,vg", [(128, 3, 2, 32), (128, 4, 2, 32), (128, 4, 4, 128), (64, 4, 4, 32),
                                        (256, 4, 4, 32), (128, 2, 8, 32), (128, 1, 3, 32), (64, 3, 8, 64),
                                        (256, 2, 2, 256)])
def test_attend_contiguous_formats(d, kb, vb, vg):
    _run_contiguous(2, 2, 8, 320, d, kb, vb, vg, seq_lens=[320, 157])


@pytest.mark.parametrize("d,kb,vb,vg", [(128, 3, 2, 32), (64, 4, 4, 64), (256, 2, 4, 32)])
def test_attend_hadamard_rotation(d, kb, vb, vg):
    # the query is rotated by the codec's (Walsh-Hadamard) rotation like the keys: scores need no un-rotation
    _run_contiguous(2, 2, 8, 320, d, kb, vb, vg, seq_lens=[320, 157], rotation="hadamard")


@pytest.mark.parametrize("hkv,hq", [(4, 4), (2, 16), (1, 8), (3, 6)])
def test_attend_gqa_groups(hkv, hq):
    _run_contiguous(1, hkv, hq, 256, 128, 3, 2, 32, seq_lens=[255])


def test_attend_split_k_and_edges():
    # long sequence with few (b, h): many splits; ragged, single-token and empty sequences
    out = _run_contiguous(4, 1, 4, 4096, 128, 3, 2, 32, seq_lens=[4096, 1, 0, 3001])
    assert np.all(out[2] == 0)
    # many (b, h): one split per CTA, written directly
    _run_contiguous(48, 8, 32, 64, 128, 4, 2, 32, check_bh=[(0, 0), (47, 7), (20, 3)])


def test_attend_repeated_calls_are_identical():
    cd, cache = build_contiguous(1, 2, 2048, 128, 3, 2, 32)
    q = synth.normal_fp16(1, synth.STREAM_Q, (1, 16, 128)).to(DEV)
    ws = tq.attend_workspace(cd, q, cache, num_kv_heads=2, v_bits=2, v_group=32, max_seq_len=2048,
                             block_table=None, seq_lens=None, scale=0.0)
    a = tq.attend_decode(cd, q, cache, num_kv_heads=2, v_bits=2, max_seq_len=2048, workspace=ws).clone()
    b = tq.attend_decode(cd, q, cache, num_kv_heads=2, v_bits=2, max_seq_len=2048, workspace=ws)
    assert torch.equal(a, b)
    ws.fill_(0xFF)                                                   # stale workspace contents do not matter
    c = tq.attend_decode(cd, q, cache, num_kv_heads=2, v_bits=2, max_seq_len=2048, workspace=ws)
    assert torch.equal(a, c)


def test_attend_paged():
    b, hkv, hq, d, kb, vb, vg = 5, 2, 8, 128, 4, 4, 32
    lens = [16 * 9, 33, 1, 100, 160]
    max_blocks = 10
    nblocks = b * max_blocks + 7
    table = synth.block_table(3, b, max_blocks, nblocks)
    cd = codec(d, kb)
    kp = torch.zeros(nblocks * hkv * 16, cd.row_bytes, dtype=torch.uint8, device=DEV)
    kn = torch.zeros(nblocks * hkv * 16, device=DEV)
    vd = torch.zeros(nblocks * hkv * 16, d * vb // 8, dtype=torch.uint8, device=DEV)
    vs = torch.zeros(nblocks * hkv * 16, d // vg, dtype=torch.float16, device=DEV)
    vz = torch.zeros_like(vs)
    cache = tq.Cache(kp, kn, vd, vs, vz)
    # write every sequence's tokens through the slot mapping, as a serving engine appends them
    rows_of = {}
    for bi in range(b):
        for h in range(hkv):
            rows_of[(bi, h)] = o.paged_rows(table.numpy(), bi, h, lens[bi], hkv, 16)
        k = synth.normal_fp16(10 + bi, synth.STREAM_K, (hkv * lens[bi], d))
        v = synth.normal_fp16(10 + bi, synth.STREAM_V, (hkv * lens[bi], d))
        slots = torch.from_numpy(np.concatenate([rows_of[(bi, h)] for h in range(hkv)])).to(DEV)
        cd.encode_k(k.to(DEV), slot_mapping=slots, packed=kp, norms=kn)
        tq.encode_v(v.to(DEV), vb, vg, slot_mapping=slots, data=vd, scales=vs, zeros=vz)
    q16 = synth.normal_fp16(2, synth.STREAM_Q, (b, hq, d))
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, v_group=vg,
                                 block_table=table.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV)))
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            ref = oracle_heads(cd, cache, q16.numpy(), bi, h, rows_of[(bi, h)], vb, vg, g)
            for gi in range(g):
                assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL


def test_attend_70b_class_full_size_sampled():
    # batch 1, 8 kv heads, 64 query heads, 131072 tokens, d = 128, K 3-bit, V 2-bit group 32
    _run_contiguous(1, 8, 64, 131072, 128, 3, 2, 32, check_bh=[(0, 0), (0, 5)])
    assert tq.read_device_flag() == 0


def test_attend_llama8b_layer_sampled():
    # batch 8, 8 kv heads, 32 query heads, 8192 tokens, d = 128, K 4-bit, V 2-bit group 32
    _run_contiguous(8, 8, 32, 8192, 128, 4, 2, 32, check_bh=[(0, 0), (7, 7), (3, 2)])


def test_attend_seq_lens_are_clamped_to_the_layout():
    # contiguous: a length past max_seq_len attends to all max_seq_len tokens, a negative one to none
    b, hkv, hq, t, d, kb, vb, vg = 3, 2, 8, 256, 128, 3, 2, 32
    cd, cache = build_contiguous(b, hkv, t, d, kb, vb, vg)
    q16 = synth.normal_fp16(4, synth.STREAM_Q, (b, hq, d))
    lens = torch.tensor([t + 1000, -7, 100], dtype=torch.int32, device=DEV)
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=t,
                                 seq_lens=lens))
    g = hq // hkv
    for bi, length in enumerate([t, 0, 100]):
        for h in range(hkv):
            rows = (bi * hkv + h) * t + np.arange(length)
            ref = oracle_heads(cd, cache, q16.numpy(), bi, h, rows, vb, vg, g)
            for gi in range(g):
                got = out[bi, h * g + gi]
                if length == 0:
                    assert np.all(got == 0)
                else:
                    assert rel_l2(got, ref[gi]) <= L2_RTOL
    # paged: a length past max_blocks * 16 attends to the table's max_blocks * 16 tokens; every pool row is filled
    b, max_blocks = 2, 4
    nblocks = b * max_blocks
    table = synth.block_table(5, b, max_blocks, nblocks)
    rows_total = nblocks * hkv * 16
    k = synth.normal_fp16(21, synth.STREAM_K, (rows_total, d)).to(DEV)
    v = synth.normal_fp16(21, synth.STREAM_V, (rows_total, d)).to(DEV)
    kp, kn = cd.encode_k(k)
    vd, vs, vz = tq.encode_v(v, vb, vg)
    pcache = tq.Cache(kp, kn, vd, vs, vz)
    plens = torch.tensor([10 ** 6, 17], dtype=torch.int32, device=DEV)
    q16 = synth.normal_fp16(6, synth.STREAM_Q, (b, hq, d))
    kw = dict(num_kv_heads=hkv, v_bits=vb, v_group=vg, block_table=table.to(DEV), seq_lens=plens)
    out = to_np(tq.attend_decode(cd, q16.to(DEV), pcache, **kw))
    scores = to_np(tq.attend_scores(cd, q16.to(DEV), pcache, **kw))
    for bi, length in enumerate([16 * max_blocks, 17]):
        assert np.all(np.isfinite(scores[bi, :, :length])) and np.all(scores[bi, :, length:] == -np.inf)
        for h in range(hkv):
            rows = o.paged_rows(table.numpy(), bi, h, length, hkv, 16)
            ref = oracle_heads(cd, pcache, q16.numpy(), bi, h, rows, vb, vg, g)
            for gi in range(g):
                assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL
    assert tq.read_device_flag() == 0
