"""GPU parity of QJL residual keys (tq_codec_create_qjl / tq_encode_k_qjl through the C ABI) with the fp64 oracle.

The MSE stage follows the key-codec rules (indices bit-exact except in-band neighbour flips, norms within 1e-6
relative).  The residual is taken from the GPU's own indices and norms: rho within 1e-5 relative; sign bits
exact except where the oracle's projection (S_op r)_i lies within 1e-5 * ||S_op row i|| * ||x|| of zero, and
such flips fewer than 1e-4 of all bits."""
import ctypes

import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, NORM_RTOL, check_key_indices, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
RHO_RTOL = 1e-5
SIGN_BAND = 1e-5
_CODECS = {}


def qcodec(d, bits, seed=0):
    key = (d, bits, seed)
    if key not in _CODECS:
        _CODECS[key] = tq.QjlCodec(d, bits, seed)
    return _CODECS[key]


def _check_residual(x16: np.ndarray, d, bits, packed, norms, signs, rho, seed=0):
    """Check the GPU's QJL output for fp16 rows x16 against the oracle; returns the sign-flip count."""
    mb = o.qjl_mse_bits(bits)
    pi, c, t = params(d, mb, seed)
    s_op = o.operational_qjl_matrix(d, seed)
    ref_idx, ref_n, y = o.encode_k(x16, pi, t)
    gidx = o.unpack_lsb(packed, mb, d)
    check_key_indices(gidx, ref_idx, y, t)
    nz = ref_n > 0
    assert np.all(np.abs(norms[nz] - ref_n[nz]) <= NORM_RTOL * ref_n[nz])
    _, _, _, ref_bits, ref_rho, proj = o.encode_k_qjl(x16, pi, c, t, s_op, idx=gidx)
    assert np.all(np.abs(rho - ref_rho) <= RHO_RTOL * np.maximum(ref_rho, 1e-30) + 1e-30)
    gbits = o.unpack_lsb(signs, 1, d).astype(bool)
    diff = gbits != ref_bits
    band = SIGN_BAND * np.linalg.norm(s_op, axis=1)[None, :] * np.linalg.norm(x16.astype(np.float64), axis=1)[:, None]
    assert np.all(np.abs(proj[diff]) < band[diff]), np.abs(proj[diff]).max() if diff.any() else 0
    assert diff.sum() <= 1e-4 * diff.size + 1, (int(diff.sum()), diff.size)
    return int(diff.sum())


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_qjl_encode_parity(d, bits):
    cd = qcodec(d, bits)
    for n in (1, 37, 1000):
        x = synth.normal_fp16(n + 31 * bits, synth.STREAM_K, (n, d))
        packed, norms, signs, rho = cd.encode_k_qjl(x.to(DEV))
        _check_residual(x.numpy(), d, bits, to_np(packed), to_np(norms), to_np(signs), to_np(rho))


def test_qjl_mse_stage_is_the_key_codec_at_one_bit_less():
    d, bits = 128, 4
    x = synth.normal_fp16(3, synth.STREAM_K, (777, d)).to(DEV)
    qp, qn, _, _ = qcodec(d, bits).encode_k_qjl(x)
    kp, kn = tq.Codec(d, bits - 1, 0).encode_k(x)
    assert torch.equal(qp, kp) and torch.equal(qn, kn)
    v = ctypes.c_int()
    assert tq.LIB.tq_codec_qjl_bits(qcodec(d, bits).handle, ctypes.byref(v)) == 0 and v.value == bits
    assert tq.LIB.tq_codec_qjl_bits(tq.Codec(d, 3, 0).handle, ctypes.byref(v)) == 0 and v.value == 0


def test_qjl_slot_mapped_scatter_and_edge_rows():
    # a permuted slot mapping with skipped rows (-1), zero and extreme rows among them
    d, bits, n, pool = 128, 3, 300, 512
    x = synth.normal_fp16(9, synth.STREAM_K, (n, d))
    x[0] = 0
    x[1, 5] = 60000.0
    x[2] = 1e-4
    slots = torch.randperm(pool, generator=torch.Generator().manual_seed(4))[:n].to(torch.int64)
    slots[7] = -1
    cd = qcodec(d, bits)
    packed = torch.full((pool, d * (bits - 1) // 8), 0xAB, dtype=torch.uint8, device=DEV)
    norms = torch.full((pool,), -1.0, device=DEV)
    signs = torch.full((pool, d // 8), 0xCD, dtype=torch.uint8, device=DEV)
    rho = torch.full((pool,), -2.0, device=DEV)
    cd.encode_k_qjl(x.to(DEV), slot_mapping=slots.to(DEV), packed=packed, norms=norms, signs=signs, rho=rho)
    keep = slots >= 0
    rows = slots[keep].numpy()
    _check_residual(x.numpy()[keep.numpy()], d, bits, to_np(packed)[rows], to_np(norms)[rows], to_np(signs)[rows],
                    to_np(rho)[rows])
    untouched = np.setdiff1d(np.arange(pool), rows)
    assert np.all(to_np(signs)[untouched] == 0xCD) and np.all(to_np(rho)[untouched] == -2.0)
    assert tq.read_device_flag() == 0


def test_qjl_rejects_a_plain_codec():
    x = torch.zeros(4, 128, dtype=torch.float16, device=DEV)
    plain = tq.Codec(128, 3, 0)
    with pytest.raises(tq.TQError, match="tq_codec_create_qjl"):
        tq.QjlCodec.encode_k_qjl(plain, x)
    with pytest.raises(tq.TQError):
        tq.QjlCodec(128, 6, 0)


# ------------------------------------------------------------------------------------------ attention

def _qjl_cache(b, hkv, t, d, bits, vb, seed=0):
    cd = qcodec(d, bits, seed)
    ks = synth.channel_scales(seed, hkv, d, "k")
    vs = synth.channel_scales(seed, hkv, d, "v")
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=DEV, scales=ks).view(-1, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=DEV, scales=vs).view(-1, d)
    kp, kn, sg, rh = cd.encode_k_qjl(k)
    vd, vsc, vz = tq.encode_v(v, vb, 32)
    return cd, tq.Cache(kp, kn, vd, vsc, vz), sg, rh


def _oracle_qjl(cd, cache, sg, rh, q16, bi, h, rows, vb, g):
    d, mb = cd.d, cd.bits
    pi, c, _ = params(d, mb, cd.seed)
    s_op = o.operational_qjl_matrix(d, cd.seed)
    r = torch.as_tensor(np.asarray(rows), device=DEV)
    idx = o.unpack_lsb(to_np(cache.k_packed[r]), mb, d)
    nrm = to_np(cache.k_norms[r]).astype(np.float64)
    bits = o.unpack_lsb(to_np(sg[r]), 1, d).astype(bool)
    rho = to_np(rh[r]).astype(np.float64)
    vh = o.decode_v(to_np(cache.v_data[r]), to_np(cache.v_scales[r]), to_np(cache.v_zeros[r]), vb, d, 32, "group")
    qs = q16[bi:bi + 1, h * g:(h + 1) * g]
    return o.attend_qjl(qs, idx[None, None], nrm[None, None], bits[None, None], rho[None, None], vh[None, None],
                        pi, c, s_op)[0]


@pytest.mark.parametrize("d,bits,vb", [(128, 4, 2), (128, 3, 4), (64, 2, 2), (256, 5, 4), (128, 5, 2)])
def test_qjl_attention_contiguous(d, bits, vb):
    b, hkv, hq, t = 2, 2, 8, 320
    cd, cache, sg, rh = _qjl_cache(b, hkv, t, d, bits, vb)
    q16 = synth.normal_fp16(7, synth.STREAM_Q, (b, hq, d))
    lens = [320, 157]
    out = to_np(tq.attend_decode_qjl(cd, q16.to(DEV), cache, sg, rh, num_kv_heads=hkv, v_bits=vb, max_seq_len=t,
                                     seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV)))
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            rows = (bi * hkv + h) * t + np.arange(lens[bi])
            ref = _oracle_qjl(cd, cache, sg, rh, q16.numpy(), bi, h, rows, vb, g)
            for gi in range(g):
                assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL, (bi, h, gi, rel_l2(out[bi, h * g + gi], ref[gi]))


def test_qjl_attention_split_k_long_sequence_and_differs_from_mse_only():
    # one long sequence over many splits; the estimator's second term changes the result
    b, hkv, hq, t, d, bits, vb = 1, 1, 8, 8192, 128, 4, 2
    cd, cache, sg, rh = _qjl_cache(b, hkv, t, d, bits, vb, seed=1)
    q16 = synth.normal_fp16(8, synth.STREAM_Q, (b, hq, d))
    out = to_np(tq.attend_decode_qjl(cd, q16.to(DEV), cache, sg, rh, num_kv_heads=hkv, v_bits=vb, max_seq_len=t))
    ref = _oracle_qjl(cd, cache, sg, rh, q16.numpy(), 0, 0, np.arange(t), vb, hq)
    for gi in range(hq):
        assert rel_l2(out[0, gi], ref[gi]) <= L2_RTOL
    mse_only = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, max_seq_len=t))
    assert rel_l2(mse_only, out) > 10 * L2_RTOL
    assert tq.read_device_flag() == 0


def test_qjl_attention_paged():
    b, hkv, hq, d, bits, vb = 3, 2, 8, 128, 3, 4
    lens = [16 * 5, 33, 1]
    max_blocks = 5
    nblocks = b * max_blocks + 3
    table = synth.block_table(4, b, max_blocks, nblocks)
    cd = qcodec(d, bits)
    rows_total = nblocks * hkv * 16
    kp = torch.zeros(rows_total, cd.row_bytes, dtype=torch.uint8, device=DEV)
    kn = torch.zeros(rows_total, device=DEV)
    sg = torch.zeros(rows_total, d // 8, dtype=torch.uint8, device=DEV)
    rh = torch.zeros(rows_total, device=DEV)
    vd = torch.zeros(rows_total, d * vb // 8, dtype=torch.uint8, device=DEV)
    vs = torch.zeros(rows_total, d // 32, dtype=torch.float16, device=DEV)
    vz = torch.zeros_like(vs)
    cache = tq.Cache(kp, kn, vd, vs, vz)
    rows_of = {}
    for bi in range(b):
        for h in range(hkv):
            rows_of[(bi, h)] = o.paged_rows(table.numpy(), bi, h, lens[bi], hkv, 16)
        k = synth.normal_fp16(20 + bi, synth.STREAM_K, (hkv * lens[bi], d))
        v = synth.normal_fp16(20 + bi, synth.STREAM_V, (hkv * lens[bi], d))
        slots = torch.from_numpy(np.concatenate([rows_of[(bi, h)] for h in range(hkv)])).to(DEV)
        cd.encode_k_qjl(k.to(DEV), slot_mapping=slots, packed=kp, norms=kn, signs=sg, rho=rh)
        tq.encode_v(v.to(DEV), vb, 32, slot_mapping=slots, data=vd, scales=vs, zeros=vz)
    q16 = synth.normal_fp16(5, synth.STREAM_Q, (b, hq, d))
    out = to_np(tq.attend_decode_qjl(cd, q16.to(DEV), cache, sg, rh, num_kv_heads=hkv, v_bits=vb,
                                     block_table=table.to(DEV),
                                     seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV)))
    g = hq // hkv
    for bi in range(b):
        for h in range(hkv):
            ref = _oracle_qjl(cd, cache, sg, rh, q16.numpy(), bi, h, rows_of[(bi, h)], vb, g)
            for gi in range(g):
                assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL


def test_qjl_attention_argument_errors():
    cd, cache, sg, rh = _qjl_cache(1, 1, 32, 128, 3, 2)
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device=DEV)
    with pytest.raises(tq.TQError, match="tq_codec_create_qjl"):
        tq.attend_decode_qjl(tq.Codec(128, 2, 0), q, cache, sg, rh, num_kv_heads=1, v_bits=2, max_seq_len=32)
    with pytest.raises(tq.TQError, match="supported: 2 or 4 bits"):
        tq.attend_decode_qjl(cd, q, cache, sg, rh, num_kv_heads=1, v_bits=3, max_seq_len=32)
