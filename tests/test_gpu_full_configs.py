"""GPU parity at the full sizes of two workloads, on sampled outputs the oracle computes row by row, plus
properties that hold at any size:

* bit-width sweep: 2^24 vectors, head_dim 128, fp16 N(0,1); key bits 1..4 and value bits 2/3/4/8 with group-32
  and per-token scales.  Sampled rows are checked against the oracle (key indices within the flip band,
  norms, decode; value payload, scales, zeros and decode bit-exact); over all 2^24 vectors the measured
  mean distortion ||x - x_hat||^2 / ||x||^2 must match the codebook's D(b, d) ("TurboQuant" paper,
  distortion theorem: the rotated coordinate follows the sphere marginal, so the per-vector error is
  d times the scalar quantizer's error under it).
* high-concurrency paged cache: 64 sequences x 4096 tokens, 8 kv heads, head_dim 64 and 256, blocks of 16
  tokens in a seeded random block table, K 4-bit / V 4-bit appended through the slot mapping, then one
  decode step of attention for 32 query heads; sampled (sequence, kv head) pairs against the oracle.
"""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, NORM_RTOL, check_key_indices, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _mean_rel_sq_error(x: torch.Tensor, xh: torch.Tensor, chunk: int = 1 << 20) -> float:
    """mean over rows of ||x - x_hat||^2 / ||x||^2, accumulated in fp64 on the device."""
    tot = torch.zeros((), dtype=torch.float64, device=x.device)
    for i in range(0, x.shape[0], chunk):
        a = x[i:i + chunk].float()
        e = (a - xh[i:i + chunk].float()).square().sum(1).double()
        tot += (e / a.square().sum(1).double()).sum()
    return float(tot) / x.shape[0]


def test_bit_sweep_full_size_sampled():
    n, d = 1 << 24, 128
    x = synth.normal_fp16(0, synth.STREAM_K, (n, d), device=DEV)
    rows = torch.randint(0, n, (2048,), generator=torch.Generator().manual_seed(11))
    rows[:2] = torch.tensor([0, n - 1])
    rd = rows.to(DEV)
    xr = x[rd].cpu()
    for kb in (1, 2, 3, 4):
        cd = tq.Codec(d, kb, 0)
        packed, norms = cd.encode_k(x)
        out = cd.decode_k(packed, norms)
        pi, c, t = params(d, kb, 0)
        ref_idx, ref_n, y = o.encode_k(xr.numpy(), pi, t)
        gidx = o.unpack_lsb(to_np(packed[rd]), kb, d)
        check_key_indices(gidx, ref_idx, y, t)
        gn = to_np(norms[rd])
        assert np.all(np.abs(gn - ref_n) <= NORM_RTOL * ref_n)
        assert rel_l2(to_np(out[rd]), o.decode_k(gidx, gn.astype(np.float64), pi, c)) <= L2_RTOL
        # over all 2^24 vectors: mean relative squared error = D(b, d) of the operational codebook.  The
        # Monte-Carlo error at this n is ~1e-3 relative; the fp16 rotation's deviation from orthogonality
        # and the fp16 output add well under 1%.
        dist = o.sphere_distortion(d, c, t)
        measured = _mean_rel_sq_error(x, out)
        assert abs(measured - dist) <= 0.02 * dist, (kb, measured, dist)
        lo, hi = o.distortion_bounds(kb)
        assert measured <= hi
        del packed, norms, out
    for vb in (2, 3, 4, 8):
        for token in (False, True):
            vg = d if token else 32
            layout = "token" if token else "group"
            data, s16, z16 = tq.encode_v(x, vb, vg)
            out = tq.decode_v(data, s16, z16, d, vb, vg, out_dtype=torch.float16)
            rdat, rs, rz, _ = o.encode_v(xr.numpy(), vb, 32, layout)
            assert np.array_equal(to_np(data[rd]), rdat), (vb, token)
            assert np.array_equal(to_np(s16[rd]).view(np.uint16), rs.view(np.uint16))
            assert np.array_equal(to_np(z16[rd]).view(np.uint16), rz.view(np.uint16))
            ref = o.decode_v(rdat, rs, rz, vb, d, 32, layout)
            assert np.array_equal(to_np(out[rd]).view(np.uint16), ref.astype(np.float16).view(np.uint16))
            del data, s16, z16, out
    assert tq.read_device_flag() == 0


@pytest.mark.parametrize("d", [64, 256])
def test_paged_high_concurrency_full_size_sampled(d):
    b, hkv, hq, t, kb, vb, vg = 64, 8, 32, 4096, 4, 4, 32
    bs = 16
    max_blocks = t // bs
    nblocks = b * max_blocks + 64                     # spare blocks the table never points to
    table = synth.block_table(5, b, max_blocks, nblocks)
    cd = tq.Codec(d, kb, 0)
    rows_total = nblocks * hkv * bs
    kp = torch.zeros(rows_total, cd.row_bytes, dtype=torch.uint8, device=DEV)
    kn = torch.zeros(rows_total, device=DEV)
    vd = torch.zeros(rows_total, d * vb // 8, dtype=torch.uint8, device=DEV)
    vs = torch.zeros(rows_total, d // vg, dtype=torch.float16, device=DEV)
    vz = torch.zeros_like(vs)
    cache = tq.Cache(kp, kn, vd, vs, vz)
    # every sequence's tokens are appended through the slot mapping: token t of (sequence bi, kv head h) goes to
    # pool row (table[bi][t // 16] * H_kv + h) * 16 + t % 16
    tab = table.to(DEV).long()
    tok = torch.arange(t, device=DEV)
    ks = synth.channel_scales(1, hkv, d, "k")
    vsc = synth.channel_scales(1, hkv, d, "v")
    for bi in range(b):
        k = synth.kv_tensor(100 + bi, synth.STREAM_K, 1, hkv, t, d, device=DEV, scales=ks).view(hkv * t, d)
        v = synth.kv_tensor(100 + bi, synth.STREAM_V, 1, hkv, t, d, device=DEV, scales=vsc).view(hkv * t, d)
        h = torch.arange(hkv, device=DEV)[:, None]
        slots = ((tab[bi][tok // bs][None, :] * hkv + h) * bs + (tok % bs)[None, :]).reshape(-1)
        cd.encode_k(k, slot_mapping=slots, packed=kp, norms=kn)
        tq.encode_v(v, vb, vg, slot_mapping=slots, data=vd, scales=vs, zeros=vz)
    lens = torch.full((b,), t, dtype=torch.int32)
    q16 = synth.normal_fp16(4, synth.STREAM_Q, (b, hq, d))
    out = to_np(tq.attend_decode(cd, q16.to(DEV), cache, num_kv_heads=hkv, v_bits=vb, v_group=vg,
                                 block_table=table.to(DEV), seq_lens=lens.to(DEV)))
    g = hq // hkv
    pi, c, tb = params(d, kb, 0)
    for bi, h in [(0, 0), (63, 7), (17, 3)]:
        rows = o.paged_rows(table.numpy(), bi, h, t, hkv, bs)
        r = torch.as_tensor(rows, device=DEV)
        # the appended payload is the codec's encode of the generated tokens, read back from the pool rows
        k_rows = synth.kv_tensor(100 + bi, synth.STREAM_K, 1, hkv, t, d, device=DEV, scales=ks).view(hkv, t, d)[h]
        ref_idx, ref_n, y = o.encode_k(k_rows[:512].cpu().numpy(), pi, tb)
        check_key_indices(o.unpack_lsb(to_np(kp[r[:512]]), kb, d), ref_idx, y, tb)
        assert np.all(np.abs(to_np(kn[r[:512]]) - ref_n) <= NORM_RTOL * ref_n)
        idx = o.unpack_lsb(to_np(kp[r]), kb, d)
        nrm = to_np(kn[r]).astype(np.float64)
        vh = o.decode_v(to_np(vd[r]), to_np(vs[r]), to_np(vz[r]), vb, d, 32, "group")
        ref = o.attend(q16.numpy()[bi:bi + 1, h * g:(h + 1) * g], idx[None, None], nrm[None, None], vh[None, None],
                       pi, c)[0]
        for gi in range(g):
            assert rel_l2(out[bi, h * g + gi], ref[gi]) <= L2_RTOL, (bi, h, gi)
    assert tq.read_device_flag() == 0
