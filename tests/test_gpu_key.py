"""GPU parity of the key codec (tq_encode_k / tq_decode_k through the C ABI) with the fp64 oracle.

Indices bit-exact except in-band neighbour flips (< 1e-4 of coordinates); norms within 1e-6 relative;
decode within 1e-3 relative L2 of the oracle's decode of the GPU's own indices and norms."""
import ctypes
import math

import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import L2_RTOL, NORM_RTOL, check_key_indices, params, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
_CODECS = {}


def codec(d, bits, seed=0):
    key = (d, bits, seed)
    if key not in _CODECS:
        _CODECS[key] = tq.Codec(d, bits, seed)
    return _CODECS[key]


def _roundtrip(x16: torch.Tensor, d, bits, seed=0, out_dtype=torch.float16):
    cd = codec(d, bits, seed)
    packed, norms = cd.encode_k(x16.to(DEV))
    out = cd.decode_k(packed, norms, out_dtype=out_dtype)
    return to_np(packed), to_np(norms), to_np(out)


def _check(x16: torch.Tensor, d, bits, seed=0, out_dtype=torch.float16):
    pi, c, t = params(d, bits, seed)
    packed, norms, out = _roundtrip(x16, d, bits, seed, out_dtype)
    ref_idx, ref_n, y = o.encode_k(x16.numpy(), pi, t)
    gidx = o.unpack_lsb(packed, bits, d)
    check_key_indices(gidx, ref_idx, y, t)
    nz = ref_n > 0
    assert np.all(np.abs(norms[nz] - ref_n[nz]) <= NORM_RTOL * ref_n[nz])
    assert np.all(norms[~nz] == 0)
    ref_dec = o.decode_k(gidx, norms.astype(np.float64), pi, c)
    for r in range(0, len(out), max(1, len(out) // 64)):
        if ref_n[r] > 0:
            assert rel_l2(out[r], ref_dec[r]) <= L2_RTOL
    assert rel_l2(out, ref_dec) <= L2_RTOL
    return gidx, norms, out


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_key_codec_parity(d, bits):
    for n in (1, 129, 1000):
        x = synth.normal_fp16(n + 17 * bits, synth.STREAM_K, (n, d))
        _check(x, d, bits)


def test_key_round_trip_k_only_config():
    # K-only round trip: 4096 fp16 N(0,1) vectors, d = 128, 4 bits, seed 0 (64 B + f32 norm per vector)
    d, bits = 128, 4
    x = synth.normal_fp16(0, synth.STREAM_K, (4096, d))
    gidx, norms, out = _check(x, d, bits, out_dtype=torch.float32)
    pi, c, t = params(d, bits, 0)
    xf = x.double().numpy()
    rel = np.sum((out - xf) ** 2, axis=1) / np.sum(xf * xf, axis=1)
    D = o.sphere_distortion(d, c, t)
    assert abs(rel.mean() - D) < 4 * rel.std() / math.sqrt(len(rel)) + 2e-4 * D
    lo, hi = o.distortion_bounds(bits)
    assert lo <= rel.mean() <= hi


def test_key_edge_cases_and_layouts():
    d, bits = 128, 3
    x = synth.normal_fp16(3, synth.STREAM_K, (300, d))
    x[0] = 0.0                                     # zero vector -> middle index, norm 0
    x[1] = 0.0
    x[1, 5] = 1.0                                  # a basis vector
    x[2] = 4000.0                                  # large entries: sum of squares far above fp16 range
    x[3] = 1e-4                                    # subnormal-scale entries
    _check(x, d, bits)
    # slot mapping with skipped rows and a strided input
    cd = codec(d, bits)
    big = torch.zeros(300, d + 24, dtype=torch.float16)
    big[:, :d] = x
    slots = torch.randperm(400, generator=torch.Generator().manual_seed(2))[:300]
    slots[::5] = -1
    packed = torch.full((400, cd.row_bytes), 0x5A, dtype=torch.uint8, device=DEV)
    norms = torch.full((400,), -1.0, device=DEV)
    cd.encode_k(big.to(DEV)[:, :d], slot_mapping=slots.to(DEV), packed=packed, norms=norms)
    ref_p, ref_n = cd.encode_k(x.to(DEV))
    keep = slots >= 0
    dst = slots[keep].to(DEV)
    assert torch.equal(packed[dst], ref_p[keep.to(DEV)])
    assert torch.equal(norms[dst], ref_n[keep.to(DEV)])
    untouched = torch.ones(400, dtype=torch.bool)
    untouched[slots[keep]] = False
    assert bool((packed[untouched.to(DEV)] == 0x5A).all()) and bool((norms[untouched.to(DEV)] == -1).all())


def test_key_full_size_sampled():
    # 70B-class cache: 1 x 8 kv heads x 131072 tokens, d = 128, K 3-bit, lognormal channel scales
    shape = (1, 8, 131072, 128)
    sc = synth.channel_scales(0, 8, 128, "k")
    x = synth.kv_tensor(0, synth.STREAM_K, *shape, device=DEV, scales=sc).view(-1, 128)
    cd = codec(128, 3)
    packed, norms = cd.encode_k(x)
    out = cd.decode_k(packed, norms)
    rows = torch.randint(0, x.shape[0], (8192,), generator=torch.Generator().manual_seed(3))
    rows[:2] = torch.tensor([0, x.shape[0] - 1])
    xr = synth.kv_rows(0, synth.STREAM_K, shape, rows, scales=sc)
    assert torch.equal(xr, x[rows.to(DEV)].cpu())
    pi, c, t = params(128, 3, 0)
    ref_idx, ref_n, y = o.encode_k(xr.numpy(), pi, t)
    gidx = o.unpack_lsb(to_np(packed[rows.to(DEV)]), 3, 128)
    check_key_indices(gidx, ref_idx, y, t)
    gn = to_np(norms[rows.to(DEV)])
    assert np.all(np.abs(gn - ref_n) <= NORM_RTOL * ref_n)
    ref_dec = o.decode_k(gidx, gn.astype(np.float64), pi, c)
    assert rel_l2(to_np(out[rows.to(DEV)]), ref_dec) <= L2_RTOL
    assert tq.read_device_flag() == 0


_DB_ALL = [(d, b) for d in (64, 128, 256) for b in range(1, 9) if b <= 4 or d <= 128]


@pytest.mark.parametrize("d,bits", _DB_ALL)
def test_key_decode_many_tiles_per_cta(d, bits):
    """Six 128-row tiles per CTA plus a ragged tail, decoded right after a decode of random codes of the same
    shape: a staging buffer refilled before every read of it had completed, or stale shared memory left by the
    previous launch, shows up as wrong rows.  Every row is checked against the oracle's decode of the GPU's
    own indices and norms."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = sms * 128 * 6 + 77
    cd = codec(d, bits)
    pi, c, t = params(d, bits, 0)
    x = synth.normal_fp16(900 + bits, synth.STREAM_K, (n, d), device=DEV)
    packed, norms = cd.encode_k(x)
    noise = torch.randint(0, 256, tuple(packed.shape), dtype=torch.uint8,
                          generator=torch.Generator().manual_seed(bits)).to(DEV)
    cd.decode_k(noise, norms, out_dtype=torch.float32)
    for out_dtype in (torch.float32, torch.float16):
        out = to_np(cd.decode_k(packed, norms, out_dtype=out_dtype)).astype(np.float64)
        ref = o.decode_k(o.unpack_lsb(to_np(packed), bits, d), to_np(norms).astype(np.float64), pi, c)
        err = np.linalg.norm(out - ref, axis=1)
        bad = np.nonzero(err > L2_RTOL * np.linalg.norm(ref, axis=1))[0]
        assert bad.size == 0, f"{bad.size} rows off, first {bad[:8].tolist()}"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 4])
def test_key_codec_parity_hadamard_rotation(d, bits):
    # the randomized Walsh-Hadamard rotation ("turbo-attn", The codec) through the same tensor-core kernels
    cd = tq.Codec(d, bits, 3, rotation="hadamard")
    pi, c, t = params(d, bits, 3, "hadamard")
    for n in (1, 300, 4097):
        x16 = synth.normal_fp16(n + bits, synth.STREAM_K, (n, d))
        packed, norms = cd.encode_k(x16.to(DEV))
        out = cd.decode_k(packed, norms)
        ref_idx, ref_n, y = o.encode_k(x16.numpy(), pi, t)
        gidx = o.unpack_lsb(to_np(packed), bits, d)
        check_key_indices(gidx, ref_idx, y, t)
        gn = to_np(norms)
        assert np.all(np.abs(gn - ref_n) <= NORM_RTOL * ref_n)
        assert rel_l2(to_np(out), o.decode_k(gidx, gn.astype(np.float64), pi, c)) <= L2_RTOL
    rot = ctypes.c_int(-1)
    assert tq.LIB.tq_codec_rotation(cd.handle, ctypes.byref(rot)) == tq.TQ_OK and rot.value == tq.TQ_ROT_HADAMARD
