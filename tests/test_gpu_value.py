"""GPU parity of the value codec (tq_encode_v / tq_decode_v through the C ABI) with the oracle:
payloads, fp16 scales and zeros bit-exact; decode bit-exact in f32 and, after round-to-nearest, in f16."""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(n, d, seed=0, scaled=True):
    x = synth.normal_fp16(seed, synth.STREAM_V, (n, d))
    if scaled:
        sc = synth.channel_scales(seed, 1, d, "v")[0]
        x = (x.float() * sc).half()
    return x


def _check(x, bits, group, layout_group):
    n, d = x.shape
    xg = x.to(DEV)
    data, sc, zr = tq.encode_v(xg, bits, layout_group)
    layout = "token" if layout_group == d else "group"
    rd, rs, rz, _ = o.encode_v(to_np(x), bits, 32, layout)
    assert np.array_equal(to_np(data), rd)
    assert np.array_equal(to_np(sc).view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(to_np(zr).view(np.uint16), rz.view(np.uint16))
    ref = o.decode_v(rd, rs, rz, bits, d, 32, layout)
    out32 = tq.decode_v(data, sc, zr, d, bits, layout_group, out_dtype=torch.float32)
    assert np.array_equal(to_np(out32).view(np.uint32), ref.view(np.uint32))
    out16 = tq.decode_v(data, sc, zr, d, bits, layout_group, out_dtype=torch.float16)
    assert np.array_equal(to_np(out16).view(np.uint16), ref.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("token", [False, True])
def test_value_codec_bit_exact(d, bits, token):
    for n in (1, 37, 2049):
        _check(_inputs(n, d, seed=n + bits), bits, 32, d if token else 32)


def test_value_edge_cases():
    d = 128
    x = torch.zeros(64, d, dtype=torch.float16)
    x[1] = 1.5                                   # constant row: scale underflows to fp16 zero
    x[2, ::2], x[2, 1::2] = -2.0, 6.0            # two-value row
    x[3] = torch.arange(d, dtype=torch.float16) * 0.5   # exact half-integer ties at 2 bits
    x[4] = 60000.0                               # large constant
    x[5, :64], x[5, 64:] = -65504.0, 65504.0     # extreme range
    x[6:] = synth.normal_fp16(9, 2, (58, d))
    for bits in (2, 3, 4, 8):
        for g in (32, d):
            _check(x, bits, 32, g)


def test_value_slot_mapping_and_stride():
    d, n = 128, 300
    x = _inputs(n, d, seed=4)
    big = torch.zeros(n, d + 40, dtype=torch.float16)
    big[:, :d] = x
    xg = big.to(DEV)[:, :d]                       # row stride d + 40 (a multiple of 8)
    perm = torch.randperm(n + 50, generator=torch.Generator().manual_seed(1))[:n]
    slots = perm.clone()
    slots[::7] = -1                                # skipped rows
    data = torch.full((n + 50, 32), 0xAB, dtype=torch.uint8, device=DEV)
    sc = torch.zeros(n + 50, 4, dtype=torch.float16, device=DEV)
    zr = torch.zeros(n + 50, 4, dtype=torch.float16, device=DEV)
    tq.encode_v(xg, 2, 32, slot_mapping=slots.to(DEV), data=data, scales=sc, zeros=zr)
    rd, rs, rz, _ = o.encode_v(to_np(x), 2)
    keep = (slots >= 0).numpy()
    dst = slots.numpy()[keep]
    assert np.array_equal(to_np(data)[dst], rd[keep])
    assert np.array_equal(to_np(sc)[dst].view(np.uint16), rs[keep].view(np.uint16))
    untouched = np.setdiff1d(np.arange(n + 50), dst)
    assert np.all(to_np(data)[untouched] == 0xAB)


def test_value_zero_rows_is_noop():
    x = torch.empty(0, 128, dtype=torch.float16, device=DEV)
    data, sc, zr = tq.encode_v(x, 2)
    assert data.shape == (0, 32)


def test_value_full_size_sampled():
    # 70B-class decode step: 1 x 8 kv heads x 131072 tokens, d = 128, V 2-bit group 32, lognormal scales
    shape = (1, 8, 131072, 128)
    sc = synth.channel_scales(0, 8, 128, "v")
    x = synth.kv_tensor(0, synth.STREAM_V, *shape, device=DEV, scales=sc).view(-1, 128)
    data, s16, z16 = tq.encode_v(x, 2, 32)
    out = tq.decode_v(data, s16, z16, 128, 2, 32, out_dtype=torch.float32)
    rows = torch.randint(0, x.shape[0], (4096,), generator=torch.Generator().manual_seed(7))
    rows[:3] = torch.tensor([0, x.shape[0] - 1, 131071])
    xr = synth.kv_rows(0, synth.STREAM_V, shape, rows, scales=sc)
    assert torch.equal(xr, x[rows.to(DEV)].cpu())
    rd, rs, rz, _ = o.encode_v(xr.numpy(), 2)
    assert np.array_equal(to_np(data[rows.to(DEV)]), rd)
    assert np.array_equal(to_np(s16[rows.to(DEV)]).view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(to_np(z16[rows.to(DEV)]).view(np.uint16), rz.view(np.uint16))
    ref = o.decode_v(rd, rs, rz, 2, 128)
    assert np.array_equal(to_np(out[rows.to(DEV)]).view(np.uint32), ref.view(np.uint32))
