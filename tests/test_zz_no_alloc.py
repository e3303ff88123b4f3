"""The allocation-free attention entry point (tq_attend_decode_noalloc), for callers that cannot allocate
device memory -- work captured into or replayed from a CUDA graph, or a server whose memory pool is fixed
at start-up.  It must give the same attention output as tq_attend_decode with a caller workspace, on two
calls in a row (the second reuses the library's scratch as the first left it), and it must refuse a
launch whose split-K partials do not fit in that fixed scratch.  This file is collected last so that a
failure here does not hide the other tests' results."""
import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from _tqh import L2_RTOL, rel_l2, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _cache(b, hkv, t, d=128, kb=3, vb=2, seed=0):
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=DEV).view(-1, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=DEV).view(-1, d)
    cd = tq.Codec(d, kb, seed)
    kp, kn = cd.encode_k(k)
    vd, vs, vz = tq.encode_v(v, vb, 32)
    return cd, tq.Cache(kp, kn, vd, vs, vz)


def test_noalloc_matches_workspace_entry_point_twice():
    b, hkv, hq, t = 2, 2, 16, 8192                     # long sequences: split-K partials go to the scratch
    cd, cache = _cache(b, hkv, t)
    q = synth.normal_fp16(5, synth.STREAM_Q, (b, hq, 128)).to(DEV)
    kw = dict(num_kv_heads=hkv, v_bits=2, v_group=32, max_seq_len=t)
    assert tq.attend_workspace_bytes(cd, q, cache, block_table=None, seq_lens=None, scale=0.0, **kw) > 0
    ref = to_np(tq.attend_decode(cd, q, cache, **kw))
    out = torch.empty(b, hq, 128, dtype=torch.float32, device=DEV)
    for _ in range(2):
        out.fill_(float("nan"))
        got = to_np(tq.attend_decode_noalloc(cd, q, cache, out=out, **kw))
        for bi in range(b):
            for h in range(hq):
                assert rel_l2(got[bi, h], ref[bi, h]) <= L2_RTOL
    assert tq.read_device_flag() == 0


def test_noalloc_rejects_launches_beyond_its_scratch():
    # A head_dim-256 shape whose split-K partials do not fit in the fixed scratch.  The cache is paged and every
    # block-table entry names its one block, so every row such a launch could read exists: if the size check
    # ever stopped refusing, the launch would read valid memory and the test would fail on the missing error.
    cd, cache = _cache(1, 1, 16, d=256, kb=4, vb=4)
    max_blocks = 256                                   # 4096 tokens per sequence
    for bh in range(150, 1200, 10):
        q = torch.zeros(bh, 4, 256, dtype=torch.float16, device=DEV)
        table = torch.zeros(bh, max_blocks, dtype=torch.int32, device=DEV)
        lens = torch.full((bh,), 16 * max_blocks, dtype=torch.int32, device=DEV)
        kw = dict(num_kv_heads=1, v_bits=4, v_group=32, block_table=table, seq_lens=lens, scale=0.0)
        need = tq.attend_workspace_bytes(cd, q, cache, max_seq_len=None, **kw)
        if need > tq.ATTEND_SCRATCH_BYTES:
            break
    else:
        pytest.skip("no shape on this device needs more split-K scratch than the fixed array holds")
    with pytest.raises(tq.TQError, match="static scratch"):
        tq.attend_decode_noalloc(cd, q, cache, out=torch.empty(bh, 4, 256, device=DEV), **kw)
    torch.cuda.synchronize()
