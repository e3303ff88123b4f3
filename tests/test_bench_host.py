"""Host-side pieces of bench.py that need no GPU: the row chunks of the pipelined end-to-end pass."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("n", [1, 127, 128, 4096, 524288, 1048576, 1048576 + 37, 1 << 24])
@pytest.mark.parametrize("chunks", [1, 3, 8, 16])
def test_chunk_bounds_cover_the_rows_in_whole_tiles(n, chunks):
    b = _bench().chunk_bounds(n, chunks)
    assert len(b) == chunks + 1 and b[0] == 0 and b[-1] == n
    assert all(x <= y for x, y in zip(b, b[1:]))                 # empty chunks allowed, never negative
    assert all(x % 128 == 0 for x in b[:-1])                      # inner starts on whole 128-row tiles
    # every pool array's chunk starts 16-byte aligned (K payload 48 B/row at 3 bits, norms 4 B, V scales 8 B)
    for row_bytes in (16, 32, 48, 64, 4, 8, 2 * 128):
        assert all((x * row_bytes) % 16 == 0 for x in b[:-1])


def test_paged_workload_bytes_per_vector_are_the_layout_sums():
    bench = _bench()
    # high-concurrency paged cache, K 4-bit / V 4-bit group 32: per vector K 164 / 644 B, V 168 / 672 B;
    # attention 76 / 292 B per (token, kv head) at head_dim 64 / 256
    for name, k, v, att in (("paged_64x4096_d64", 164, 168, 76), ("paged_64x4096_d256", 644, 672, 292)):
        b = bench.algorithmic_bytes(bench.WORKLOADS[name])
        assert (b["encode_k"], b["encode_v"], b["attend"], b["append"]) == (k, v, att, k + v)
    # K-only round trip: 4096 x 128, 4 bits: 64 B of codes + a 4-byte norm + 256 B of fp16 per vector
    assert bench.algorithmic_bytes(bench.WORKLOADS["k_roundtrip_4096"])["encode_k"] == 324
    assert bench.algorithmic_bytes(bench.WORKLOADS["70b_decode_128k"])["attend"] == 100


def test_paged_slots_follow_the_block_table():
    import numpy as np
    import torch
    from kv_cache_vector_norm_b200 import synth
    from oracle import tq_oracle as o
    bench = _bench()
    b, hkv, t = 3, 2, 70
    per_seq = t // 16 + 1
    table = synth.block_table(1, b, per_seq, b * per_seq + 4)
    slots, new_slots = bench.paged_slots(table, hkv, t)
    s = slots.view(b, hkv, t).numpy()
    for bi in range(b):
        for h in range(hkv):
            rows = o.paged_rows(table.numpy(), bi, h, t + 1, hkv, 16)
            assert np.array_equal(s[bi, h], rows[:t])
            assert int(new_slots.view(b, hkv)[bi, h]) == rows[t]
    assert len(set(slots.tolist()) | set(new_slots.tolist())) == b * hkv * (t + 1)   # no slot written twice
