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
