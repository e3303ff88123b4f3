"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds none of the codec's arithmetic: it only draws numbers.  Both the CUDA path (bench,
tests) and the oracle (tests) take their inputs from here, and the same call gives bit-identical
values on the CPU and on a CUDA device, for the whole tensor or any subset of rows:

* every element's 64-bit random word is output number (flat index) of SplitMix64 whose state is seeded
  with mix(seed * golden + stream) -- integer arithmetic only;
* an fp16 standard normal is read off that word by an exact inverse-CDF table: the top 40 bits are
  compared with round(2^40 * Phi(m)) at the midpoints m between consecutive fp16 values (|x| <= 8), so
  the value equals fp16(Z) for Z ~ N(0, 1) up to a 2^-40 probability error;
* per-channel scales are lognormal(0, 1) drawn per (kv head, channel), with round(0.01 d) (at least
  one) outlier channels per kv head multiplied by 20, chosen without replacement; the product with the
  normal is taken in fp32 and rounded to fp16.

Streams: K=1, V=2, Q=3, K scales=4, K outliers=5, block table=6, V scales=7, V outliers=8.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from scipy import special

STREAM_K, STREAM_V, STREAM_Q = 1, 2, 3
STREAM_K_SCALE, STREAM_K_OUTLIER, STREAM_BLOCKS, STREAM_V_SCALE, STREAM_V_OUTLIER = 4, 5, 6, 7, 8

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1


def _signed(v: int) -> int:
    v &= _MASK
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def stream_state(seed: int, stream: int) -> int:
    return _mix_int(seed * _GOLDEN + stream)


def _srl(x: torch.Tensor, k: int) -> torch.Tensor:
    return (x >> k) & ((1 << (64 - k)) - 1)


def random_words(seed: int, stream: int, index: torch.Tensor) -> torch.Tensor:
    """64-bit words (as int64) for the given flat element indices (int64 tensor, any device)."""
    z = index.to(torch.int64) + 1
    z = z * _signed(_GOLDEN) + _signed(stream_state(seed, stream))
    z = (z ^ _srl(z, 30)) * _signed(_M1)
    z = (z ^ _srl(z, 27)) * _signed(_M2)
    return z ^ _srl(z, 31)


_TABLE = {}


def _normal_table(device):
    key = str(device)
    if key not in _TABLE:
        pos = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
        pos = pos[pos <= 8.0]
        vals = np.concatenate([-pos[::-1], pos[1:]])
        mids = 0.5 * (vals[:-1] + vals[1:])
        thr = np.floor(special.ndtr(mids) * 2.0 ** 40).astype(np.int64)
        _TABLE[key] = (torch.from_numpy(vals.astype(np.float16)).to(device), torch.from_numpy(thr).to(device))
    return _TABLE[key]


def normal_fp16_at(seed: int, stream: int, index: torch.Tensor) -> torch.Tensor:
    """fp16 N(0, 1) draws for the given flat indices."""
    vals, thr = _normal_table(index.device)
    u = _srl(random_words(seed, stream, index), 24)
    return vals[torch.searchsorted(thr, u, right=True)]


def normal_fp16(seed: int, stream: int, shape, device="cpu", chunk: int = 1 << 24) -> torch.Tensor:
    """A whole fp16 N(0, 1) tensor of `shape` (element counter = row-major flat index)."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.float16, device=device)
    for s in range(0, n, chunk):
        idx = torch.arange(s, min(n, s + chunk), dtype=torch.int64, device=device)
        out[s:s + idx.numel()] = normal_fp16_at(seed, stream, idx)
    return out.view(*shape)


def uniform01(seed: int, stream: int, count: int) -> np.ndarray:
    """float64 uniforms in (0, 1) from the top 53 bits (host side, small counts)."""
    w = random_words(seed, stream, torch.arange(count, dtype=torch.int64)).numpy().view(np.uint64)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def channel_scales(seed: int, num_kv_heads: int, d: int, which: str = "k", outlier_frac: float = 0.01,
                   outlier_mult: float = 20.0) -> torch.Tensor:
    """fp32 [H_kv, d]: lognormal(0, 1) per (kv head, channel); round(outlier_frac * d) channels per kv head
    (at least one when outlier_frac > 0, none when it is 0) are multiplied by outlier_mult."""
    s_stream, o_stream = (STREAM_K_SCALE, STREAM_K_OUTLIER) if which == "k" else (STREAM_V_SCALE, STREAM_V_OUTLIER)
    u1 = uniform01(seed, s_stream, num_kv_heads * d)
    u2 = uniform01(seed + 1, s_stream, num_kv_heads * d)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    scales = np.exp(z).reshape(num_kv_heads, d)
    n_out = max(1, int(round(outlier_frac * d))) if outlier_frac > 0 else 0
    for h in range(num_kv_heads):
        keys = random_words(seed, o_stream, torch.arange(h * d, (h + 1) * d, dtype=torch.int64))
        chosen = torch.argsort(keys, stable=True)[:n_out].numpy()
        scales[h, chosen] *= outlier_mult
    return torch.from_numpy(scales.astype(np.float32))


def kv_tensor(seed: int, stream: int, batch: int, num_kv_heads: int, tokens: int, d: int, device="cpu",
              scales: torch.Tensor | None = None) -> torch.Tensor:
    """fp16 [B, H_kv, T, d]: N(0, 1), optionally times per-(kv head, channel) fp32 scales (rounded once)."""
    x = normal_fp16(seed, stream, (batch, num_kv_heads, tokens, d), device)
    if scales is not None:
        x = (x.float() * scales.to(device)[None, :, None, :]).half()
    return x


def kv_rows(seed: int, stream: int, shape, rows: torch.Tensor, scales: torch.Tensor | None = None) -> torch.Tensor:
    """The rows `rows` (flat row index over [B, H_kv, T]) of kv_tensor(...) without building the rest."""
    b, h, t, d = shape
    rows = rows.to(torch.int64)
    idx = rows[:, None] * d + torch.arange(d, dtype=torch.int64, device=rows.device)[None, :]
    x = normal_fp16_at(seed, stream, idx.reshape(-1)).view(-1, d)
    if scales is not None:
        head = (rows // t) % h
        x = (x.float() * scales.to(rows.device)[head]).half()
    return x


def block_table(seed: int, batch: int, blocks_per_seq: int, num_blocks: int) -> torch.Tensor:
    """int32 [B, blocks_per_seq]: a seeded permutation of the physical blocks, first B*blocks_per_seq taken."""
    keys = random_words(seed, STREAM_BLOCKS, torch.arange(num_blocks, dtype=torch.int64))
    perm = torch.argsort(keys, stable=True)[: batch * blocks_per_seq]
    return perm.to(torch.int32).view(batch, blocks_per_seq)
