"""Helpers shared by the GPU parity tests: oracle parameters and the comparison rules.

Rules (the tolerances of the parity contract):
* value payloads, scales and zeros: bit-exact;
* key indices: bit-exact except where the oracle's fp64 rotated coordinate y lies within 1e-5 of the
  boundary between the two indices; such flips must be fewer than 1e-4 of all coordinates;
* key norms: relative error <= 1e-6;
* decoded keys / values and attention outputs: relative L2 <= 1e-3 against the oracle applied to the
  GPU's own indices.
"""
import functools
import json
import os

import numpy as np
import torch

from oracle import tq_oracle as o

_GOLDEN_CB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "sphere_codebooks_b7_b8.json")


@functools.lru_cache(maxsize=None)
def sphere_codebook(d: int, bits: int) -> np.ndarray:
    """The oracle's c* (sphere_codebook); the 7- and 8-bit ones at d = 64, 128, 256 come from the file
    tests/golden/make_sphere_codebooks.py wrote with the oracle (their plain iteration takes minutes)."""
    if bits >= 7:
        with open(_GOLDEN_CB) as f:
            book = json.load(f)["codebooks"].get(f"{d}/{bits}")
        if book is not None:
            return np.array([float.fromhex(h) for h in book])
    return o.sphere_codebook(d, bits)

BAND = 1e-5
FLIP_LIMIT = 1e-4
NORM_RTOL = 1e-6
L2_RTOL = 1e-3


@functools.lru_cache(maxsize=None)
def params(d: int, bits: int, seed: int, rotation: str = "haar"):
    pi_op = o.operational_rotation(d, seed, rotation)
    c_op, t = o.operational_codebook(d, bits, levels=sphere_codebook(d, bits))
    return pi_op, c_op, t


def check_key_indices(gpu_idx: np.ndarray, ref_idx: np.ndarray, y: np.ndarray, t: np.ndarray):
    """Return (mismatches, total); assert every mismatch is a neighbour flip inside the band."""
    diff = gpu_idx != ref_idx
    nmis = int(diff.sum())
    if nmis:
        gi, ri, yy = gpu_idx[diff], ref_idx[diff], y[diff]
        assert np.all(np.abs(gi - ri) == 1), "index differs by more than one level"
        b = np.minimum(gi, ri)
        assert np.all(np.abs(yy - t[b]) < BAND), f"flip outside the band: {np.abs(yy - t[b]).max()}"
    assert nmis <= FLIP_LIMIT * gpu_idx.size, (nmis, gpu_idx.size)
    return nmis, gpu_idx.size


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
