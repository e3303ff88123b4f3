"""CPU-side checks of libtq: every symbol include/tq.h declares is exported, the host parameter
builders agree with the oracle (independent algorithms: Householder vs Gram-Schmidt QR, Gauss-Legendre
quadrature vs incomplete-beta Lloyd steps), and argument errors are reported without touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import tq
from oracle import tq_oracle as o
from _tqh import sphere_codebook

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 14
    lib = ctypes.CDLL(tq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(tq.SIGNATURES), set(names) ^ set(tq.SIGNATURES)


@pytest.mark.parametrize("d", [3, 8, 64, 128, 256])
def test_rotation_matches_oracle(d):
    for seed in (0, 12345):
        pi, pi16 = tq.make_rotation(d, seed)
        ref = o.haar_rotation(d, seed)
        assert np.max(np.abs(pi - ref)) < 1e-12
        assert np.array_equal(pi16.astype(np.float64), o.to_fp16_values(ref))


@pytest.mark.parametrize("d", [2, 64, 128, 256, 1024])
def test_hadamard_rotation_matches_oracle(d):
    pi, pi16 = tq.make_rotation(d, 17, "hadamard")
    ref = o.hadamard_rotation(d, 17)
    assert np.array_equal(pi, ref)
    assert np.array_equal(pi16.astype(np.float64), o.to_fp16_values(ref))
    assert np.array_equal(pi16.astype(np.float64), o.operational_rotation(d, 17, "hadamard"))


def test_window_argument_errors():
    a = tq.AttendArgs()
    a.batch, a.num_q_heads, a.num_kv_heads, a.head_dim, a.v_bits, a.v_group = 1, 8, 1, 128, 2, 32
    a.max_seq_len = 64
    nb = ctypes.c_size_t(7)
    assert tq.LIB.tq_attend_window_workspace_bytes(ctypes.byref(a), None, ctypes.byref(nb)) == tq.TQ_ERR_INVALID_ARG
    w = tq.AttendWindow()
    for bad in (0, tq.ATTEND_WINDOW_MAX + 1):
        w.max_len = bad
        assert tq.LIB.tq_attend_window_workspace_bytes(ctypes.byref(a), ctypes.byref(w), ctypes.byref(nb)) == \
            tq.TQ_ERR_INVALID_ARG
        assert b"max_len" in tq.LIB.tq_last_error()
    w.max_len = 128
    assert tq.LIB.tq_attend_window_workspace_bytes(ctypes.byref(a), ctypes.byref(w), ctypes.byref(nb)) == tq.TQ_OK
    # one split plus the window's partial, after the prepared query
    assert nb.value == (128 // 16 * 32 + 2) * 16 + 2 * (16 + 8 * 128) * 4
    assert tq.LIB.tq_attend_decode_window(None, ctypes.byref(a), ctypes.byref(w), None) == tq.TQ_ERR_INVALID_ARG


def test_rotation_kind_errors():
    out = np.empty(96 * 96)
    assert tq.LIB.tq_make_rotation_ex(96, 0, tq.TQ_ROT_HADAMARD, out.ctypes.data, None) == tq.TQ_ERR_INVALID_ARG
    assert b"power of two" in tq.LIB.tq_last_error()
    assert tq.LIB.tq_make_rotation_ex(64, 0, 7, out.ctypes.data, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.LIB.tq_codec_create_ex(128, 4, 0, 7, ctypes.byref(ctypes.c_void_p())) == tq.TQ_ERR_INVALID_ARG
    assert tq.LIB.tq_version() == 101


@pytest.mark.parametrize("d", [3, 64, 128, 256, 1024])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle(d, bits):
    cb = tq.build_codebook(d, bits)
    c = o.sphere_codebook(d, bits)
    assert np.max(np.abs(cb["centroids"] - c)) < 1e-12 * max(1.0, np.max(np.abs(c)))
    if d >= 64:
        c_op, t = o.operational_codebook(d, bits)
        assert np.array_equal(cb["centroids_f16"].astype(np.float64), c_op)
        assert np.array_equal(cb["boundaries"].astype(np.float64), t)
        assert abs(cb["distortion"] - o.sphere_distortion(d, c_op, t)) < 1e-10


def test_argument_errors_are_reported():
    st = tq.LIB.tq_make_rotation(1, 0, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and b"d=1" in tq.LIB.tq_last_error()
    assert tq.LIB.tq_build_codebook(128, 9, None, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.LIB.tq_encode_k(None, None, 10, 128, None, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert b"codec" in tq.LIB.tq_last_error()
    st = tq.LIB.tq_encode_v(128, 5, 32, None, 10, 128, None, None, None, None, None)
    assert st == tq.TQ_ERR_UNSUPPORTED and b"bits=5" in tq.LIB.tq_last_error()
    assert tq.LIB.tq_encode_v(128, 2, 48, None, 10, 128, None, None, None, None, None) == tq.TQ_ERR_UNSUPPORTED
    assert tq.LIB.tq_decode_v(96, 2, 32, None, None, None, 10, None, 0, None) == tq.TQ_ERR_UNSUPPORTED
    assert tq.LIB.tq_decode_k(None, None, None, 1, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    a = tq.AttendArgs()
    a.batch, a.num_q_heads, a.num_kv_heads, a.head_dim, a.v_bits, a.v_group = 1, 12, 1, 128, 2, 32
    a.max_seq_len = 64
    nb = ctypes.c_size_t(123)
    assert tq.LIB.tq_attend_workspace_bytes(ctypes.byref(a), ctypes.byref(nb)) == tq.TQ_ERR_UNSUPPORTED  # GQA 12 > 8
    assert nb.value == 0
    a.num_q_heads = 8
    a.max_seq_len = 40
    assert tq.LIB.tq_attend_workspace_bytes(ctypes.byref(a), ctypes.byref(nb)) == tq.TQ_ERR_INVALID_ARG  # not 16k
    a.max_seq_len = 4096
    assert tq.LIB.tq_attend_workspace_bytes(ctypes.byref(a), ctypes.byref(nb)) == tq.TQ_OK
    assert nb.value > 0                                                     # one sequence: split over the SMs
    a.batch, a.num_kv_heads, a.max_seq_len = 3, 2, 16                       # one chunk per sequence: one split
    assert tq.LIB.tq_attend_workspace_bytes(ctypes.byref(a), ctypes.byref(nb)) == tq.TQ_OK
    assert nb.value == 3 * 2 * (128 // 16 * 32 + 2) * 16                   # only the prepared query fragments
    assert tq.LIB.tq_attend_decode(None, ctypes.byref(a), None) == tq.TQ_ERR_INVALID_ARG
    assert tq.LIB.tq_codec_create(96, 4, 0, ctypes.byref(ctypes.c_void_p())) == tq.TQ_ERR_UNSUPPORTED
    # key widths 1..8; from 5 bits only at d <= 128
    assert tq.LIB.tq_codec_create(256, 5, 0, ctypes.byref(ctypes.c_void_p())) == tq.TQ_ERR_UNSUPPORTED
    assert b"d <= 128" in tq.LIB.tq_last_error()
    assert tq.LIB.tq_codec_create(128, 9, 0, ctypes.byref(ctypes.c_void_p())) == tq.TQ_ERR_UNSUPPORTED
    assert tq.LIB.tq_codec_create(128, 0, 0, ctypes.byref(ctypes.c_void_p())) == tq.TQ_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_codec_create_without_device_reports_cuda_error():
    h = ctypes.c_void_p()
    assert tq.LIB.tq_codec_create(128, 4, 0, ctypes.byref(h)) == tq.TQ_ERR_CUDA
    assert h.value is None


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_qjl_matrix_matches_oracle(d):
    for seed in (0, 77):
        s, s16 = tq.make_qjl_matrix(d, seed)
        assert np.max(np.abs(s - o.qjl_matrix(d, seed))) < 1e-12      # libm last-ulp differences only
        assert np.array_equal(s16.astype(np.float64), o.operational_qjl_matrix(d, seed))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [5, 6, 7, 8])
def test_high_width_codebook_matches_oracle(d, bits):
    # the library solves the Lloyd fixed point by Newton's method; the oracle by the plain iteration (its 7- and
    # 8-bit fixed points are the stored ones): same levels, the same fp16 operational levels and boundaries
    cb = tq.build_codebook(d, bits)
    c = sphere_codebook(d, bits)
    assert np.max(np.abs(cb["centroids"] - c)) < 1e-12 * np.max(np.abs(c))
    c_op, t = o.operational_codebook(d, bits, levels=c)
    assert np.array_equal(cb["centroids_f16"].astype(np.float64), c_op)
    assert np.array_equal(cb["boundaries"].astype(np.float64), t)
    assert abs(cb["distortion"] - o.sphere_distortion(d, c_op, t)) < 1e-10
