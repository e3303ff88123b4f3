"""Python binding of libtq (include/tq.h): argument marshalling only.

Every computation runs in the library's CUDA kernels (or, for tq_make_rotation / tq_build_codebook, in
its host C++).  PyTorch provides device memory and the current stream.  If libtq.so is missing this
module raises at import time -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_DEVICE_FLAG = range(5)
TQ_F16, TQ_F32 = 0, 1
TQ_ROT_HAAR, TQ_ROT_HADAMARD = 0, 1
ROTATIONS = {"haar": TQ_ROT_HAAR, "hadamard": TQ_ROT_HADAMARD}

_c_i64p = ctypes.POINTER(ctypes.c_int64)


class AttendArgs(ctypes.Structure):
    """Mirror of tq_attend_args."""
    _fields_ = [
        ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("v_bits", ctypes.c_int), ("v_group", ctypes.c_int),
        ("scale", ctypes.c_float), ("max_seq_len", ctypes.c_int64),
        ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int), ("block_size", ctypes.c_int),
        ("seq_lens", ctypes.c_void_p), ("q", ctypes.c_void_p), ("k_packed", ctypes.c_void_p),
        ("k_norms", ctypes.c_void_p), ("v_data", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
        ("v_zeros", ctypes.c_void_p), ("out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


# name -> (restype, argtypes)
class AttendWindow(ctypes.Structure):
    """Mirror of tq_attend_window."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("lens", ctypes.c_void_p), ("max_len", ctypes.c_int)]


class QjlKeys(ctypes.Structure):
    """Mirror of tq_qjl_keys."""
    _fields_ = [("signs", ctypes.c_void_p), ("rho", ctypes.c_void_p)]


SIGNATURES = {
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_version": (ctypes.c_int, []),
    "tq_make_rotation": (ctypes.c_int, [ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_make_rotation_ex": (ctypes.c_int, [ctypes.c_int, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p]),
    "tq_build_codebook": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p]),
    "tq_codec_create": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.POINTER(ctypes.c_void_p)]),
    "tq_codec_create_ex": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_void_p)]),
    "tq_codec_rotation": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]),
    "tq_codec_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "tq_codec_info": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_encode_k": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_decode_k": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                   ctypes.c_int, ctypes.c_void_p]),
    "tq_encode_v": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p]),
    "tq_decode_v": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "tq_attend_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(AttendArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "tq_attend_decode": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(AttendArgs), ctypes.c_void_p]),
    "tq_attend_decode_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(AttendArgs), ctypes.c_void_p]),
    "tq_attend_scores": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(AttendArgs), ctypes.c_void_p, ctypes.c_void_p]),
    "tq_attend_window_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(AttendArgs), ctypes.POINTER(AttendWindow),
                                                        ctypes.POINTER(ctypes.c_size_t)]),
    "tq_attend_decode_window": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(AttendArgs),
                                               ctypes.POINTER(AttendWindow), ctypes.c_void_p]),
    "tq_read_device_flag": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_int]),
    "tq_codec_create_qjl": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_void_p)]),
    "tq_codec_qjl_bits": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]),
    "tq_make_qjl_matrix": (ctypes.c_int, [ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_stream_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int]),
    "tq_debug_encode_k_stalled": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p]),
    "tq_attend_qjl_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(AttendArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "tq_attend_decode_qjl": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(AttendArgs), ctypes.POINTER(QjlKeys),
                                            ctypes.c_void_p]),
    "tq_encode_k_qjl": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so not found at {LIB_PATH}; build it with "
                          "`python -m kv_cache_vector_norm_b200._build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


class TQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = LIB.tq_last_error().decode(errors="replace")
        super().__init__(f"{fn} failed with status {status}: {msg}")


def _check(fn: str, status: int):
    if status != TQ_OK:
        raise TQError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")


# ------------------------------------------------------------------------------- host parameters

def make_rotation(d: int, seed: int, rotation: str = "haar"):
    """(Pi fp64 [d, d], Pi_op fp16 [d, d]) from tq_make_rotation_ex."""
    pi = np.empty((d, d), np.float64)
    pi16 = np.empty((d, d), np.uint16)
    _check("tq_make_rotation_ex", LIB.tq_make_rotation_ex(d, seed, ROTATIONS[rotation], pi.ctypes.data,
                                                          pi16.ctypes.data))
    return pi, pi16.view(np.float16)


def build_codebook(d: int, bits: int):
    """dict(centroids fp64, centroids_f16, boundaries f32, distortion) from tq_build_codebook."""
    k = 1 << bits
    c = np.empty(k, np.float64)
    c16 = np.empty(k, np.uint16)
    t = np.empty(max(k - 1, 1), np.float32)
    dist = ctypes.c_double()
    _check("tq_build_codebook", LIB.tq_build_codebook(d, bits, c.ctypes.data, c16.ctypes.data, t.ctypes.data,
                                                      ctypes.byref(dist)))
    return {"centroids": c, "centroids_f16": c16.view(np.float16), "boundaries": t[:k - 1], "distortion": dist.value}


# ------------------------------------------------------------------------------------ key codec

class Codec:
    """A key codec (rotation + codebook resident on the current CUDA device).  rotation: "haar" (the seeded
    Haar rotation) or "hadamard" (the seeded randomized Walsh-Hadamard rotation)."""

    def __init__(self, d: int, bits: int, seed: int = 0, rotation: str = "haar"):
        h = ctypes.c_void_p()
        _check("tq_codec_create_ex", LIB.tq_codec_create_ex(d, bits, seed, ROTATIONS[rotation], ctypes.byref(h)))
        self._h = h
        self.d, self.bits, self.seed, self.rotation = d, bits, seed, rotation
        self.row_bytes = d * bits // 8

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            LIB.tq_codec_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def encode_k(self, x: torch.Tensor, slot_mapping: torch.Tensor | None = None,
                 packed: torch.Tensor | None = None, norms: torch.Tensor | None = None):
        """x: [N, d] fp16 (row stride a multiple of 8).  Returns (packed u8 [rows, d*b/8], norms f32 [rows])."""
        _need_cuda(x, "x", torch.float16)
        if x.dim() != 2 or x.shape[1] != self.d or x.stride(1) != 1:
            raise ValueError(f"x must be [N, {self.d}] with unit column stride")
        n = x.shape[0]
        if packed is None:
            packed = torch.empty((n, self.row_bytes), dtype=torch.uint8, device=x.device)
        if norms is None:
            norms = torch.empty((packed.shape[0],), dtype=torch.float32, device=x.device)
        if slot_mapping is not None:
            _need_cuda(slot_mapping, "slot_mapping", torch.int64)
        _check("tq_encode_k", LIB.tq_encode_k(self._h, _ptr(x), n, x.stride(0), _ptr(slot_mapping), _ptr(packed),
                                              _ptr(norms), _stream(x.device)))
        return packed, norms

    def decode_k(self, packed: torch.Tensor, norms: torch.Tensor, out_dtype=torch.float16,
                 out: torch.Tensor | None = None):
        _need_cuda(packed, "packed", torch.uint8)
        _need_cuda(norms, "norms", torch.float32)
        n = packed.shape[0]
        if out is None:
            out = torch.empty((n, self.d), dtype=out_dtype, device=packed.device)
        dt = TQ_F32 if out.dtype == torch.float32 else TQ_F16
        _check("tq_decode_k", LIB.tq_decode_k(self._h, _ptr(packed), _ptr(norms), n, _ptr(out), dt,
                                              _stream(packed.device)))
        return out


def make_qjl_matrix(d: int, seed: int = 0):
    """(S fp64 [d, d], fp16(S) as float16 [d, d]) of a QJL codec, built by the library on the host."""
    s = np.empty((d, d), dtype=np.float64)
    s16 = np.empty((d, d), dtype=np.uint16)
    _check("tq_make_qjl_matrix", LIB.tq_make_qjl_matrix(d, seed, s.ctypes.data, s16.ctypes.data))
    return s, s16.view(np.float16)


class QjlCodec(Codec):
    """A QJL key codec: the MSE stage at bits - 1 (an ordinary Codec of bits - 1 for encode_k / decode_k /
    attend_decode) plus the seeded Gaussian sketch S of the residual."""

    def __init__(self, d: int, bits: int, seed: int = 0, rotation: str = "haar"):
        h = ctypes.c_void_p()
        _check("tq_codec_create_qjl", LIB.tq_codec_create_qjl(d, bits, seed, ROTATIONS[rotation], ctypes.byref(h)))
        self._h = h
        self.d, self.bits, self.seed, self.rotation = d, bits - 1, seed, rotation
        self.qjl_bits = bits
        self.row_bytes = d * (bits - 1) // 8

    def encode_k_qjl(self, x: torch.Tensor, slot_mapping: torch.Tensor | None = None,
                     packed: torch.Tensor | None = None, norms: torch.Tensor | None = None,
                     signs: torch.Tensor | None = None, rho: torch.Tensor | None = None):
        """x: [N, d] fp16.  Returns (packed u8 [rows, d*(bits-1)/8], norms f32 [rows], signs u8 [rows, d/8],
        rho f32 [rows])."""
        _need_cuda(x, "x", torch.float16)
        if x.dim() != 2 or x.shape[1] != self.d or x.stride(1) != 1:
            raise ValueError(f"x must be [N, {self.d}] with unit column stride")
        n = x.shape[0]
        if packed is None:
            packed = torch.empty((n, self.row_bytes), dtype=torch.uint8, device=x.device)
        rows = packed.shape[0]
        if norms is None:
            norms = torch.empty((rows,), dtype=torch.float32, device=x.device)
        if signs is None:
            signs = torch.empty((rows, self.d // 8), dtype=torch.uint8, device=x.device)
        if rho is None:
            rho = torch.empty((rows,), dtype=torch.float32, device=x.device)
        if slot_mapping is not None:
            _need_cuda(slot_mapping, "slot_mapping", torch.int64)
        _check("tq_encode_k_qjl", LIB.tq_encode_k_qjl(self._h, _ptr(x), n, x.stride(0), _ptr(slot_mapping),
                                                      _ptr(packed), _ptr(norms), _ptr(signs), _ptr(rho),
                                                      _stream(x.device)))
        return packed, norms, signs, rho


# ---------------------------------------------------------------------------------- value codec

def v_row_bytes(d: int, bits: int) -> int:
    return (d * bits + 7) // 8


def encode_v(x: torch.Tensor, bits: int, group: int = 32, slot_mapping: torch.Tensor | None = None,
             data: torch.Tensor | None = None, scales: torch.Tensor | None = None,
             zeros: torch.Tensor | None = None):
    """x: [N, d] fp16.  Returns (data u8 [rows, (d*b+7)/8], scales f16 [rows, d/group], zeros f16)."""
    _need_cuda(x, "x", torch.float16)
    n, d = x.shape
    if x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    g = d // group
    if data is None:
        data = torch.empty((n, v_row_bytes(d, bits)), dtype=torch.uint8, device=x.device)
    rows = data.shape[0]
    if scales is None:
        scales = torch.empty((rows, g), dtype=torch.float16, device=x.device)
    if zeros is None:
        zeros = torch.empty((rows, g), dtype=torch.float16, device=x.device)
    if slot_mapping is not None:
        _need_cuda(slot_mapping, "slot_mapping", torch.int64)
    _check("tq_encode_v", LIB.tq_encode_v(d, bits, group, _ptr(x), n, x.stride(0), _ptr(slot_mapping), _ptr(data),
                                          _ptr(scales), _ptr(zeros), _stream(x.device)))
    return data, scales, zeros


def decode_v(data: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, d: int, bits: int, group: int = 32,
             out_dtype=torch.float16, out: torch.Tensor | None = None):
    _need_cuda(data, "data", torch.uint8)
    n = data.shape[0]
    if out is None:
        out = torch.empty((n, d), dtype=out_dtype, device=data.device)
    dt = TQ_F32 if out.dtype == torch.float32 else TQ_F16
    _check("tq_decode_v", LIB.tq_decode_v(d, bits, group, _ptr(data), _ptr(scales), _ptr(zeros), n, _ptr(out), dt,
                                          _stream(data.device)))
    return out


# ------------------------------------------------------------------------------------ attention

@dataclass
class Cache:
    """Device pools of one layer's compressed cache (rows in the layouts of tq.h)."""
    k_packed: torch.Tensor
    k_norms: torch.Tensor
    v_data: torch.Tensor
    v_scales: torch.Tensor
    v_zeros: torch.Tensor


ATTEND_WINDOW_MAX = 256


def _window(win_k: torch.Tensor, win_v: torch.Tensor, win_lens: torch.Tensor | None, q) -> AttendWindow:
    _need_cuda(win_k, "win_k", torch.float16)
    _need_cuda(win_v, "win_v", torch.float16)
    if win_k.dim() != 4 or win_k.shape != win_v.shape or not win_k.is_contiguous() or not win_v.is_contiguous():
        raise ValueError("win_k and win_v must be contiguous [B, H_kv, W, d] fp16 tensors of one shape")
    if win_k.shape[0] != q.shape[0] or win_k.shape[3] != q.shape[2]:
        raise ValueError("the window's batch and head_dim must match q")
    w = AttendWindow()
    w.k, w.v = win_k.data_ptr(), win_v.data_ptr()
    if win_lens is not None:
        _need_cuda(win_lens, "win_lens", torch.int32)
    w.lens = win_lens.data_ptr() if win_lens is not None else None
    w.max_len = win_k.shape[2]
    return w


def _attend_args(codec: Codec, q, cache: Cache, *, num_kv_heads, v_bits, v_group, max_seq_len, block_table,
                 seq_lens, scale, out, workspace):
    b, hq, d = q.shape
    a = AttendArgs()
    a.batch, a.num_q_heads, a.num_kv_heads, a.head_dim = b, hq, num_kv_heads, d
    a.v_bits, a.v_group, a.scale = v_bits, v_group, float(scale)
    a.max_seq_len = int(max_seq_len or 0)
    a.block_table = block_table.data_ptr() if block_table is not None else None
    a.max_blocks = block_table.shape[1] if block_table is not None else 0
    a.block_size = 16 if block_table is not None else 0
    a.seq_lens = seq_lens.data_ptr() if seq_lens is not None else None
    a.q = q.data_ptr()
    a.k_packed, a.k_norms = cache.k_packed.data_ptr(), cache.k_norms.data_ptr()
    a.v_data, a.v_scales, a.v_zeros = cache.v_data.data_ptr(), cache.v_scales.data_ptr(), cache.v_zeros.data_ptr()
    a.out = out.data_ptr() if out is not None else None
    a.workspace = workspace.data_ptr() if workspace is not None else None
    a.workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return a


def attend_workspace_bytes(codec: Codec, q, cache: Cache, **kw) -> int:
    a = _attend_args(codec, q, cache, out=None, workspace=None, **kw)
    nb = ctypes.c_size_t()
    _check("tq_attend_workspace_bytes", LIB.tq_attend_workspace_bytes(ctypes.byref(a), ctypes.byref(nb)))
    return nb.value


def attend_workspace(codec: Codec, q, cache: Cache, **kw) -> torch.Tensor:
    """A workspace of the size tq_attend_workspace_bytes asks for (at least 16 bytes)."""
    return torch.empty(max(16, attend_workspace_bytes(codec, q, cache, **kw)), dtype=torch.uint8, device=q.device)


def attend_window_workspace(codec: Codec, q, cache: Cache, win_k, win_v, win_lens=None, **kw) -> torch.Tensor:
    """A workspace of the size tq_attend_window_workspace_bytes asks for."""
    a = _attend_args(codec, q, cache, out=None, workspace=None, **kw)
    w = _window(win_k, win_v, win_lens, q)
    nb = ctypes.c_size_t()
    _check("tq_attend_window_workspace_bytes",
           LIB.tq_attend_window_workspace_bytes(ctypes.byref(a), ctypes.byref(w), ctypes.byref(nb)))
    return torch.empty(max(16, nb.value), dtype=torch.uint8, device=q.device)


def attend_decode(codec: Codec, q: torch.Tensor, cache: Cache, *, num_kv_heads: int, v_bits: int, v_group: int = 32,
                  max_seq_len: int | None = None, block_table: torch.Tensor | None = None,
                  seq_lens: torch.Tensor | None = None, scale: float = 0.0, out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, win_k: torch.Tensor | None = None,
                  win_v: torch.Tensor | None = None, win_lens: torch.Tensor | None = None) -> torch.Tensor:
    """One decode step: q [B, H_q, d] fp16 against the compressed cache, plus (win_k, win_v: [B, H_kv, W, d]
    fp16, win_lens: [B] int32 or None) a window of recent uncompressed tokens.  Returns out [B, H_q, d] f32."""
    _need_cuda(q, "q", torch.float16)
    kw = dict(num_kv_heads=num_kv_heads, v_bits=v_bits, v_group=v_group, max_seq_len=max_seq_len,
              block_table=block_table, seq_lens=seq_lens, scale=scale)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if win_k is None:
        if workspace is None:
            workspace = attend_workspace(codec, q, cache, **kw)
        a = _attend_args(codec, q, cache, out=out, workspace=workspace, **kw)
        _check("tq_attend_decode", LIB.tq_attend_decode(codec.handle, ctypes.byref(a), _stream(q.device)))
        return out
    if workspace is None:
        workspace = attend_window_workspace(codec, q, cache, win_k, win_v, win_lens, **kw)
    a = _attend_args(codec, q, cache, out=out, workspace=workspace, **kw)
    w = _window(win_k, win_v, win_lens, q)
    _check("tq_attend_decode_window", LIB.tq_attend_decode_window(codec.handle, ctypes.byref(a), ctypes.byref(w),
                                                                  _stream(q.device)))
    return out


def attend_scores(codec: Codec, q: torch.Tensor, cache: Cache, *, num_kv_heads: int, v_bits: int, v_group: int = 32,
                  max_seq_len: int | None = None, block_table: torch.Tensor | None = None,
                  seq_lens: torch.Tensor | None = None, scale: float = 0.0,
                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The compressed path's attention logits [B, H_q, L] f32 (L = max_seq_len, or max_blocks * 16 when paged);
    -inf past each sequence's length."""
    _need_cuda(q, "q", torch.float16)
    kw = dict(num_kv_heads=num_kv_heads, v_bits=v_bits, v_group=v_group, max_seq_len=max_seq_len,
              block_table=block_table, seq_lens=seq_lens, scale=scale)
    length = block_table.shape[1] * 16 if block_table is not None else int(max_seq_len)
    scores = torch.empty((q.shape[0], q.shape[1], length), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = attend_workspace(codec, q, cache, **kw)
    a = _attend_args(codec, q, cache, out=None, workspace=workspace, **kw)
    _check("tq_attend_scores", LIB.tq_attend_scores(codec.handle, ctypes.byref(a), scores.data_ptr(), _stream(q.device)))
    return scores


def attend_decode_qjl(codec: "QjlCodec", q: torch.Tensor, cache: Cache, signs: torch.Tensor, rho: torch.Tensor, *,
                      num_kv_heads: int, v_bits: int, v_group: int = 32, max_seq_len: int | None = None,
                      block_table: torch.Tensor | None = None, seq_lens: torch.Tensor | None = None,
                      scale: float = 0.0, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Decode attention over QJL residual keys: cache holds the MSE stage (codes at bits - 1, norms) and the
    values; signs [rows, d/8] u8 and rho [rows] f32 the residual sketch.  Returns out [B, H_q, d] f32."""
    _need_cuda(q, "q", torch.float16)
    _need_cuda(signs, "signs", torch.uint8)
    _need_cuda(rho, "rho", torch.float32)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    kw = dict(num_kv_heads=num_kv_heads, v_bits=v_bits, v_group=v_group, max_seq_len=max_seq_len,
              block_table=block_table, seq_lens=seq_lens, scale=scale)
    if workspace is None:
        a0 = _attend_args(codec, q, cache, out=None, workspace=None, **kw)
        nb = ctypes.c_size_t()
        _check("tq_attend_qjl_workspace_bytes", LIB.tq_attend_qjl_workspace_bytes(ctypes.byref(a0), ctypes.byref(nb)))
        workspace = torch.empty(max(16, nb.value), dtype=torch.uint8, device=q.device)
    a = _attend_args(codec, q, cache, out=out, workspace=workspace, **kw)
    keys = QjlKeys(signs.data_ptr(), rho.data_ptr())
    _check("tq_attend_decode_qjl", LIB.tq_attend_decode_qjl(codec.handle, ctypes.byref(a), ctypes.byref(keys),
                                                            _stream(q.device)))
    return out


ATTEND_SCRATCH_BYTES = 4 << 20


def attend_decode_noalloc(codec: Codec, q: torch.Tensor, cache: Cache, *, num_kv_heads: int, v_bits: int,
                          v_group: int = 32, max_seq_len: int | None = None, block_table: torch.Tensor | None = None,
                          seq_lens: torch.Tensor | None = None, scale: float = 0.0,
                          out: torch.Tensor | None = None) -> torch.Tensor:
    """attend_decode without a workspace: the library's fixed device scratch (ATTEND_SCRATCH_BYTES) holds the
    split-K partials, so the call itself allocates nothing on the device; for callers that cannot allocate
    (graph capture or replay, fixed memory pools).  Calls that overlap on the GPU share that scratch and
    must be serialised.  `out` should be passed in by such callers, since creating it here allocates."""
    _need_cuda(q, "q", torch.float16)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    a = _attend_args(codec, q, cache, num_kv_heads=num_kv_heads, v_bits=v_bits, v_group=v_group,
                     max_seq_len=max_seq_len, block_table=block_table, seq_lens=seq_lens, scale=scale, out=out,
                     workspace=None)
    _check("tq_attend_decode_noalloc", LIB.tq_attend_decode_noalloc(codec.handle, ctypes.byref(a), _stream(q.device)))
    return out


def stream_status(device=None, clear: bool = True) -> int:
    """tq_stream_status on the current stream of `device`: the status code (0 or TQ_ERR_DEVICE_FLAG); raises on
    any other error."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = LIB.tq_stream_status(_stream(dev), 1 if clear else 0)
    if st not in (TQ_OK, TQ_ERR_DEVICE_FLAG):
        _check("tq_stream_status", st)
    return st


def read_device_flag(clear: bool = True) -> int:
    v = ctypes.c_int()
    _check("tq_read_device_flag", LIB.tq_read_device_flag(ctypes.byref(v), 1 if clear else 0))
    return v.value
