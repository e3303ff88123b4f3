"""The bounded-wait failure path on the GPU, exercised without a fault: the key encoder runs with its first tile's
copy withheld (tq_debug_encode_k_stalled) and a 2^22-cycle wait limit.  Nothing it waits on is in flight, so
every wait on that tile runs out: the kernel raises the device flag, drains the copies it did issue, frees its
tensor memory and returns.  The test checks the status the host reads (tq_stream_status -> TQ_ERR_DEVICE_FLAG),
the flag itself, and that the context still encodes correctly afterwards."""
import time

import numpy as np
import pytest
import torch

from kv_cache_vector_norm_b200 import synth, tq
from oracle import tq_oracle as o
from _tqh import NORM_RTOL, check_key_indices, params, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_expired_wait_is_reported_and_the_context_stays_usable():
    d, bits = 128, 3
    cd = tq.Codec(d, bits, 0)
    tq.read_device_flag(clear=True)
    assert tq.stream_status() == tq.TQ_OK
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = sms * 128 * 2                                   # every CTA owns two tiles; its first one is withheld
    x = synth.normal_fp16(1, synth.STREAM_K, (n, d)).to(DEV)
    packed = torch.empty(n, d * bits // 8, dtype=torch.uint8, device=DEV)
    norms = torch.empty(n, dtype=torch.float32, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.time()
    st = tq.LIB.tq_debug_encode_k_stalled(cd.handle, x.data_ptr(), n, packed.data_ptr(), norms.data_ptr(), 1 << 22,
                                          stream)
    assert st == tq.TQ_OK, tq.LIB.tq_last_error()
    assert tq.stream_status(clear=False) == tq.TQ_ERR_DEVICE_FLAG
    assert time.time() - t0 < 30.0                      # the waits ended on their own, milliseconds each
    assert b"bounded wait expired" in tq.LIB.tq_last_error()
    assert tq.read_device_flag(clear=True) & 1          # the wait-timeout bit
    assert tq.stream_status() == tq.TQ_OK               # cleared
    # the same context keeps working: a normal encode matches the oracle
    y = synth.normal_fp16(2, synth.STREAM_K, (1000, d))
    gp, gn = cd.encode_k(y.to(DEV))
    pi, c, t = params(d, bits, 0)
    ref_idx, ref_n, yy = o.encode_k(y.numpy(), pi, t)
    check_key_indices(o.unpack_lsb(to_np(gp), bits, d), ref_idx, yy, t)
    assert np.all(np.abs(to_np(gn) - ref_n) <= NORM_RTOL * ref_n)
    assert tq.stream_status() == tq.TQ_OK


def test_stalled_encode_argument_checks():
    cd = tq.Codec(128, 3, 0)
    x = torch.zeros(128, 128, dtype=torch.float16, device=DEV)
    p = torch.empty(128, 48, dtype=torch.uint8, device=DEV)
    nr = torch.empty(128, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert tq.LIB.tq_debug_encode_k_stalled(cd.handle, x.data_ptr(), 128, p.data_ptr(), nr.data_ptr(), 10,
                                            stream) == tq.TQ_ERR_INVALID_ARG
    assert tq.LIB.tq_debug_encode_k_stalled(None, x.data_ptr(), 128, p.data_ptr(), nr.data_ptr(), 1 << 22,
                                            stream) == tq.TQ_ERR_INVALID_ARG
    assert tq.stream_status() == tq.TQ_OK
