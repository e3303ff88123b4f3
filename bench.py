#!/usr/bin/env python
"""Benchmark of the TurboQuant-style KV-cache hot path on B200.

One step = the whole path over one synthetic layer cache: key encode, value encode, key decode, value
decode and one fused decode-attention step over the compressed cache.  Default workload: the 70B-class
GQA decode step (batch 1, 8 KV heads, 64 query heads, 131072 tokens, head_dim 128, K 3-bit, V 2-bit
group 32, lognormal channel scales).

`value` is whole-job throughput in Mvectors/s, one "vector" being one (token, kv head) key/value pair
carried through encode + decode + attention; every kernel starts with a cold L2 (a 256 MiB write flushes
it before each launch, outside the timed interval) and only kernel time counts.  The per-kernel table
gives Mvectors/s and algorithmic GB/s against the measured HBM copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference] [--workload NAME]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "encode/decode Mvectors/s; fused compressed-KV decode-attn GB/s vs HBM peak"

WORKLOADS = {
    "70b_decode_128k": dict(batch=1, kv_heads=8, q_heads=64, tokens=131072, d=128, k_bits=3, v_bits=2, v_group=32,
                            outliers=0.0,
                            desc="70B-class GQA decode step: batch 1, 8 KV heads, 64 query heads, 131072-token "
                                 "cache, head_dim 128, K 3-bit, V 2-bit group 32, fp16 N(0,1) x lognormal channel "
                                 "scales"),
    "llama3_8b_layer": dict(batch=8, kv_heads=8, q_heads=32, tokens=8192, d=128, k_bits=4, v_bits=2, v_group=32,
                            outliers=0.01,
                            desc="Llama-3-8B-shaped layer: batch 8, 8 KV heads, 32 query heads, 8192 tokens, "
                                 "head_dim 128, K 4-bit, V 2-bit group 32, lognormal channel scales, 1% outlier "
                                 "channels x20"),
}


def algorithmic_bytes(w):
    d, kb, vb, g = w["d"], w["k_bits"], w["v_bits"], w["v_group"]
    k = 2 * d + d * kb // 8 + 4
    v = 2 * d + (d * vb + 7) // 8 + 4 * (d // g)
    att = (d * kb // 8 + 4) + ((d * vb + 7) // 8 + 4 * (d // g))
    return {"encode_k": k, "decode_k": k, "encode_v": v, "decode_v": v, "attend": att}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json: STREAM-style copy)"
    except Exception:
        return 6650.0, "fallback (6.65 TB/s)"


# sources each kernel's code and launch configuration come from: a recorded DRAM traffic figure stays valid
# only while these files are unchanged
KERNEL_SOURCES = {
    "encode_k": ("tq_device.cuh", "tq_codec_kernels.cuh", "tq_lib.cu"),
    "decode_k": ("tq_device.cuh", "tq_codec_kernels.cuh", "tq_lib.cu"),
    "encode_v": ("tq_device.cuh", "tq_codec_kernels.cuh", "tq_lib.cu"),
    "decode_v": ("tq_device.cuh", "tq_codec_kernels.cuh", "tq_lib.cu"),
    "attend": ("tq_device.cuh", "tq_attend_kernel.cuh", "tq_lib.cu"),
}


def source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_vector_norm_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        e = rec.get(workload, {}).get(kernel)
        if e and e.get("source_hash") == source_hash(kernel):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                pr = torch.cuda.get_device_properties(index)
                bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                                       getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                r = self._reasons_fn(self.h) if self._reasons_fn else 0
                if util > 0:
                    self.samples.append(mhz)
                    for bit, name in self.REASONS.items():
                        if r & bit and name != "gpu_idle":
                            self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------ GPU arm

def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's); x itself with one rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def chunk_bounds(n: int, chunks: int) -> list:
    """Row boundaries of the end-to-end pass's chunks: nondecreasing, from 0 to n, every inner boundary a
    multiple of 128 rows (whole key-codec tiles; every pool array then starts each chunk 16-byte aligned)."""
    chunks = max(1, chunks)
    return [((n * j // chunks) // 128) * 128 for j in range(chunks)] + [n]


def job_value(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput in M units/s: every rank processes units_per_rank per step (weak scaling)."""
    return world * units_per_rank / (ms_per_step / 1000.0) / 1e6


def gpu_arm(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from kv_cache_vector_norm_b200 import synth, tq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    b, hkv, hq, t, d = w["batch"], w["kv_heads"], w["q_heads"], w["tokens"], w["d"]
    kb, vb, vg = w["k_bits"], w["v_bits"], w["v_group"]
    n = b * hkv * t
    seed = rank
    ks = synth.channel_scales(seed, hkv, d, "k", outlier_frac=w["outliers"])
    vs = synth.channel_scales(seed, hkv, d, "v", outlier_frac=w["outliers"])
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=dev, scales=ks).view(n, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=dev, scales=vs).view(n, d)
    q = synth.normal_fp16(seed, synth.STREAM_Q, (b, hq, d), device=dev)
    codec = tq.Codec(d, kb, 0, rotation=args.rotation)
    kp = torch.empty(n, d * kb // 8, dtype=torch.uint8, device=dev)
    kn = torch.empty(n, dtype=torch.float32, device=dev)
    vd = torch.empty(n, (d * vb + 7) // 8, dtype=torch.uint8, device=dev)
    vsc = torch.empty(n, d // vg, dtype=torch.float16, device=dev)
    vz = torch.empty(n, d // vg, dtype=torch.float16, device=dev)
    kdec = torch.empty(n, d, dtype=torch.float16, device=dev)
    vdec = torch.empty(n, d, dtype=torch.float16, device=dev)
    out = torch.empty(b, hq, d, dtype=torch.float32, device=dev)
    cache = tq.Cache(kp, kn, vd, vsc, vz)
    akw = dict(num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=t, block_table=None, seq_lens=None, scale=0.0)
    if args.window > 0:
        # recent uncompressed tokens beside the compressed cache ("KV Cache API" store.py buffer)
        win_k = synth.normal_fp16(0, 21, (b, hkv, args.window, d), device=dev)
        win_v = synth.normal_fp16(0, 22, (b, hkv, args.window, d), device=dev)
        akw.update(win_k=win_k, win_v=win_v)
        ws = tq.attend_window_workspace(codec, q, cache, win_k, win_v, None,
                                        **{k: v for k, v in akw.items() if not k.startswith("win_")})
    else:
        ws = tq.attend_workspace(codec, q, cache, **akw)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    kernels = [
        ("encode_k", lambda: codec.encode_k(k, packed=kp, norms=kn)),
        ("encode_v", lambda: tq.encode_v(v, vb, vg, data=vd, scales=vsc, zeros=vz)),
        ("decode_k", lambda: codec.decode_k(kp, kn, out=kdec)),
        ("decode_v", lambda: tq.decode_v(vd, vsc, vz, d, vb, vg, out=vdec)),
        ("attend", lambda: tq.attend_decode(codec, q, cache, out=out, workspace=ws, **akw)),
    ]

    if args.only:
        if args.only in ("decode_k", "decode_v", "attend"):
            # the compressed cache these kernels read is written once, outside the timed launches
            kernels[0][1]()
            kernels[1][1]()
        kernels = [kv for kv in kernels if kv[0] == args.only]

    def one_step(record):
        for name, fn in kernels:
            flush_buf.fill_(1)
            if record is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                record.append((name, e0, e1))
            else:
                fn()

    for _ in range(args.warmup):
        one_step(None)
    torch.cuda.synchronize()
    if tq.read_device_flag() != 0:
        raise RuntimeError("a kernel raised the device error flag during warm-up")

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    events = []
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        for _ in range(args.steps):
            one_step(events)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    per = {name: 0.0 for name, _ in kernels}
    for name, e0, e1 in events:
        per[name] += e0.elapsed_time(e1)
    if args.only:
        return dict(per=per, launch_ms=[e0.elapsed_time(e1) for _, e0, e1 in events], n=n)
    total_ms = max_over_ranks(sum(per.values()), world, dev)
    ms_per_step = total_ms / args.steps

    # ---------------------------------------------------------------- end to end through host buffers
    k_host = k.cpu().pin_memory()
    v_host = v.cpu().pin_memory()
    q_host = q.cpu().pin_memory()
    kdec_host = torch.empty_like(kdec, device="cpu").pin_memory()
    vdec_host = torch.empty_like(vdec, device="cpu").pin_memory()
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 20))

    # The cache moves in row chunks on three streams: host-to-device copies, the codec kernels, and
    # device-to-host copies, so both PCIe directions and the kernels overlap; attention runs once every
    # chunk is encoded.  Events order each chunk's buffers between consecutive steps.
    nch = max(1, args.e2e_chunks)
    bounds = chunk_bounds(n, nch)
    s_cmp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nch)]
    ev_enc = [torch.cuda.Event() for _ in range(nch)]
    ev_dec = [torch.cuda.Event() for _ in range(nch)]
    ev_out = [torch.cuda.Event() for _ in range(nch)]
    ev_att, ev_q = torch.cuda.Event(), torch.cuda.Event()

    def e2e_step():
        for j in range(nch):
            r0, r1 = bounds[j], bounds[j + 1]
            s_in.wait_event(ev_enc[j])                    # the previous step's encoders are done with chunk j
            with torch.cuda.stream(s_in):
                k[r0:r1].copy_(k_host[r0:r1], non_blocking=True)
                v[r0:r1].copy_(v_host[r0:r1], non_blocking=True)
            ev_in[j].record(s_in)
        s_in.wait_event(ev_att)                           # the previous step's attention is done with q
        with torch.cuda.stream(s_in):
            q.copy_(q_host, non_blocking=True)
        ev_q.record(s_in)
        for j in range(nch):
            r0, r1 = bounds[j], bounds[j + 1]
            s_cmp.wait_event(ev_in[j])
            codec.encode_k(k[r0:r1], packed=kp[r0:r1], norms=kn[r0:r1])
            tq.encode_v(v[r0:r1], vb, vg, data=vd[r0:r1], scales=vsc[r0:r1], zeros=vz[r0:r1])
            ev_enc[j].record(s_cmp)
            s_cmp.wait_event(ev_out[j])                   # the previous step's copies of chunk j have left
            codec.decode_k(kp[r0:r1], kn[r0:r1], out=kdec[r0:r1])
            tq.decode_v(vd[r0:r1], vsc[r0:r1], vz[r0:r1], d, vb, vg, out=vdec[r0:r1])
            ev_dec[j].record(s_cmp)
        s_cmp.wait_event(ev_q)
        kernels[-1][1]()                                  # attention over the whole compressed cache
        ev_att.record(s_cmp)
        for j in range(nch):
            r0, r1 = bounds[j], bounds[j + 1]
            s_out.wait_event(ev_dec[j])
            with torch.cuda.stream(s_out):
                kdec_host[r0:r1].copy_(kdec[r0:r1], non_blocking=True)
                vdec_host[r0:r1].copy_(vdec[r0:r1], non_blocking=True)
            ev_out[j].record(s_out)
        s_out.wait_event(ev_att)
        with torch.cuda.stream(s_out):
            out_host.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_cmp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    done = torch.cuda.Event()
    done.record(s_out)
    s_cmp.wait_event(done)
    s_in_done = torch.cuda.Event()
    s_in_done.record(s_in)
    s_cmp.wait_event(s_in_done)
    e1.record(s_cmp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = (k_host.numel() + v_host.numel() + q_host.numel()) * 2
    d2h = (kdec_host.numel() + vdec_host.numel()) * 2 + out_host.numel() * 4
    if tq.read_device_flag() != 0:
        raise RuntimeError("a kernel raised the device error flag during timing")
    # kernels per call: one each for the codec calls; attention = query preparation + split kernel
    # (+ the split merge when the workspace holds split-K partials beyond the query fragments)
    qfrag_bytes = b * hkv * ((d // 16) * 32 + 2) * 16
    per_call = {"attend": 3 if ws.numel() > qfrag_bytes else 2}
    launches = sum(per_call.get(name, 1) for name, _, _ in events)
    fid = None
    if args.fidelity:
        # logits of the compressed path vs the exact fp16 ones, over every (sequence, query head) of the step
        from kv_cache_vector_norm_b200 import fidelity
        codec.encode_k(k, packed=kp, norms=kn)
        approx = tq.attend_scores(codec, q, cache, **{kk: vv for kk, vv in akw.items() if not kk.startswith("win_")})
        fid = fidelity.score_fidelity(approx, fidelity.exact_scores(q, k.view(b, hkv, t, d)))
    return dict(per=per, ms_per_step=ms_per_step, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, n=n,
                clocks=sampler.summary(), launches=launches, fidelity=fid)


# ----------------------------------------------------------------------------- bit-width sweep

def sweep_arm(args):
    """Encode and decode throughput of every key width (1..4 bits) and value width (2/3/4/8 bits, group 32
    and one group per token) on 2^24 fp16 N(0,1) vectors of d = 128, each launch with a cold L2, plus the
    measured key distortion mean ||x_hat - x||^2 / ||x||^2 against the codebook's D(b, d)."""
    import torch
    from kv_cache_vector_norm_b200 import synth, tq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n, d = args.sweep_rows, 128
    x = synth.normal_fp16(0, synth.STREAM_K, (n, d), device=dev)
    out = torch.empty(n, d, dtype=torch.float16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    hbm, peak_src = peaks()

    def timeit(fn):
        ms = []
        for i in range(args.warmup + args.steps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            if i >= args.warmup:
                ms.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ms)

    def entry(kind, bits, layout, bpv, ms):
        gbps = bpv * n / (ms / 1e3) / 1e9
        return {"kernel": kind, "bits": bits, "layout": layout, "us": ms * 1e3, "Mvectors_s": n / (ms / 1e3) / 1e6,
                "GBps": gbps, "frac_of_hbm": gbps / hbm, "bytes_per_vector": bpv}

    rows = []
    for kb in (1, 2, 3, 4):
        codec = tq.Codec(d, kb, 0)
        kp = torch.empty(n, d * kb // 8, dtype=torch.uint8, device=dev)
        kn = torch.empty(n, dtype=torch.float32, device=dev)
        bpv = 2 * d + d * kb // 8 + 4
        rows.append(entry("encode_k", kb, "-", bpv, timeit(lambda: codec.encode_k(x, packed=kp, norms=kn))))
        rows.append(entry("decode_k", kb, "-", bpv, timeit(lambda: codec.decode_k(kp, kn, out=out))))
        # evaluation of the round trip (not part of the timed path): mean relative squared error
        acc, cnt = 0.0, 0
        for r0 in range(0, n, 1 << 20):
            xf = x[r0:r0 + (1 << 20)].float()
            e = (out[r0:r0 + (1 << 20)].float() - xf).pow(2).sum(1) / xf.pow(2).sum(1).clamp_min(1e-30)
            acc += float(e.double().sum())
            cnt += e.numel()
        rows[-1]["mse_rel"] = acc / cnt
        rows[-1]["distortion_D_b_d"] = tq.build_codebook(d, kb)["distortion"]
        del codec, kp, kn
    for vb in (2, 3, 4, 8):
        for g in (32, d):
            vd = torch.empty(n, (d * vb + 7) // 8, dtype=torch.uint8, device=dev)
            vs = torch.empty(n, d // g, dtype=torch.float16, device=dev)
            vz = torch.empty(n, d // g, dtype=torch.float16, device=dev)
            bpv = 2 * d + (d * vb + 7) // 8 + 4 * (d // g)
            lay = "group32" if g == 32 else "token"
            rows.append(entry("encode_v", vb, lay, bpv,
                              timeit(lambda: tq.encode_v(x, vb, g, data=vd, scales=vs, zeros=vz))))
            rows.append(entry("decode_v", vb, lay, bpv,
                              timeit(lambda: tq.decode_v(vd, vs, vz, d, vb, g, out=out))))
            del vd, vs, vz
    if tq.read_device_flag() != 0:
        raise RuntimeError("a kernel raised the device error flag during the sweep")
    print(json.dumps({"mode": "bit-width sweep", "vectors": n, "head_dim": d, "data": "synthetic fp16 N(0,1), seed 0",
                      "l2": "flushed by a 256 MiB write before every launch", "steps": args.steps,
                      "hbm_peak_GBps": hbm, "peak_source": peak_src, "rows": rows}))


# ------------------------------------------------------------------------------------- CPU (oracle)

def oracle_sample(w, tokens, seed=0):
    """The oracle on one kv head's first `tokens` tokens of the workload: key and value encode and
    decode of those vectors, then attention of that kv head's query heads over them.  Returns
    seconds."""
    import numpy as np
    import torch
    from kv_cache_vector_norm_b200 import synth
    from oracle import tq_oracle as o

    d, kb, vb, vg = w["d"], w["k_bits"], w["v_bits"], w["v_group"]
    g = w["q_heads"] // w["kv_heads"]
    shape = (w["batch"], w["kv_heads"], w["tokens"], d)
    rows = torch.arange(tokens, dtype=torch.int64)
    ks = synth.channel_scales(seed, w["kv_heads"], d, "k", outlier_frac=w["outliers"])
    vs = synth.channel_scales(seed, w["kv_heads"], d, "v", outlier_frac=w["outliers"])
    k = synth.kv_rows(seed, synth.STREAM_K, shape, rows, scales=ks).numpy()
    v = synth.kv_rows(seed, synth.STREAM_V, shape, rows, scales=vs).numpy()
    q = synth.normal_fp16(seed, synth.STREAM_Q, (1, g, d)).numpy()
    pi = o.operational_rotation(d, 0)
    c, t = o.operational_codebook(d, kb)
    layout = "token" if vg == d else "group"
    t0 = time.perf_counter()
    idx, nrm, _ = o.encode_k(k, pi, t)
    packed = o.pack_lsb(idx, kb)
    nrm32 = nrm.astype(np.float32)
    data, s16, z16, _ = o.encode_v(v, vb, 32, layout)
    kidx = o.unpack_lsb(packed, kb, d)
    o.decode_k(kidx, nrm32.astype(np.float64), pi, c)
    vhat = o.decode_v(data, s16, z16, vb, d, 32, layout)
    o.attend(q, kidx[None, None], nrm32.astype(np.float64)[None, None], vhat[None, None], pi, c)
    return time.perf_counter() - t0


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, budget_s=15.0):
    probe = 2048
    dt = oracle_sample(w, probe)
    tokens = int(min(w["tokens"], max(probe, probe * budget_s / max(dt, 1e-3))))
    tokens = max(16, (tokens // 16) * 16)
    dt = oracle_sample(w, tokens)
    return {"value": tokens / dt / 1e6, "unit": "Mvectors/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"one kv head x {tokens} tokens of the workload: key+value encode and decode of {tokens} "
                      f"vectors each and attention of {w['q_heads'] // w['kv_heads']} query heads over them "
                      f"(fp64 numpy oracle, {dt:.1f} s)"}


# --------------------------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--workload", default="70b_decode_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fidelity", action="store_true",
                    help="also report the attention-score fidelity (cosine, top-1, top-5) of the workload's cache")
    ap.add_argument("--window", type=int, default=0,
                    help="recent uncompressed tokens per (sequence, kv head) attended beside the compressed cache")
    ap.add_argument("--rotation", default="haar", choices=["haar", "hadamard"],
                    help="key rotation: seeded Haar (default) or randomized Walsh-Hadamard; same kernels")
    ap.add_argument("--only", choices=["encode_k", "encode_v", "decode_k", "decode_v", "attend"],
                    help="time one kernel of the path alone (profiling aid; prints its per-launch times)")
    ap.add_argument("--sweep", action="store_true",
                    help="bit-width sweep instead of the step: encode/decode of every key and value width on "
                         "--sweep-rows vectors (one JSON line of per-kernel rows)")
    ap.add_argument("--sweep-rows", type=int, default=1 << 24)
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="row chunks of the end-to-end pass (host copies overlap the kernels across chunks)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's cache length (a multiple of 16; profiling aid for small captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = dict(WORKLOADS[args.workload])
    if args.tokens > 0:
        if args.tokens % 16:
            ap.error("--tokens must be a multiple of 16")
        w["tokens"] = args.tokens
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    bpv = algorithmic_bytes(w)
    config = {"workload": args.workload, "description": w["desc"], "batch": w["batch"], "kv_heads": w["kv_heads"],
              "q_heads": w["q_heads"], "tokens": w["tokens"], "head_dim": w["d"], "k_bits": w["k_bits"],
              "v_bits": w["v_bits"], "v_group": w["v_group"], "rotation": args.rotation, "window": args.window,
              "vector": "one (token, kv head) key/value pair through encode + decode + attention",
              "l2": "flushed by a 256 MiB write before every kernel launch (outside the timed interval)",
              "e2e": f"pinned host buffers, {max(1, args.e2e_chunks)} row chunks pipelined over host-to-device, kernel "
                     "and device-to-host streams",
              "parallelism": f"replicas x{world} (independent caches, no collective on the data path)"}

    if args.impl == "reference":
        if rank != 0:
            return
        total = args.steps + args.warmup
        per_step_budget = max(0.05, 150.0 / total)
        probe = 1024
        dt = oracle_sample(w, probe)
        tokens = int(max(16, min(w["tokens"], probe * per_step_budget / max(dt, 1e-4))) // 16 * 16)
        for _ in range(args.warmup):
            oracle_sample(w, tokens)
        times = [oracle_sample(w, tokens) for _ in range(args.steps)]
        ms = 1000.0 * sum(times) / len(times)
        value = tokens / (ms / 1000.0) / 1e6
        line = {"metric": METRIC, "value": value, "unit": "Mvectors/s", "impl": "reference", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64 (f32 for the value format)",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": "Mvectors/s", "cores": cpu_threads(), "kind": "oracle",
                                 "sample": f"one kv head x {tokens} tokens per step"},
                "e2e": {"value": value, "unit": "Mvectors/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if args.sweep:
        sweep_arm(args)
        return
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = gpu_arm(args, w, rank, world, local_rank)
    if args.only:
        if rank == 0:
            bpv_k = algorithmic_bytes(w)[args.only]
            ms = [round(x, 5) for x in r["launch_ms"]]
            print(json.dumps({"mode": "single-kernel", "kernel": args.only, "workload": args.workload,
                              "launch_ms": ms, "GBps_median": bpv_k * r["n"] / (statistics.median(ms) / 1e3) / 1e9}))
        return
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm, peak_src = peaks()
    n = r["n"]
    kern = {}
    for name, tot in r["per"].items():
        ms = tot / args.steps
        units = n if name != "attend" else n
        gbps = bpv[name] * units / (ms / 1000.0) / 1e9
        kern[name] = {"ms": ms, "Mvectors_s": units / (ms / 1000.0) / 1e6, "GBps": gbps, "frac_of_hbm": gbps / hbm,
                      "bytes_per_vector": bpv[name]}
    dom = max(kern, key=lambda x: kern[x]["ms"])
    value = job_value(world, n, r["ms_per_step"])
    line = {
        "metric": METRIC, "value": value, "unit": "Mvectors/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 in, f32 accumulate, u8 codes", "data": "synthetic (seeded, counter-based)",
        "config": config, "kernels": kern,
        "attend_GBps": kern["attend"]["GBps"], "attend_frac_of_hbm": kern["attend"]["frac_of_hbm"],
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["GBps"], "peak": hbm, "unit": "GB/s",
                     "frac": kern[dom]["GBps"] / hbm, "peak_source": peak_src,
                     "traffic": traffic_record(dom, args.workload),
                     "algorithmic_bytes_per_launch": bpv[dom] * n},
        "e2e": {"value": job_value(world, n, r["e2e_ms"]), "unit": "Mvectors/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"], "clocks": r["clocks"],
    }
    if r.get("fidelity") is not None:
        line["fidelity"] = r["fidelity"]
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
