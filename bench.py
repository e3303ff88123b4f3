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
    "paged_64x4096_d64": dict(kind="paged", batch=64, kv_heads=8, q_heads=32, tokens=4096, d=64, k_bits=4, v_bits=4,
                              v_group=32, outliers=0.0,
                              desc="high-concurrency paged cache: 64 sequences x 4096 tokens, 8 KV heads, head_dim 64, "
                                   "16-token blocks of a seeded permuted block table; K 4-bit / V 4-bit group 32 bulk "
                                   "encode through slots, decode of the pool, then one appended token per sequence "
                                   "and a decode-step attend of 32 query heads over 4097 tokens"),
    "paged_64x4096_d256": dict(kind="paged", batch=64, kv_heads=8, q_heads=32, tokens=4096, d=256, k_bits=4,
                               v_bits=4, v_group=32, outliers=0.0,
                               desc="high-concurrency paged cache: 64 sequences x 4096 tokens, 8 KV heads, head_dim "
                                    "256, 16-token blocks of a seeded permuted block table; K 4-bit / V 4-bit group 32 "
                                    "bulk encode through slots, decode of the pool, then one appended token per "
                                    "sequence and a decode-step attend of 32 query heads over 4097 tokens"),
    "k_roundtrip_4096": dict(kind="k_only", batch=1, kv_heads=1, q_heads=1, tokens=4096, d=128, k_bits=4, v_bits=2,
                             v_group=32, outliers=0.0, scaled=False,
                             desc="K-only round trip: 4096 key vectors, head_dim 128, fp16 N(0,1) iid, 4-bit codebook, "
                                  "one seeded 128x128 Haar rotation; encode to 64 B + f32 norm per vector, then "
                                  "decode"),
}


def algorithmic_bytes(w):
    """Bytes per unit of each launch: per vector for the codec calls (the appended token counts its key and
    value), per (token, kv head) for attention.  With QJL keys of k_bits total bits the key is the MSE stage at
    k_bits - 1 plus d/8 bytes of signs and a 4-byte residual norm; its decode reads the MSE stage only."""
    d, kb, vb, g = w["d"], w["k_bits"], w["v_bits"], w["v_group"]
    v = 2 * d + (d * vb + 7) // 8 + 4 * (d // g)
    vrow = (d * vb + 7) // 8 + 4 * (d // g)
    if w.get("qjl"):
        mse = d * (kb - 1) // 8 + 4
        k_enc = 2 * d + mse + d // 8 + 4
        return {"encode_k": k_enc, "decode_k": 2 * d + mse, "encode_v": v, "decode_v": v, "append": k_enc + v,
                "attend": mse + d // 8 + 4 + vrow}
    k = 2 * d + d * kb // 8 + 4
    att = (d * kb // 8 + 4) + vrow
    return {"encode_k": k, "decode_k": k, "encode_v": v, "decode_v": v, "append": k + v, "attend": att}


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
    "append": ("tq_device.cuh", "tq_codec_kernels.cuh", "tq_lib.cu"),
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
                # the sampler runs only while the timed launches are in flight: every sample counts
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self._reasons_fn(self.h) if self._reasons_fn else 0
                self.samples.append(mhz)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

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


def paged_slots(table, hkv: int, t: int):
    """Pool rows of a paged cache with 16-token blocks: (slots of tokens 0..t-1 in (sequence, kv head, token)
    order, slots of the appended token t in (sequence, kv head) order); row = (block * H_kv + h) * 16 + t % 16
    with block = table[sequence][t / 16]."""
    import torch
    dev = table.device
    tt = torch.arange(t, device=dev)
    hh = torch.arange(hkv, device=dev)
    blk = table[:, tt // 16].to(torch.int64)                                          # [b][t]
    slots = ((blk[:, None, :] * hkv + hh[None, :, None]) * 16 + (tt % 16)[None, None, :]).reshape(-1)
    nb = table[:, t // 16].to(torch.int64)                                            # [b]
    new_slots = ((nb[:, None] * hkv + hh[None, :]) * 16 + t % 16).reshape(-1)
    return slots, new_slots


def build_workload(w, dev, seed, rotation):
    """Device buffers and the calls of one step of the workload: the codec launches over row ranges (so the
    end-to-end pass can pipeline them in chunks) and the attention launch.

    kind "contiguous": the cache rows are (b * H_kv + h) * T + t; encode writes them in place.
    kind "paged": 16-token blocks; the block table is a seeded permutation of B * (T/16 + 1) physical blocks;
    encode scatters every token through its slot, decode reads the whole pool, and the attention step first
    appends one token per (sequence, kv head) through its slot, then attends over T + 1 tokens.
    kind "k_only": the key round trip (encode, decode) with no values and no attention.
    """
    import torch
    from kv_cache_vector_norm_b200 import synth, tq

    kind = w.get("kind", "contiguous")
    b, hkv, hq, t, d = w["batch"], w["kv_heads"], w["q_heads"], w["tokens"], w["d"]
    kb, vb, vg = w["k_bits"], w["v_bits"], w["v_group"]
    n_in = b * hkv * t
    has_v = kind != "k_only"
    scaled = w.get("scaled", True)
    ks = synth.channel_scales(seed, hkv, d, "k", outlier_frac=w["outliers"]) if scaled else None
    vs = synth.channel_scales(seed, hkv, d, "v", outlier_frac=w["outliers"]) if scaled else None
    k = synth.kv_tensor(seed, synth.STREAM_K, b, hkv, t, d, device=dev, scales=ks).view(n_in, d)
    v = synth.kv_tensor(seed, synth.STREAM_V, b, hkv, t, d, device=dev, scales=vs).view(n_in, d) if has_v else None
    q = synth.normal_fp16(seed, synth.STREAM_Q, (b, hq, d), device=dev) if has_v else None
    qjl = bool(w.get("qjl"))
    codec = tq.QjlCodec(d, kb, 0, rotation=rotation) if qjl else tq.Codec(d, kb, 0, rotation=rotation)
    kbm = kb - 1 if qjl else kb                           # bits of the stored codes
    slots = table = lens = k_new = v_new = new_slots = None
    if kind == "paged":
        per_seq = t // 16 + 1                             # room for the appended token
        table = synth.block_table(seed, b, per_seq, b * per_seq).to(dev)
        n_pool = b * per_seq * hkv * 16
        slots, new_slots = paged_slots(table, hkv, t)
        k_new = synth.normal_fp16(seed, 23, (b * hkv, d), device=dev)
        v_new = synth.normal_fp16(seed, 24, (b * hkv, d), device=dev)
        lens = torch.full((b,), t + 1, dtype=torch.int32, device=dev)
    else:
        n_pool = n_in
    kp = torch.zeros(n_pool, d * kbm // 8, dtype=torch.uint8, device=dev)
    kn = torch.zeros(n_pool, dtype=torch.float32, device=dev)
    ksg = torch.zeros(n_pool, d // 8, dtype=torch.uint8, device=dev) if qjl else None
    krho = torch.zeros(n_pool, dtype=torch.float32, device=dev) if qjl else None
    kdec = torch.empty(n_pool, d, dtype=torch.float16, device=dev)
    vd = vsc = vz = vdec = out = cache = ws = akw = None
    if has_v:
        vd = torch.zeros(n_pool, (d * vb + 7) // 8, dtype=torch.uint8, device=dev)
        vsc = torch.zeros(n_pool, d // vg, dtype=torch.float16, device=dev)
        vz = torch.zeros(n_pool, d // vg, dtype=torch.float16, device=dev)
        vdec = torch.empty(n_pool, d, dtype=torch.float16, device=dev)
        out = torch.empty(b, hq, d, dtype=torch.float32, device=dev)
        cache = tq.Cache(kp, kn, vd, vsc, vz)
        if kind == "paged":
            akw = dict(num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=None, block_table=table, seq_lens=lens,
                       scale=0.0)
        else:
            akw = dict(num_kv_heads=hkv, v_bits=vb, v_group=vg, max_seq_len=t, block_table=None, seq_lens=None,
                       scale=0.0)
        ws = tq.attend_workspace(codec, q, cache, **akw)
        if qjl:
            a0 = tq._attend_args(codec, q, cache, out=None, workspace=None, **akw)
            import ctypes
            nb = ctypes.c_size_t()
            tq.LIB.tq_attend_qjl_workspace_bytes(ctypes.byref(a0), ctypes.byref(nb))
            ws = torch.empty(max(16, nb.value), dtype=torch.uint8, device=dev)

    def enc_k(r0, r1):
        if qjl:
            if slots is None:
                codec.encode_k_qjl(k[r0:r1], packed=kp[r0:r1], norms=kn[r0:r1], signs=ksg[r0:r1], rho=krho[r0:r1])
            else:
                codec.encode_k_qjl(k[r0:r1], slot_mapping=slots[r0:r1], packed=kp, norms=kn, signs=ksg, rho=krho)
        elif slots is None:
            codec.encode_k(k[r0:r1], packed=kp[r0:r1], norms=kn[r0:r1])
        else:
            codec.encode_k(k[r0:r1], slot_mapping=slots[r0:r1], packed=kp, norms=kn)

    def enc_v(r0, r1):
        if slots is None:
            tq.encode_v(v[r0:r1], vb, vg, data=vd[r0:r1], scales=vsc[r0:r1], zeros=vz[r0:r1])
        else:
            tq.encode_v(v[r0:r1], vb, vg, slot_mapping=slots[r0:r1], data=vd, scales=vsc, zeros=vz)

    def dec_k(r0, r1):
        codec.decode_k(kp[r0:r1], kn[r0:r1], out=kdec[r0:r1])

    def dec_v(r0, r1):
        tq.decode_v(vd[r0:r1], vsc[r0:r1], vz[r0:r1], d, vb, vg, out=vdec[r0:r1])

    def append():
        if qjl:
            codec.encode_k_qjl(k_new, slot_mapping=new_slots, packed=kp, norms=kn, signs=ksg, rho=krho)
        else:
            codec.encode_k(k_new, slot_mapping=new_slots, packed=kp, norms=kn)
        tq.encode_v(v_new, vb, vg, slot_mapping=new_slots, data=vd, scales=vsc, zeros=vz)

    def attend():
        if qjl:
            tq.attend_decode_qjl(codec, q, cache, ksg, krho, out=out, workspace=ws, **akw)
        else:
            tq.attend_decode(codec, q, cache, out=out, workspace=ws, **akw)

    kernels = [("encode_k", lambda: enc_k(0, n_in))]
    if has_v:
        kernels.append(("encode_v", lambda: enc_v(0, n_in)))
    kernels.append(("decode_k", lambda: dec_k(0, n_pool)))
    if has_v:
        kernels.append(("decode_v", lambda: dec_v(0, n_pool)))
    if kind == "paged":
        kernels.append(("append", append))
    if has_v:
        kernels.append(("attend", attend))
    att_tokens = (t + 1) if kind == "paged" else t
    # launches per call: one for each codec call; attention = query preparation + split kernel (+ the split
    # merge when the workspace holds split-K partials beyond the query fragments)
    qfrag_bytes = b * hkv * ((d // 16) * 32 + 2) * 16 * (2 if qjl else 1)
    per_call = {"append": 3 if qjl else 2, "attend": (3 if ws.numel() > qfrag_bytes else 2) if has_v else 0,
                "encode_k": 2 if qjl else 1}
    return dict(kind=kind, n_in=n_in, n_pool=n_pool, att_units=b * hkv * att_tokens, kernels=kernels,
                per_call=per_call, enc_k=enc_k, enc_v=enc_v, dec_k=dec_k, dec_v=dec_v, append=append, attend=attend,
                k=k, v=v, q=q, k_new=k_new, v_new=v_new, kdec=kdec, vdec=vdec, out=out, has_v=has_v,
                codec=codec, cache=cache, akw=akw, kp=kp, kn=kn)


def kernel_units(wl, w):
    """Units each timed call processes: vectors for the codec calls, (token, kv head) pairs for attention."""
    return {"encode_k": wl["n_in"], "encode_v": wl["n_in"], "decode_k": wl["n_pool"], "decode_v": wl["n_pool"],
            "append": w["batch"] * w["kv_heads"], "attend": wl["att_units"]}


def gpu_arm(args, w, rank, world, local_rank):
    import torch
    from kv_cache_vector_norm_b200 import tq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = build_workload(w, dev, rank, args.rotation)
    if args.window > 0 and wl["kind"] == "contiguous":
        # recent uncompressed tokens beside the compressed cache ("KV Cache API" store.py buffer)
        from kv_cache_vector_norm_b200 import synth
        b, hkv, d = w["batch"], w["kv_heads"], w["d"]
        win_k = synth.normal_fp16(0, 21, (b, hkv, args.window, d), device=dev)
        win_v = synth.normal_fp16(0, 22, (b, hkv, args.window, d), device=dev)
        akw = wl["akw"]
        ws = tq.attend_window_workspace(wl["codec"], wl["q"], wl["cache"], win_k, win_v, None, **akw)
        out, codec, q, cache = wl["out"], wl["codec"], wl["q"], wl["cache"]
        wl["attend"] = lambda: tq.attend_decode(codec, q, cache, out=out, workspace=ws, win_k=win_k, win_v=win_v,
                                                **akw)
        wl["kernels"][-1] = ("attend", wl["attend"])
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    kernels = wl["kernels"]
    if args.only:
        if args.only in ("decode_k", "decode_v", "attend", "append"):
            # the compressed cache these kernels read is written once, outside the timed launches
            for name, fn in kernels:
                if name.startswith("encode"):
                    fn()
        kernels = [kv for kv in kernels if kv[0] == args.only]
        if not kernels:
            raise SystemExit(f"--only {args.only}: the workload has no such kernel")

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
        import torch.distributed as dist
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
        return dict(per=per, launch_ms=[e0.elapsed_time(e1) for _, e0, e1 in events], wl=wl)
    total_ms = max_over_ranks(sum(per.values()), world, dev)
    ms_per_step = total_ms / args.steps
    e2e_ms, h2d, d2h = e2e_pass(args, wl, world, dev)
    if tq.read_device_flag() != 0:
        raise RuntimeError("a kernel raised the device error flag during timing")
    launches = sum(wl["per_call"].get(name, 1) for name, _, _ in events)
    fid = None
    if args.fidelity and wl["has_v"] and wl["kind"] == "contiguous":
        # logits of the compressed path vs the exact fp16 ones, over every (sequence, query head) of the step
        from kv_cache_vector_norm_b200 import fidelity
        b, hkv, t, d = w["batch"], w["kv_heads"], w["tokens"], w["d"]
        wl["enc_k"](0, wl["n_in"])
        approx = tq.attend_scores(wl["codec"], wl["q"], wl["cache"], **wl["akw"])
        fid = fidelity.score_fidelity(approx, fidelity.exact_scores(wl["q"], wl["k"].view(b, hkv, t, d)))
    return dict(per=per, ms_per_step=ms_per_step, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, wl=wl,
                clocks=sampler.summary(), launches=launches, fidelity=fid)


def e2e_pass(args, wl, world, dev):
    """The same step through host buffers: every step copies the inputs (keys, values, query, appended token)
    from pinned host memory and the results (decoded keys and values, attention output) back, inside the timed
    interval.  The cache moves in row chunks on three streams -- host-to-device copies, the codec kernels and
    device-to-host copies -- so both PCIe directions overlap the kernels; attention runs once every chunk is
    encoded.  Events order each chunk's buffers between consecutive steps.  Returns (ms per step, H2D bytes,
    D2H bytes per step)."""
    import torch

    has_v = wl["has_v"]
    ins = [x for x in (wl["k"], wl["v"]) if x is not None]
    small_in = [x for x in (wl["q"], wl["k_new"], wl["v_new"]) if x is not None]
    outs = [x for x in (wl["kdec"], wl["vdec"]) if x is not None]
    ins_h = [x.cpu().pin_memory() for x in ins]
    small_h = [x.cpu().pin_memory() for x in small_in]
    outs_h = [torch.empty_like(x, device="cpu").pin_memory() for x in outs]
    out_h = torch.empty_like(wl["out"], device="cpu").pin_memory() if has_v else None
    e2e_steps = max(3, min(args.steps, 20))
    nch = max(1, args.e2e_chunks)
    bin_, bpool = chunk_bounds(wl["n_in"], nch), chunk_bounds(wl["n_pool"], nch)
    s_cmp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nch)]
    ev_dec = [torch.cuda.Event() for _ in range(nch)]
    ev_out = [torch.cuda.Event() for _ in range(nch)]
    ev_enc_all, ev_att, ev_small = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
    ev_enc_all.record(s_cmp)
    ev_att.record(s_cmp)

    def step():
        s_in.wait_event(ev_enc_all)                       # the previous step's encoders are done with the inputs
        for j in range(nch):
            r0, r1 = bin_[j], bin_[j + 1]
            with torch.cuda.stream(s_in):
                for x, xh in zip(ins, ins_h):
                    x[r0:r1].copy_(xh[r0:r1], non_blocking=True)
            ev_in[j].record(s_in)
        s_in.wait_event(ev_att)                           # the previous step's attention is done with q
        with torch.cuda.stream(s_in):
            for x, xh in zip(small_in, small_h):
                x.copy_(xh, non_blocking=True)
        ev_small.record(s_in)
        def decode(j):
            r0, r1 = bpool[j], bpool[j + 1]
            s_cmp.wait_event(ev_out[j])                   # the previous step's copies of chunk j have left
            wl["dec_k"](r0, r1)
            if has_v:
                wl["dec_v"](r0, r1)
            ev_dec[j].record(s_cmp)

        # contiguous rows: chunk j decodes as soon as it is encoded; a scatter through slots can write any pool
        # row, so the paged pool is decoded after every chunk is encoded
        interleave = wl["kind"] != "paged"
        for j in range(nch):
            r0, r1 = bin_[j], bin_[j + 1]
            s_cmp.wait_event(ev_in[j])
            wl["enc_k"](r0, r1)
            if has_v:
                wl["enc_v"](r0, r1)
            if interleave:
                decode(j)
        ev_enc_all.record(s_cmp)
        if not interleave:
            for j in range(nch):
                decode(j)
        if has_v:
            s_cmp.wait_event(ev_small)
            if wl["kind"] == "paged":
                wl["append"]()
            wl["attend"]()
        ev_att.record(s_cmp)
        for j in range(nch):
            r0, r1 = bpool[j], bpool[j + 1]
            s_out.wait_event(ev_dec[j])
            with torch.cuda.stream(s_out):
                for x, xh in zip(outs, outs_h):
                    xh[r0:r1].copy_(x[r0:r1], non_blocking=True)
            ev_out[j].record(s_out)
        if has_v:
            s_out.wait_event(ev_att)
            with torch.cuda.stream(s_out):
                out_h.copy_(wl["out"], non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_cmp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(e2e_steps):
        step()
    for s in (s_in, s_out):
        ev = torch.cuda.Event()
        ev.record(s)
        s_cmp.wait_event(ev)
    e1.record(s_cmp)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = sum(x.numel() * x.element_size() for x in ins_h + small_h)
    d2h = sum(x.numel() * x.element_size() for x in outs_h) + (out_h.numel() * 4 if has_v else 0)
    return ms, h2d, d2h


# ----------------------------------------------------------------------------- bit-width sweep

def sweep_arm(args):
    """Encode and decode throughput of every key width (1..8 bits; --sweep-key-bits) and value width (2/3/4/8
    bits, group 32 and one group per token) on 2^24 fp16 N(0,1) vectors of d = 128, each launch with a cold L2,
    plus the measured key distortion mean ||x_hat - x||^2 / ||x||^2 against the codebook's D(b, d)."""
    import torch
    from kv_cache_vector_norm_b200 import synth, tq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n, d = args.sweep_rows, 128
    x = synth.normal_fp16(0, synth.STREAM_K, (n, d), device=dev)
    out = torch.empty(n, d, dtype=torch.float16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    hbm, peak_src = peaks()

    all_reasons = set()

    def timeit(fn):
        # returns (median ms, clocks seen while those launches ran)
        ms = []
        sampler = ClockSampler(0)
        with sampler:
            for i in range(args.warmup + args.steps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                if i >= args.warmup:
                    ms.append((e0, e1))
            torch.cuda.synchronize()
        all_reasons.update(sampler.reasons)
        return statistics.median(a.elapsed_time(b) for a, b in ms), sampler.summary()

    def entry(kind, bits, layout, bpv, timed):
        ms, clk = timed
        gbps = bpv * n / (ms / 1e3) / 1e9
        return {"kernel": kind, "bits": bits, "layout": layout, "us": ms * 1e3, "Mvectors_s": n / (ms / 1e3) / 1e6,
                "GBps": gbps, "frac_of_hbm": gbps / hbm, "bytes_per_vector": bpv, "sm_mhz": clk["sm_mhz"]}

    rows = []
    for kb in args.sweep_key_bits:
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
                      "hbm_peak_GBps": hbm, "peak_source": peak_src,
                      "clocks": {"sm_max_mhz": ClockSampler(0).max_mhz, "reasons": sorted(all_reasons)},
                      "rows": rows}))


# ------------------------------------------------------------------------------------- CPU (oracle)

def oracle_sample(w, tokens, seed=0, head=0):
    """The oracle on kv head `head`'s first `tokens` tokens of the workload: key (and value) encode and decode
    of those vectors, then attention of that kv head's query heads over them (the key round trip only for the
    K-only workload; the paged layout permutes rows, not arithmetic, so contiguous rows stand in for it).
    Returns seconds."""
    import numpy as np
    import torch
    from kv_cache_vector_norm_b200 import synth
    from oracle import tq_oracle as o

    d, kb, vb, vg = w["d"], w["k_bits"], w["v_bits"], w["v_group"]
    g = w["q_heads"] // w["kv_heads"]
    has_v = w.get("kind", "contiguous") != "k_only"
    shape = (w["batch"], w["kv_heads"], w["tokens"], d)
    head = head % (w["batch"] * w["kv_heads"])
    rows = head * w["tokens"] + torch.arange(tokens, dtype=torch.int64)
    scaled = w.get("scaled", True)
    ks = synth.channel_scales(seed, w["kv_heads"], d, "k", outlier_frac=w["outliers"]) if scaled else None
    vs = synth.channel_scales(seed, w["kv_heads"], d, "v", outlier_frac=w["outliers"]) if scaled else None
    k = synth.kv_rows(seed, synth.STREAM_K, shape, rows, scales=ks).numpy()
    v = synth.kv_rows(seed, synth.STREAM_V, shape, rows, scales=vs).numpy() if has_v else None
    q = synth.normal_fp16(seed, synth.STREAM_Q, (1, g, d)).numpy()
    qjl = bool(w.get("qjl"))
    kbm = kb - 1 if qjl else kb
    pi = o.operational_rotation(d, 0)
    c, t = o.operational_codebook(d, kbm)
    s_op = o.operational_qjl_matrix(d, 0) if qjl else None
    layout = "token" if vg == d else "group"
    t0 = time.perf_counter()
    if qjl:
        idx, nrm, _, sbits, rho, _ = o.encode_k_qjl(k, pi, c, t, s_op)
        signs = o.pack_lsb(sbits.astype(np.int64), 1)
    else:
        idx, nrm, _ = o.encode_k(k, pi, t)
    packed = o.pack_lsb(idx, kbm)
    nrm32 = nrm.astype(np.float32)
    kidx = o.unpack_lsb(packed, kbm, d)
    o.decode_k(kidx, nrm32.astype(np.float64), pi, c)
    if has_v:
        data, s16, z16, _ = o.encode_v(v, vb, 32, layout)
        vhat = o.decode_v(data, s16, z16, vb, d, 32, layout)
        n64 = nrm32.astype(np.float64)[None, None]
        if qjl:
            bits = o.unpack_lsb(signs, 1, d).astype(bool)
            o.attend_qjl(q, kidx[None, None], n64, bits[None, None], rho.astype(np.float32).astype(np.float64)[None, None],
                         vhat[None, None], pi, c, s_op)
        else:
            o.attend(q, kidx[None, None], n64, vhat[None, None], pi, c)
    return time.perf_counter() - t0


def _limit_blas_threads(n=1):
    """Keep numpy's BLAS pool at n threads in this process (so one process is one busy core)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=n)
    except Exception:
        return None


def _oracle_worker(w, tokens, head, barrier):
    """One process of the multi-process CPU baseline: a warm-up sample, then a timed one started together
    with the other processes.  Returns (start, end) wall-clock seconds of the timed sample."""
    _limit_blas_threads(1)
    oracle_sample(w, min(tokens, 256), head=head)
    barrier.wait()
    t0 = time.time()
    oracle_sample(w, tokens, head=head)
    return t0, time.time()


def cpu_baseline(w, budget_s=10.0):
    """The oracle as it stands, timed on the host cores: one process on one core (BLAS limited to one thread),
    then one process per core each on its own kv head's slice, started together; the rate of the second is the
    reported value.  Both are extrapolated from the bounded samples they time (Mvectors/s of the sample)."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor

    lim = _limit_blas_threads(1)
    probe = 1024
    dt = oracle_sample(w, probe)
    tokens = int(min(w["tokens"], max(probe, probe * budget_s / max(dt, 1e-3))))
    tokens = max(16, (tokens // 16) * 16)
    dt1 = oracle_sample(w, tokens)
    if lim is not None:
        lim.restore_original_limits()
    single = tokens / dt1 / 1e6
    procs = max(1, os.cpu_count() or 1)
    ctx = mp.get_context("spawn")                     # after CUDA work a forked child would hang
    multi, span = None, None
    try:
        with ctx.Manager() as mgr:
            barrier = mgr.Barrier(procs)
            with ProcessPoolExecutor(max_workers=procs, mp_context=ctx) as ex:
                futs = [ex.submit(_oracle_worker, w, tokens, i, barrier) for i in range(procs)]
                spans = [f.result(timeout=600) for f in futs]
        span = max(e for _, e in spans) - min(s for s, _ in spans)
        multi = procs * tokens / span / 1e6
    except Exception as exc:                          # report the single-core figure if the pool cannot run
        sys.stderr.write(f"multi-process CPU baseline skipped: {exc}\n")
    what = ("key encode and decode" if w.get("kind") == "k_only" else
            f"key+value encode and decode and attention of {w['q_heads'] // w['kv_heads']} query heads")
    out = {"value": multi if multi is not None else single, "unit": "Mvectors/s",
           "cores": procs if multi is not None else 1, "kind": "oracle",
           "sample": (f"{procs if multi is not None else 1} process(es), one core each (BLAS limited to one thread), "
                      f"each on one kv head x {tokens} tokens of the workload ({what}); rate extrapolated from "
                      f"that bounded sample, fp64 numpy oracle"),
           "single_core": {"value": single, "seconds": dt1, "tokens": tokens}}
    if multi is not None:
        out["multi_process"] = {"value": multi, "processes": procs, "seconds": span}
    return out


def _oracle_step(w, tokens, head):
    _limit_blas_threads(1)
    t0 = time.time()
    oracle_sample(w, tokens, head=head)
    return t0, time.time()


def reference_arm(args, w, config):
    """The oracle as the reference arm: each step runs one bounded sample per host core (one process per core,
    BLAS limited to one thread, each on its own kv head's slice), sized so the whole run ends in a few minutes;
    the step's time is the wall-clock span of its processes."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor

    total = args.steps + args.warmup
    per_step_budget = max(0.05, 150.0 / total)
    _limit_blas_threads(1)
    probe = 1024
    dt = oracle_sample(w, probe)
    tokens = int(max(16, min(w["tokens"], probe * per_step_budget / max(dt, 1e-4))) // 16 * 16)
    procs = max(1, os.cpu_count() or 1)
    ctx = mp.get_context("spawn")
    spans = []
    with ProcessPoolExecutor(max_workers=procs, mp_context=ctx) as ex:
        for i in range(total):
            res = [f.result() for f in [ex.submit(_oracle_step, w, tokens, j) for j in range(procs)]]
            if i >= args.warmup:
                spans.append(max(e for _, e in res) - min(s for s, _ in res))
    ms = 1000.0 * sum(spans) / len(spans)
    value = procs * tokens / (ms / 1000.0) / 1e6
    sample = (f"{procs} processes, one core each (BLAS limited to one thread), each on one kv head x {tokens} "
              f"tokens of the workload per step; fp64 numpy oracle")
    return {"metric": METRIC, "value": value, "unit": "Mvectors/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (f32 for the value format)",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": "Mvectors/s", "cores": procs, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mvectors/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


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
    ap.add_argument("--sweep-key-bits", type=lambda v: [int(x) for x in v.split(",")], default=[1, 2, 3, 4, 5, 6, 7, 8],
                    help="key widths of the sweep (comma-separated)")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="row chunks of the end-to-end pass (host copies overlap the kernels across chunks)")
    ap.add_argument("--qjl", action="store_true",
                    help="QJL residual keys of the workload's key bits (MSE stage at bits - 1 + sign sketch)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's cache length (a multiple of 16; profiling aid for small captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = dict(WORKLOADS[args.workload])
    if args.qjl:
        w["qjl"] = True
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
              "qjl": bool(w.get("qjl")),
              "vector": "one (token, kv head) key/value pair through encode + decode + attention",
              "l2": "flushed by a 256 MiB write before every kernel launch (outside the timed interval)",
              "e2e": f"pinned host buffers, {max(1, args.e2e_chunks)} row chunks pipelined over host-to-device, kernel "
                     "and device-to-host streams",
              "parallelism": f"replicas x{world} (independent caches, no collective on the data path)"}

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(args, w, config)))
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
            units = kernel_units(r["wl"], w)[args.only]
            print(json.dumps({"mode": "single-kernel", "kernel": args.only, "workload": args.workload,
                              "launch_ms": ms, "GBps_median": bpv_k * units / (statistics.median(ms) / 1e3) / 1e9}))
        return
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm, peak_src = peaks()
    n = r["wl"]["n_in"]
    units_of = kernel_units(r["wl"], w)
    kern = {}
    for name, tot in r["per"].items():
        ms = tot / args.steps
        units = units_of[name]
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
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["GBps"], "peak": hbm, "unit": "GB/s",
                     "frac": kern[dom]["GBps"] / hbm, "peak_source": peak_src,
                     "traffic": traffic_record(dom, args.workload),
                     "algorithmic_bytes_per_launch": bpv[dom] * units_of[dom]},
        "e2e": {"value": job_value(world, n, r["e2e_ms"]), "unit": "Mvectors/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"], "clocks": r["clocks"],
    }
    if "attend" in kern:
        line["attend_GBps"] = kern["attend"]["GBps"]
        line["attend_frac_of_hbm"] = kern["attend"]["frac_of_hbm"]
    if r.get("fidelity") is not None:
        line["fidelity"] = r["fidelity"]
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
