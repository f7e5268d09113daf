#!/usr/bin/env python3
"""Benchmark of the transformed-KV 2-bit decode hot path on B200.

One step = one decode step of the serving loop on the Qwen3-8B-shaped high-concurrency
workload (batch 64, 32 query / 8 KV heads, head_dim 128, ragged contexts uniform in
[12288, 16384], 2-bit keys and values, group 128, bf16 queries and output):
    kvq_quantize_append  the newest token of every sequence (transform, clip, quantize,
                         pack) at position seqlen_b - 1
    kvq_decode_attention over positions [0, seqlen_b) of every sequence
All inputs are seeded synthetic stand-ins (tests/synth.py) for Qwen3-8B activations.
The cache (~530 MB) is larger than the 126 MB L2, so no flush is needed between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
Under torchrun (N > 1) every rank runs its own batch (weak scaling, no collective on the
data path); timing is the max over ranks. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tests import synth  # noqa: E402  (seeded input generators only)

METRIC = "2-bit KV decode attention: achieved HBM GB/s and % of B200 peak; append tok/s"
CONFIG_IDX = 2
# dram__bytes_read.sum + dram__bytes_write.sum of one decode_kernel launch on this workload
# (ncu --set full --clock-control none, profiles directory); None once the kernel changes.
DECODE_TRAFFIC_BYTES = 546806272
DECODE_TRAFFIC_KERNEL = "decode_kernel<128,4,2,2>"
APPEND_CONFIG_IDX = 4
DECODE_CONFIGS = (1, 3, 4)       # further decode shapes timed as extras


def step_bytes(cfg, seqlens):
    """Algorithmic bytes of one step.

    decode: sum_b seqlen_b * Hkv * (d*bk/8 + 4*d/g + d*bv/8 + 4*d/g) + q + out
    append: new k, v (bf16) + their codes and (s, z) + T_k, T_v once
    """
    ng = cfg.d // cfg.group
    per_tok = cfg.Hkv * (cfg.d * cfg.bits_k // 8 + 4 * ng + cfg.d * cfg.bits_v // 8 + 4 * ng)
    qo = 2 * cfg.B * cfg.Hq * cfg.d * 2
    decode = int(np.sum(seqlens)) * per_tok + qo
    append = cfg.B * cfg.Hkv * (2 * cfg.d * 2) + cfg.B * per_tok + 2 * cfg.Hkv * cfg.d * cfg.d * 4
    return decode, append


def reduce_max(x: float, world: int, device="cpu") -> float:
    """Max of a per-rank scalar over all ranks (the timing rule: slowest rank counts)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_gbs(bytes_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job GB/s: every rank processes its own batch of the same size, so the job
    moves world * bytes_per_rank per step in the slowest rank's step time."""
    return world * bytes_per_rank / (ms_per_step_max * 1e-3) / 1e9


def rank_sequence_offset(b: int, rank: int, B: int) -> int:
    """Index of the synthetic sequence that rank `rank` uses as its sequence b."""
    return b + rank * B


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows
                                    if r[3].replace(".", "").isdigit()), default=None)}


# ----------------------------------------------------------------------------- GPU workload

class Workload:
    """Config-2 cache built by the library's own quantize-append, plus step inputs."""

    def __init__(self, cfg, rank, device, with_bf16=True):
        import torch
        import decode_attention_post_b200 as kvq
        self.cfg, self.dev = cfg, device
        self.qp = kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)
        self.cache = kvq.KVCache.allocate(cfg.B, cfg.Hkv, cfg.T_cap, cfg.d, self.qp, device=device)
        self.seqlens = synth.seqlens(cfg)
        Tk, Tv, Tit = synth.transforms(cfg)
        g = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.Tk, self.Tv, self.Tit = g(Tk), g(Tv), g(Tit)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device).to(torch.bfloat16)
        self.kb = self.vb = None
        if with_bf16:
            self.kb = torch.zeros((cfg.B, cfg.Hkv, cfg.T_cap, cfg.d), dtype=torch.bfloat16,
                                  device=device)
            self.vb = torch.zeros_like(self.kb)
        knew = np.empty((cfg.B, 1, cfg.Hkv, cfg.d), np.float32)
        vnew = np.empty_like(knew)
        zero = torch.zeros(1, dtype=torch.int32, device=device)
        for b in range(cfg.B):
            n = int(self.seqlens[b])
            src = rank_sequence_offset(b, rank, cfg.B)   # each rank its own sequences
            k = synth.keys(cfg, src, 0, n)
            v = synth.values(cfg, src, 0, n)
            kd, vd = bf(k), bf(v)                        # [n][Hkv][d] bf16
            view = self.cache.view_sequence(b)
            kvq.quantize_append(kd[None], vd[None], self.Tk, self.Tv, self.qp, view, zero)
            if with_bf16:
                self.kb[b, :, :n] = kd.transpose(0, 1)
                self.vb[b, :, :n] = vd.transpose(0, 1)
            knew[b, 0] = k[n - 1]
            vnew[b, 0] = v[n - 1]
        self.knew, self.vnew = bf(knew), bf(vnew)
        self.q = bf(synth.queries(cfg))
        self.pos = g(self.seqlens - 1)
        self.seq_d = g(self.seqlens)
        self.max_seqlen = cfg.T_cap
        self.out = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(kvq.decode_workspace_bytes(self.cache, cfg.Hq, self.max_seqlen),
                              dtype=torch.uint8, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        torch.cuda.synchronize()

    def append(self):
        import decode_attention_post_b200 as kvq
        kvq.quantize_append(self.knew, self.vnew, self.Tk, self.Tv, self.qp, self.cache, self.pos,
                            n=1, dev_err=self.err)

    def decode(self):
        import decode_attention_post_b200 as kvq
        kvq.decode_attention(self.q, self.Tit, self.cache, self.seq_d, self.max_seqlen, self.out,
                             self.ws, dev_err=self.err)

    def step(self):
        self.append()
        self.decode()


class E2EStep:
    """One serving step through the public API with host buffers. Two pinned host staging
    buffers: the append's inputs (the new token's k and v, positions) and the decode's
    (q, seqlens). The append's buffer is copied first and the append starts as soon as it
    lands, while the decode's buffer is copied on a second stream; the decode waits for
    both; the bf16 output is copied back to pinned host memory. The sequence is captured
    once in a CUDA graph and replayed."""

    def __init__(self, w):
        import torch
        self.w = w
        self.side = torch.cuda.Stream(device=w.dev)

        def staging(parts):
            sizes = [t.numel() * t.element_size() for t in parts]
            offs = np.concatenate([[0], np.cumsum([(n + 255) // 256 * 256 for n in sizes])])
            dev = torch.empty(int(offs[-1]), dtype=torch.uint8, device=w.dev)
            host = torch.empty(int(offs[-1]), dtype=torch.uint8).pin_memory()
            views = []
            for t, o, n in zip(parts, offs[:-1], sizes):
                hv = host[int(o):int(o) + n].view(t.dtype).view(t.shape)
                hv.copy_(t.cpu())
                views.append(dev[int(o):int(o) + n].view(t.dtype).view(t.shape))
            return dev, host, views, int(sum(sizes))

        self.app_d, self.app_h, (self.knew, self.vnew, self.pos), na = staging(
            [w.knew, w.vnew, w.pos])
        self.dec_d, self.dec_h, (self.q, self.seq_d), nd = staging([w.q, w.seq_d])
        self.out_h = torch.empty(w.out.shape, dtype=w.out.dtype).pin_memory()
        self.h2d_bytes = na + nd
        self.d2h_bytes = self.out_h.numel() * self.out_h.element_size()

    def step(self):
        import torch
        import decode_attention_post_b200 as kvq
        w = self.w
        main = torch.cuda.current_stream()
        self.app_d.copy_(self.app_h, non_blocking=True)
        self.side.wait_stream(main)                 # the decode inputs follow the append's
        with torch.cuda.stream(self.side):
            self.dec_d.copy_(self.dec_h, non_blocking=True)
        kvq.quantize_append(self.knew, self.vnew, w.Tk, w.Tv, w.qp, w.cache, self.pos, n=1,
                            dev_err=w.err)
        main.wait_stream(self.side)
        kvq.decode_attention(self.q, w.Tit, w.cache, self.seq_d, w.max_seqlen, w.out, w.ws,
                             dev_err=w.err)
        self.out_h.copy_(w.out, non_blocking=True)

    def copies(self):
        """The step's host<->device copies alone, in the same streams and order."""
        import torch
        main = torch.cuda.current_stream()
        self.app_d.copy_(self.app_h, non_blocking=True)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self.dec_d.copy_(self.dec_h, non_blocking=True)
        main.wait_stream(self.side)
        self.out_h.copy_(self.w.out, non_blocking=True)

    def time(self, iters, stream, barrier, fn=None):
        import torch
        fn = fn or self.step
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        del g
        return e0.elapsed_time(e1) / iters


def time_events(fn, iters, stream, per_graph=1):
    """Mean device time of one fn() call: fn is captured `per_graph` times into a CUDA
    graph, each replay is bracketed by CUDA events on the launching stream, so host
    launch overhead does not leak into the measurement."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(per_graph):
            fn()
    g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for a, b in evs:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) / per_graph for a, b in evs]
    del g
    return times


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import decode_attention_post_b200 as kvq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(device))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, device)

    cfg = synth.CONFIGS[CONFIG_IDX]
    w = Workload(cfg, rank, device, with_bf16=not args.no_extras)
    stream = torch.cuda.current_stream()
    dec_bytes, app_bytes = step_bytes(cfg, w.seqlens)

    # ---- warm-up, then capture one step in a CUDA graph (3 kernels per replay)
    for _ in range(max(args.warmup, 3)):
        w.step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        w.step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, barrier + synchronize on both sides
    K = args.steps
    sampler = ClockSampler(local)
    with sampler:
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(K):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = sampler.summary()
    ms_total = max_over_ranks(t0.elapsed_time(t1))
    ms_step = ms_total / K
    value = weak_scaling_gbs(dec_bytes + app_bytes, ms_step, world)

    # ---- the dominant kernel (the decode call: q prologue + split-K decode) timed alone
    dec_ms = statistics.mean(time_events(w.decode, min(K, 500), stream))
    app_ms = statistics.mean(time_events(w.append, min(K, 200), stream, per_graph=20))
    dec_ms = max_over_ranks(dec_ms)
    peak, peak_kind = peaks()
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    dev_err = int(w.err.item())

    # ---- end to end through the public API: the step's inputs (q, the new token's k and
    #      v, seqlens, positions) packed in one pinned host buffer and moved by one
    #      host->device copy, the step, and the output read back to pinned host memory;
    #      the whole sequence is replayed as a CUDA graph
    e2e = E2EStep(w)
    e2e_ms = max_over_ranks(e2e.time(min(K, 500), stream, barrier))
    copies_ms = max_over_ranks(e2e.time(min(K, 500), stream, barrier, fn=e2e.copies))
    e2e_value = weak_scaling_gbs(dec_bytes + app_bytes, e2e_ms, world)
    h2d, d2h = e2e.h2d_bytes, e2e.d2h_bytes

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "2-bit codes -> int8 mma (keys), f16 mma (values), f32 softmax", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                   "T_cap": cfg.T_cap, "seqlens": f"U[{cfg.seq_lo},{cfg.seq_hi}]",
                   "sum_seqlens": int(np.sum(w.seqlens)), "bits_k": cfg.bits_k,
                   "bits_v": cfg.bits_v, "group": cfg.group, "clip_alpha": cfg.clip_alpha,
                   "q_out_dtype": "bf16", "step": "append 1 token/seq + decode",
                   "l2": "inputs larger than L2 (decode reads ~%.0f MB per step)" % (dec_bytes / 1e6),
                   "parallelism": f"dp{world} (independent batches)", "cuda_graph": True},
        "roofline": {"bound": "hbm", "kernel": "kvq_decode_attention (qprep + decode_kernel)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_nominal_8000": round(achieved / 8000.0, 4),
                     "bytes_per_launch": dec_bytes, "ms_per_launch": round(dec_ms, 5),
                     "traffic": DECODE_TRAFFIC_BYTES, "traffic_kernel": DECODE_TRAFFIC_KERNEL},
        "append_decode_time": {"append_ms": round(app_ms, 5), "decode_ms": round(dec_ms, 5),
                               "append_tok_per_s": round(cfg.B / (app_ms * 1e-3), 1)},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copies_only_ms": round(copies_ms, 5),
                "how": "pinned staging buffers: H2D of the append inputs, then append while "
                       "q and seqlens copy on a second stream, decode, D2H of the output; "
                       "replayed as a CUDA graph"},
        "gpu_launches": 3 * K,
        "dev_err": dev_err,
        "clocks": clocks,
    }

    if not args.no_extras:
        line["bf16_comparator"] = bf16_comparator(w, cfg, K, stream, dec_ms)
        line["paged_decode"] = paged_decode(w, cfg, K, stream, dec_ms, dec_bytes)
        line["window_decode"] = window_decode(w, cfg, stream, dec_ms, peak)
        line["vq_decode"] = vq_decode(w, cfg, stream, dec_ms, peak)
        del w
        torch.cuda.empty_cache()
        line["chunk_append"] = chunk_append(device, stream)
        line["chunk_append_d128"] = chunk_append(device, stream, d128=True)
        line["append_config0"] = append_config0(device, stream)
        line["decode_configs"] = [decode_config_line(i, device, stream, peak)
                                  for i in DECODE_CONFIGS]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def build_cache(cfg, device, append_n=None):
    """The workload's cache filled by the library's own quantize-append from the seeded
    synthetic keys and values, one sequence at a time (seqlens as drawn)."""
    import torch
    import decode_attention_post_b200 as kvq
    qp = kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)
    cache = kvq.KVCache.allocate(cfg.B, cfg.Hkv, cfg.T_cap, cfg.d, qp, device=device)
    seql = synth.seqlens(cfg)
    Tk, Tv, Tit = synth.transforms(cfg)
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    Tk, Tv, Tit = g(Tk), g(Tv), g(Tit)
    zero = torch.zeros(1, dtype=torch.int32, device=device)
    for b in range(cfg.B):
        n = int(seql[b])
        kd = g(synth.keys(cfg, b, 0, n)).to(torch.bfloat16)
        vd = g(synth.values(cfg, b, 0, n)).to(torch.bfloat16)
        kvq.quantize_append(kd[None], vd[None], Tk, Tv, qp, cache.view_sequence(b), zero)
        del kd, vd
    torch.cuda.synchronize()
    return cache, seql, Tit


def decode_bytes(cfg, seql):
    ng = cfg.d // cfg.group
    per_tok = cfg.Hkv * (cfg.d * cfg.bits_k // 8 + 4 * ng + cfg.d * cfg.bits_v // 8 + 4 * ng)
    return int(np.sum(seql)) * per_tok + 2 * cfg.B * cfg.Hq * cfg.d * 2


def decode_config_line(idx, device, stream, peak):
    """Decode call (q prologue + split-K decode) at one more workload shape."""
    import torch
    import decode_attention_post_b200 as kvq
    cfg = synth.CONFIGS[idx]
    cache, seql, Tit = build_cache(cfg, device)
    q = torch.from_numpy(synth.queries(cfg)).to(device).to(torch.bfloat16)
    sd = torch.from_numpy(seql).to(device)
    out = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)
    ws = torch.empty(kvq.decode_workspace_bytes(cache, cfg.Hq, cfg.T_cap), dtype=torch.uint8,
                     device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    fn = lambda: kvq.decode_attention(q, Tit, cache, sd, cfg.T_cap, out, ws, dev_err=err)
    ms = statistics.mean(time_events(fn, 200, stream))
    nbytes = decode_bytes(cfg, seql)
    res = {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
           "bits_k": cfg.bits_k, "bits_v": cfg.bits_v,
           "seqlens": f"U[{cfg.seq_lo},{cfg.seq_hi}]", "sum_seqlens": int(np.sum(seql)),
           "bytes_per_launch": nbytes, "ms_per_launch": round(ms, 5),
           "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
           "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4),
           "dev_err": int(err.item())}
    del cache, ws
    torch.cuda.empty_cache()
    return res


def decode_split_sweep(idx, device, stream, peak, splits):
    """Decode time of one workload for several split counts (KVQ_DECODE_SPLITS), one cache."""
    import torch
    import decode_attention_post_b200 as kvq
    cfg = synth.CONFIGS[idx]
    cache, seql, Tit = build_cache(cfg, device)
    q = torch.from_numpy(synth.queries(cfg)).to(device).to(torch.bfloat16)
    sd = torch.from_numpy(seql).to(device)
    out = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    nbytes = decode_bytes(cfg, seql)
    res = []
    for sp in [0] + list(splits):
        if sp:
            os.environ["KVQ_DECODE_SPLITS"] = str(sp)
        else:
            os.environ.pop("KVQ_DECODE_SPLITS", None)
        ws = torch.empty(kvq.decode_workspace_bytes(cache, cfg.Hq, cfg.T_cap), dtype=torch.uint8,
                         device=device)
        fn = lambda: kvq.decode_attention(q, Tit, cache, sd, cfg.T_cap, out, ws, dev_err=err)
        ms = statistics.mean(time_events(fn, 100, stream))
        res.append({"splits": sp or "default", "ms": round(ms, 5),
                    "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4)})
        del ws
    os.environ.pop("KVQ_DECODE_SPLITS", None)
    return res


def append_config0(device, stream):
    """Prefill append of the tiny float32 workload (1 sequence, 2048 tokens, 1 KV head,
    d 128): float32 CUDA-core transform path."""
    import torch
    import decode_attention_post_b200 as kvq
    cfg = synth.CONFIGS[0]
    qp = kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)
    cache = kvq.KVCache.allocate(cfg.B, cfg.Hkv, cfg.T_cap, cfg.d, qp, device=device)
    Tk, Tv, _ = synth.transforms(cfg)
    k, v = synth.kv_batch(cfg, 0, cfg.T_cap)
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    kd, vd, Tk, Tv = g(k), g(v), g(Tk), g(Tv)
    pos = torch.zeros(cfg.B, dtype=torch.int32, device=device)
    fn = lambda: kvq.quantize_append(kd, vd, Tk, Tv, qp, cache, pos)
    ms = statistics.mean(time_events(fn, 50, stream))
    tokheads = cfg.B * cfg.T_cap * cfg.Hkv
    nbytes = tokheads * (2 * cfg.d * 4 + cfg.d * (cfg.bits_k + cfg.bits_v) // 8 + 8) + \
        2 * cfg.Hkv * cfg.d * cfg.d * 4
    return {"workload": cfg.name, "ms": round(ms, 4),
            "tok_per_s": round(cfg.B * cfg.T_cap / (ms * 1e-3), 1),
            "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "bytes": nbytes}


def bf16_comparator(w, cfg, K, stream, dec_ms):
    import torch
    import decode_attention_post_b200 as kvq
    out = torch.empty_like(w.out)
    ws = torch.empty(kvq.bf16_decode_workspace_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.T_cap),
                     dtype=torch.uint8, device=w.dev)
    fn = lambda: kvq.bf16_decode(w.q, w.kb, w.vb, w.seq_d, cfg.T_cap, out, ws, dev_err=w.err)
    ms = statistics.mean(time_events(fn, min(K, 200), stream))
    nbytes = int(np.sum(w.seqlens)) * cfg.Hkv * cfg.d * 2 * 2 + 2 * cfg.B * cfg.Hq * cfg.d * 2
    return {"ms_per_launch": round(ms, 5), "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "bytes_per_launch": nbytes, "speedup_of_2bit_decode": round(ms / dec_ms, 2)}


def paged_decode(w, cfg, K, stream, dec_ms, dec_bytes, page_tokens=256):
    """The same decode over a page pool: the workload's cache moved into shuffled pages of
    `page_tokens` positions (block table read by the kernels at every call)."""
    import torch
    import decode_attention_post_b200 as kvq
    per = cfg.T_cap // page_tokens
    num_pages = cfg.B * per + 64
    perm = np.random.default_rng(1000 * cfg.idx + 7).permutation(num_pages)[:cfg.B * per]
    table = torch.from_numpy(perm.reshape(cfg.B, per).astype(np.int32)).to(w.dev)
    pc = kvq.KVCache.allocate_paged(num_pages, page_tokens, table, cfg.Hkv, cfg.d, w.qp,
                                    device=w.dev, zero=False)
    idx = table.reshape(-1).long()
    for src, dst in zip((w.cache.k_codes, w.cache.k_sz, w.cache.v_codes, w.cache.v_sz),
                        (pc.k_codes, pc.k_sz, pc.v_codes, pc.v_sz)):
        tb = src.numel() // (cfg.B * cfg.Hkv * cfg.T_cap)
        s5 = src.view(cfg.B, cfg.Hkv, per, page_tokens, tb).permute(0, 2, 1, 3, 4)
        dst.view(num_pages, cfg.Hkv, page_tokens, tb).index_copy_(
            0, idx, s5.reshape(cfg.B * per, cfg.Hkv, page_tokens, tb))
    out = torch.empty_like(w.out)
    fn = lambda: kvq.decode_attention(w.q, w.Tit, pc, w.seq_d, w.max_seqlen, out, w.ws,
                                      dev_err=w.err)
    ms = statistics.mean(time_events(fn, min(K, 500), stream))
    w.decode()
    torch.cuda.synchronize()
    same = bool(torch.equal(out.view(torch.int16), w.out.view(torch.int16)))
    del pc
    return {"page_tokens": page_tokens, "num_pages": num_pages, "ms_per_launch": round(ms, 5),
            "GB_s": round(dec_bytes / (ms * 1e-3) / 1e9, 1),
            "time_vs_contiguous": round(ms / dec_ms, 4), "output_identical": same}


def window_decode(w, cfg, stream, dec_ms, peak, S_sink=64, S_keep=256, S_flush=128):
    """The same sequences with a full-precision window (WUSH-KV section 4.4): the state is
    built by kvq_window_append (one call per sequence over its whole context), then the
    windowed decode (q prologue + window kernel + decode of the quantized middle) is timed,
    and one decode-time step (window append of 1 token per sequence + windowed decode)."""
    import torch
    import decode_attention_post_b200 as kvq
    B, Hkv, d = cfg.B, cfg.Hkv, cfg.d
    R = S_keep + S_flush
    z = lambda n: torch.zeros((B, Hkv, n, d), dtype=torch.bfloat16, device=w.dev)
    ks, vs, kr, vr = z(S_sink), z(S_sink), z(R), z(R)
    cache = kvq.KVCache.allocate(B, Hkv, cfg.T_cap, d, w.qp, device=w.dev, zero=False)
    zero = torch.zeros(1, dtype=torch.int32, device=w.dev)
    for b in range(B):
        L = int(w.seqlens[b]) - 1                    # the step appends the last token
        kb = w.kb[b, :, :L].transpose(0, 1).contiguous()[None]
        vb = w.vb[b, :, :L].transpose(0, 1).contiguous()[None]
        kvq.window_append(kb, vb, w.Tk, w.Tv, w.qp, cache.view_sequence(b), S_sink, S_keep,
                          S_flush, ks[b:b + 1], vs[b:b + 1], kr[b:b + 1], vr[b:b + 1], zero,
                          dev_err=w.err)
    torch.cuda.synchronize()
    prev = torch.from_numpy((w.seqlens - 1).astype(np.int32)).to(w.dev)
    kvq.window_append(w.knew, w.vnew, w.Tk, w.Tv, w.qp, cache, S_sink, S_keep, S_flush, ks, vs,
                      kr, vr, prev, dev_err=w.err)
    out = torch.empty_like(w.out)
    ws = torch.empty(kvq.decode_workspace_bytes(cache, cfg.Hq, cfg.T_cap), dtype=torch.uint8,
                     device=w.dev)
    dec = lambda: kvq.decode_attention_window(w.q, w.Tit, cache, S_sink, S_keep, S_flush, ks, vs,
                                              kr, vr, w.Tv, w.seq_d, cfg.T_cap, out, ws,
                                              dev_err=w.err)
    ms = statistics.mean(time_events(dec, 200, stream))
    # one serving step: re-append the newest token (the state for seqlens - 1 positions
    # plus that token is the same state) and decode
    step = lambda: (kvq.window_append(w.knew, w.vnew, w.Tk, w.Tv, w.qp, cache, S_sink, S_keep,
                                      S_flush, ks, vs, kr, vr, prev, dev_err=w.err), dec())
    step_ms = statistics.mean(time_events(step, 100, stream))
    Q = np.array([(max(0, L - S_sink - S_keep) // S_flush) * S_flush for L in w.seqlens])
    nwin = w.seqlens - Q
    ng = d // cfg.group
    per_q = Hkv * (d * (cfg.bits_k + cfg.bits_v) // 8 + 8 * ng)
    nbytes = int(Q.sum()) * per_q + int(nwin.sum()) * Hkv * 2 * d * 2 + \
        2 * Hkv * d * d * 4 + 2 * B * cfg.Hq * d * 2
    torch.cuda.synchronize()
    res = {"S_sink": S_sink, "S_keep": S_keep, "S_flush": S_flush,
           "window_positions": int(nwin.sum()), "quantized_positions": int(Q.sum()),
           "bytes_per_launch": nbytes, "ms_per_launch": round(ms, 5),
           "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
           "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4),
           "time_vs_plain_decode": round(ms / dec_ms, 4),
           "step_ms_append_plus_decode": round(step_ms, 5), "dev_err": int(w.err.item())}
    del cache, ks, vs, kr, vr, ws
    torch.cuda.empty_cache()
    return res


def vq_decode(w, cfg, stream, dec_ms, peak):
    """The same sequences in the vector-quantized cache (NOVA-KV: codebook lookup plus one
    multiply; synthetic codebooks): encoded by kvq_vq_append, then the VQ decode timed, and
    a decode-time step (VQ append of the newest token + decode)."""
    import torch
    import decode_attention_post_b200 as kvq
    cb_k, cb_v = synth.codebooks(cfg)
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(w.dev)
    ck, cv = f16(cb_k), f16(cb_v)
    cache = kvq.VQCache.allocate(cfg.B, cfg.Hkv, cfg.T_cap, cfg.d, device=w.dev, zero=False)
    for b in range(cfg.B):
        L = int(w.seqlens[b])
        kb = w.kb[b, :, :L].transpose(0, 1).contiguous()[None]
        vb = w.vb[b, :, :L].transpose(0, 1).contiguous()[None]
        one = kvq.VQCache(1, cfg.Hkv, cfg.T_cap, cfg.d,
                          [p[b * (p.numel() // cfg.B):(b + 1) * (p.numel() // cfg.B)]
                           for p in (cache.k_idx, cache.k_gain, cache.v_idx, cache.v_gain)])
        kvq.vq_append(kb, vb, w.Tk, w.Tv, ck, cv, one, torch.zeros(1, dtype=torch.int32,
                                                                    device=w.dev))
    torch.cuda.synchronize()
    out = torch.empty_like(w.out)
    ws = torch.empty(kvq.vq_decode_workspace_bytes(cache, cfg.Hq, cfg.T_cap), dtype=torch.uint8,
                     device=w.dev)
    dec = lambda: kvq.vq_decode_attention(w.q, w.Tit, ck, cv, cache, w.seq_d, cfg.T_cap, out, ws,
                                          dev_err=w.err)
    ms = statistics.mean(time_events(dec, 200, stream))
    step = lambda: (kvq.vq_append(w.knew, w.vnew, w.Tk, w.Tv, ck, cv, cache, w.pos, n=1,
                                  dev_err=w.err), dec())
    step_ms = statistics.mean(time_events(step, 100, stream))
    per_tok = cfg.Hkv * 2 * (cfg.d // 4 + 2)
    nbytes = int(np.sum(w.seqlens)) * per_tok + 2 * cfg.B * cfg.Hq * cfg.d * 2 + \
        2 * cfg.Hkv * 256 * 4 * 2
    torch.cuda.synchronize()
    res = {"bits_per_element": round(8 * (cfg.d // 4 + 2) / cfg.d, 4),
           "bytes_per_launch": nbytes, "ms_per_launch": round(ms, 5),
           "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
           "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4),
           "time_vs_scalar_decode": round(ms / dec_ms, 4),
           "step_ms_append_plus_decode": round(step_ms, 5), "dev_err": int(w.err.item())}
    del cache, ws
    torch.cuda.empty_cache()
    return res


def chunk_append(device, stream, d128=False):
    """32768-token chunk append of the GPT-OSS-20B-like shape (batch 8, 8 KV heads, d 64);
    d128: a 16384-token chunk of the Qwen3-8B-like heads (batch 8, 8 KV heads, d 128)."""
    import torch
    import decode_attention_post_b200 as kvq
    if d128:
        cfg = synth.CONFIGS[CONFIG_IDX].with_(B=8)
        n = 16384
    else:
        cfg = synth.CONFIGS[APPEND_CONFIG_IDX]
        n = cfg.append_n
    qp = kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)
    cache = kvq.KVCache.allocate(cfg.B, cfg.Hkv, cfg.T_cap, cfg.d, qp, device=device)
    Tk, Tv, _ = synth.transforms(cfg)
    k, v = synth.kv_batch(cfg, 0, n)
    bf = lambda a: torch.from_numpy(a).to(device).to(torch.bfloat16)
    kd, vd = bf(k), bf(v)
    del k, v
    Tk, Tv = torch.from_numpy(Tk).to(device), torch.from_numpy(Tv).to(device)
    pos = torch.zeros(cfg.B, dtype=torch.int32, device=device)
    fn = lambda: kvq.quantize_append(kd, vd, Tk, Tv, qp, cache, pos)
    ms = statistics.mean(time_events(fn, 10, stream))
    ng = cfg.d // cfg.group
    tokheads = cfg.B * n * cfg.Hkv
    nbytes = tokheads * (2 * cfg.d * 2 + cfg.d * (cfg.bits_k + cfg.bits_v) // 8 + 8 * ng) + \
        2 * cfg.Hkv * cfg.d * cfg.d * 4
    flops = tokheads * 4 * cfg.d * cfg.d
    return {"workload": cfg.name if not d128 else "qwen3-8b-like-b8-d128-append16k",
            "ms": round(ms, 4),
            "tok_per_s": round(cfg.B * n / (ms * 1e-3), 1),
            "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "TFLOP_s": round(flops / (ms * 1e-3) / 1e12, 2), "bytes": nbytes}


# ----------------------------------------------------------------------------- oracle (CPU)

class OracleSample:
    """A bounded sample of the config-2 step for the float64 CPU oracle: the first
    `nseq` sequences, all heads, the cache built by the oracle itself."""

    def __init__(self, cfg, nseq):
        import oracle
        self.oracle = oracle
        self.cfg = cfg.with_(B=nseq)
        self.seqlens = synth.seqlens(cfg)[:nseq]
        Tk, Tv, self.Tit = synth.transforms(cfg)
        self.Tk, self.Tv = Tk, Tv
        self.cache = oracle.Cache.for_config(self.cfg)
        knew = np.empty((nseq, 1, cfg.Hkv, cfg.d), np.uint16)
        vnew = np.empty_like(knew)
        for b in range(nseq):
            n = int(self.seqlens[b])
            k = synth.as_dtype(synth.keys(cfg, b, 0, n), "bf16")
            v = synth.as_dtype(synth.values(cfg, b, 0, n), "bf16")
            one = oracle.Cache(1, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
            oracle.quantize_append(k[None], v[None], Tk, Tv, cfg.bits_k, cfg.bits_v, cfg.group,
                                   cfg.clip_alpha, one, [0])
            for dst, src in zip(self.cache.planes(), one.planes()):
                m = src.size
                dst[b * m:(b + 1) * m] = src
            knew[b, 0], vnew[b, 0] = k[n - 1], v[n - 1]
        self.knew, self.vnew = knew, vnew
        self.q = synth.as_dtype(synth.queries(cfg), "bf16")[:nseq].copy()

    def step(self, sel=None):
        c = self.cfg
        self.oracle.quantize_append(self.knew, self.vnew, self.Tk, self.Tv, c.bits_k, c.bits_v,
                                    c.group, c.clip_alpha, self.cache, self.seqlens - 1)
        return self.oracle.decode(self.q, self.Tit, self.cache, self.seqlens, sel=sel)

    def bytes(self, heads=None):
        """Algorithmic bytes of the sample; decode bytes scale with the query heads run."""
        d, a = step_bytes(self.cfg, self.seqlens)
        frac = 1.0 if heads is None else heads / self.cfg.Hq
        return d * frac + a


def cpu_baseline(cfg, budget_s=12.0):
    """The float64 oracle on the host cores: all threads, then one thread (a quarter of
    the budget), on one sequence of the workload."""
    import oracle
    s = OracleSample(cfg, 1)
    cores = oracle.get_threads()

    def timed(budget):
        t = time.perf_counter()
        s.step()
        one = time.perf_counter() - t
        reps = max(1, int(budget / max(one, 1e-3)))
        t = time.perf_counter()
        for _ in range(reps):
            s.step()
        return (time.perf_counter() - t) / reps, reps
    el, reps = timed(budget_s)
    oracle.set_threads(1)
    el1, reps1 = timed(budget_s / 4)
    oracle.set_threads(cores)
    return {"value": round(s.bytes() / el / 1e9, 4), "unit": "GB/s",
            "cores": cores, "kind": "oracle",
            "single_thread_value": round(s.bytes() / el1 / 1e9, 5),
            "sample": f"1 of {cfg.B} sequences (seqlen {int(s.seqlens[0])}), all {cfg.Hq} "
                      f"query heads: append 1 token + decode, {reps} reps at {cores} threads "
                      f"({el:.3f} s per step), {reps1} reps at 1 thread ({el1:.3f} s)"}


def run_reference(args):
    """The float64 oracle as the reference arm, timed on the host cores. Each step is a
    bounded sample of the config-2 step (the newest token of one sequence appended, then
    the decode of that sequence for as many query heads as keep K steps within ~2 minutes)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cfg = synth.CONFIGS[CONFIG_IDX]
    s = OracleSample(cfg, 1)
    t = time.perf_counter()
    s.step()
    full = time.perf_counter() - t
    K = args.steps
    heads = int(min(cfg.Hq, max(1, round(cfg.Hq * 120.0 / (max(K, 1) * full)))))
    sel = np.array([[0, h] for h in range(heads)], np.int32)
    for _ in range(max(args.warmup, 3)):
        s.step(sel)
    t = time.perf_counter()
    for _ in range(K):
        s.step(sel)
    el = (time.perf_counter() - t) / K
    value = s.bytes(heads) / el / 1e9
    cores = oracle.get_threads()
    sample = (f"sequence 0 of {cfg.B} (seqlen {int(s.seqlens[0])}): append 1 token (all KV "
              f"heads) + decode of {heads} of {cfg.Hq} query heads per step")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": K, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv,
                       "d": cfg.d, "T_cap": cfg.T_cap, "bits_k": cfg.bits_k,
                       "bits_v": cfg.bits_v, "sample": sample},
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def profile_case(name):
    """One kernel's workload on its own, a few launches, for an ncu capture of that kernel
    (the command is recorded in the profiles directory). Prints one JSON line."""
    import torch
    import decode_attention_post_b200 as kvq
    torch.cuda.set_device(0)
    device, stream = "cuda:0", torch.cuda.current_stream()
    peak, _ = peaks()
    if name == "chunk_append":
        res = chunk_append(device, stream)
    elif name == "chunk_append_d128":
        res = chunk_append(device, stream, d128=True)
    elif name == "append_config0":
        res = append_config0(device, stream)
    elif name.startswith("decode_config"):
        idx = int(name[len("decode_config"):])
        sweep = os.environ.get("KVQ_BENCH_SPLIT_SWEEP")    # e.g. "2,4,8": splits to time
        if sweep:
            res = {"sweep": decode_split_sweep(idx, device, stream, peak,
                                               [int(x) for x in sweep.split(",")])}
        else:
            res = decode_config_line(idx, device, stream, peak)
    elif name in ("vq_config1", "window_config1"):
        # a Workload at the batch-16 / 16K shape (bf16 tokens kept), then the VQ or the
        # windowed decode line on it
        cfg = synth.CONFIGS[1]
        w = Workload(cfg, 0, device, with_bf16=True)
        dec_ms = statistics.mean(time_events(w.decode, 50, stream))
        res = (vq_decode if name == "vq_config1" else window_decode)(w, cfg, stream, dec_ms, peak)
    elif name == "bf16_config1":
        # the uncompressed comparator at the batch-16 / 16K shape (1.07 GB of bf16 K and V);
        # its time does not depend on the values, so they are drawn on the device
        cfg = synth.CONFIGS[1]
        gen = torch.Generator(device=device)
        gen.manual_seed(1000 * cfg.idx + synth.STREAM_CACHE)
        shape = (cfg.B, cfg.Hkv, cfg.T_cap, cfg.d)
        kb = torch.randn(shape, generator=gen, device=device).to(torch.bfloat16)
        vb = torch.randn(shape, generator=gen, device=device).to(torch.bfloat16)
        q = torch.from_numpy(synth.queries(cfg)).to(device).to(torch.bfloat16)
        sd = torch.from_numpy(synth.seqlens(cfg)).to(device)
        out = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)
        ws = torch.empty(kvq.bf16_decode_workspace_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.T_cap),
                         dtype=torch.uint8, device=device)
        fn = lambda: kvq.bf16_decode(q, kb, vb, sd, cfg.T_cap, out, ws)
        ms = statistics.mean(time_events(fn, 20, stream))
        nbytes = int(np.sum(synth.seqlens(cfg))) * cfg.Hkv * cfg.d * 4 + 2 * cfg.B * cfg.Hq * cfg.d * 2
        res = {"workload": cfg.name, "ms": round(ms, 5),
               "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "bytes": nbytes}
    else:
        raise SystemExit(f"unknown profile case {name}")
    print(json.dumps({"case": name, **res}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("kvq", "reference"), default="kvq")
    ap.add_argument("--no-extras", action="store_true", help="skip bf16 comparator and chunk append")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile-case", default=None,
                    help="run one kernel's workload alone (chunk_append, chunk_append_d128, "
                         "append_config0, "
                         "decode_config1/2/3/4, bf16_config1, vq_config1, window_config1) "
                         "for an ncu capture")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
