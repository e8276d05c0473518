"""Benchmark of the LoD attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: decode_gqa_128k_bf16 (batch 4, 64 query / 8 KV heads,
head dim 128, context 131072, bf16; top-8 groups, top-2 pages, window 512,
4 sinks).  One step = one lod_decode call for the whole batch (every query
head of every sequence, one layer).  Inputs are seeded synthetic data resident
in HBM; L2 is flushed (a 256 MiB write) between timed steps and each step is
timed alone with CUDA events on the launching stream.  Rank 0 prints one JSON
line.  Under torchrun every rank runs its own replica (the path shards by
sequence with no exchange), and the line reports the aggregate over ranks with
the max-over-ranks time.

The line also carries the chunked prefill (prefill_128k_bf16) and index build
(build_128k_bf16, k=4) numbers measured in the same run, the roofline of the
decode call, the oracle's CPU throughput on a bounded sample, the end-to-end
rate through the public API with host buffers, and the SM clocks sampled
during the timed region.

--impl reference times the CPU oracle instead (rank 0 only), on bounded
samples of the same workload, with the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np
import torch

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = "/tmp/lod_clocks_%d_%d.csv" % (os.getpid(), gpu_index)

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1].split()[0]), float(parts[2].split()[0]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        sm = sorted(r[0] for r in rows)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- helpers

def csrc_hash(files=None) -> str:
    """SHA-256 over the library's CUDA sources (file names and contents): all
    of them, or the listed ones."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "hierarchical_long_context_b200", "csrc")
    names = sorted(files) if files else sorted(f for f in os.listdir(d) if f.endswith((".cu", ".cuh")))
    for f in names:
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kind: str, workload: str):
    """DRAM bytes (read + write) per launch from the committed ncu summary
    profiles/<kind>_<workload>.md, or None when that summary is missing or was
    captured from CUDA sources other than the current ones (the summary's
    `csrc_files:` line names the sources its kernels are built from)."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kind, workload))
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as fh:
        for line in fh:
            for key in ("traffic_bytes_per_launch:", "csrc_sha256:", "csrc_files:"):
                if line.strip().startswith(key):
                    vals[key] = line.strip()[len(key):].strip()
    files = vals.get("csrc_files:", "").split() or None
    if vals.get("csrc_sha256:", "").split()[:1] != [csrc_hash(files)] or "traffic_bytes_per_launch:" not in vals:
        return None
    return int(vals["traffic_bytes_per_launch:"].split()[0])


def l2_flusher(dev):
    buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    return lambda: buf.zero_()


def time_steps(fn, steps, warmup, flush, stream):
    """Per-step device time (ms) with events on `stream`; fn(i) runs step i.
    `flush` (when given) writes a buffer larger than L2 before every step,
    outside the timed region."""
    for i in range(warmup):
        if flush:
            flush()
        fn(i)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        if flush:
            flush()
        a.record(stream)
        fn(i)
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_region(fn, steps, warmup, stream):
    """Device time (ms) of `steps` back-to-back steps fn(i), one event pair
    around the whole region (consecutive steps may overlap their launches)."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_max(x: float, world: int, device: str = "cuda") -> float:
    """Max of x over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


# ---------------------------------------------------------------- workloads

def params_for(w, k=None, kv_bits=0):
    from hierarchical_long_context_b200 import api
    return api.Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, Tmax=((w.T + 255) // 256) * 256,
                      dtype=w.torch_dtype, clusters=k or w.clusters[0], kmeans_iters=w.iters,
                      top_groups=w.top_groups, top_pages=w.top_pages, window=w.window, sinks=w.sinks,
                      seed=w.seed, kv_bits=kv_bits,
                      head_shard=(w.hkv_model << 16) | w.kvh0 if w.hkv_model else 0)


def run_decode(w, args, dev, stream, world, rank, peaks):
    from hierarchical_long_context_b200 import api, metrics
    qf = world if args.shard == "batch" else 1  # sequences decoded per step, over all ranks, / w.B
    p = params_for(w, kv_bits=args.kv_bits)
    K, V = synth_kv(w)
    Kd, Vd = K.to(dev), V.to(dev)
    ix = api.Index(p, dev)
    api.lod_build_index(p, Kd, Vd, 0, w.T // 256, ix, stream=stream)
    q = synth_q(w).to(dev)
    sl = torch.full((w.B,), w.T, dtype=torch.int64, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE, dev)
    out = torch.empty_like(q)
    sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
    spg = torch.empty(w.B, w.Hq, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
    api.lod_decode(p, q, Kd, Vd, sl, ix, out=out, sel_groups=sg, sel_pages=spg, ws=ws, stream=stream)
    torch.cuda.synchronize()
    touched = metrics.decode_touched_bytes(p, ix, sl, sg, spg)
    # Inputs larger than L2: R device replicas of everything a step reads
    # (cache, index, queries, lengths, workspace), used in rotation, so a
    # step's data was last touched R - 1 steps (R - 1 x the touched bytes)
    # earlier.  The kernels' code stays cached, as across the layers of a model.
    R = max(1, args.replicas)
    reps = [(q, Kd, Vd, sl, ix, ws, out)]
    for _ in range(R - 1):
        ixr = api.Index(p, dev)
        for f in api._lib.INDEX_FIELDS:
            getattr(ixr, f).copy_(getattr(ix, f))
        reps.append((q.clone(), Kd.clone(), Vd.clone(), sl.clone(), ixr, torch.zeros_like(ws), torch.empty_like(out)))
    torch.cuda.synchronize()
    flush = l2_flusher(dev) if R == 1 else None

    def step(i):
        qr, Kr, Vr, slr, ixr, wsr, outr = reps[i % R]
        api.lod_decode(p, qr, Kr, Vr, slr, ixr, out=outr, ws=wsr, stream=stream)
    barrier(world)
    with ClockSampler(torch.cuda.current_device() if world == 1 else int(os.environ.get("LOCAL_RANK", 0))) as cs:
        t0 = time.perf_counter()
        if flush is None:  # inputs larger than L2: the K steps back to back, one event pair
            total = time_region(step, args.steps, args.warmup, stream)
            wall = time.perf_counter() - t0
            ts = time_steps(step, min(args.steps, 500), 3, None, stream)  # per-step spread only
            ms_region = total / args.steps
        else:
            ts = time_steps(step, args.steps, args.warmup, flush, stream)
            wall = time.perf_counter() - t0
            ms_region = None
    barrier(world)
    status = 0
    for r in reps:
        status |= api.lod_get_status(r[5], stream)
    ms = ms_region if ms_region is not None else float(np.mean(ts))
    ms_max = dist_max(ms, world)
    # end to end through the public API, inputs and result in pinned host
    # memory: one buffer in (q and this token's K and V rows), out back.  Main
    # form: the kernels read q and the new rows straight from the pinned
    # buffer and the refine kernel stores out straight into pinned memory (no
    # copy-engine transfer).  Second form, for comparison: a copy-engine copy
    # of the input buffer to the device and of the output back.  Each step is
    # one CUDA graph.
    qn, rown = q.numel(), w.B * w.Hkv * w.d
    hin = torch.empty(qn + 2 * rown, dtype=w.torch_dtype).pin_memory()
    hin[:qn] = q.cpu().reshape(-1)
    hin[qn:qn + rown] = K[:, :, w.T - 1].reshape(-1)
    hin[qn + rown:] = V[:, :, w.T - 1].reshape(-1)
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    stage = [torch.empty(qn + 2 * rown, dtype=w.torch_dtype, device=dev) for _ in range(R)]
    hq = hin[:qn].view(q.shape)
    hk, hv = hin[qn:qn + rown].view(w.B, w.Hkv, w.d), hin[qn + rown:].view(w.B, w.Hkv, w.d)

    def e2e_direct(r, strm):
        qr, Kr, Vr, slr, ixr, wsr, outr = reps[r]
        api.lod_append_kv(p, Kr, Vr, slr, hk, hv, stream=strm)
        api.lod_decode(p, hq, Kr, Vr, slr, ixr, out=hout, ws=wsr, stream=strm)

    def e2e_copy(r, strm):
        qr, Kr, Vr, slr, ixr, wsr, outr = reps[r]
        st = stage[r]
        st.copy_(hin, non_blocking=True)
        api.lod_append_kv(p, Kr, Vr, slr, st[qn:qn + rown].view(w.B, w.Hkv, w.d),
                          st[qn + rown:].view(w.B, w.Hkv, w.d), stream=strm)
        api.lod_decode(p, st[:qn].view(q.shape), Kr, Vr, slr, ixr, out=outr, ws=wsr, stream=strm)
        hout.copy_(outr, non_blocking=True)

    e2e_steps = max(10, min(args.steps, 1000))
    expect = reps[0][6].cpu()  # every replica holds the same inputs, so the same output

    def e2e_time(body):
        graphs = None
        if args.graphs:
            try:
                graphs = []
                for r in range(R):
                    body(r, stream)  # warm (attributes set, lazy state built) before capture
                torch.cuda.synchronize()
                for r in range(R):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        body(r, None)
                    graphs.append(g)
                torch.cuda.synchronize()
            except Exception as ex:  # capture not possible here: eager steps instead
                print("e2e graph capture failed (%s); eager steps" % ex, file=sys.stderr)
                graphs = None
        fn = (lambda i: graphs[i % R].replay()) if graphs else (lambda i: body(i % R, stream))
        hout.zero_()
        if flush is None:
            t = dist_max(time_region(fn, e2e_steps, 5, stream) / e2e_steps, world)
        else:
            t = dist_max(float(np.mean(time_steps(fn, e2e_steps, 3, flush, stream))), world)
        torch.cuda.synchronize()
        assert torch.equal(hout, expect), "e2e output mismatch"
        return t, graphs is not None

    e2e_ms, g1 = e2e_time(e2e_direct)
    e2e_copy_ms, g2 = e2e_time(e2e_copy)
    achieved = touched / (ms * 1e-3) / 1e9
    res = dict(
        metric="LoD decode queries/s (batch 4 x 64 heads at 128K context, one layer)",
        value=qf * w.B / (ms_max * 1e-3), unit="queries/s", ms_per_step=ms_max,
        ms_p10=float(np.percentile(ts, 10)), ms_p90=float(np.percentile(ts, 90)),
        head_rows_per_s=world * w.B * w.Hq / (ms_max * 1e-3), wall_s_timed=wall,
        status_word=status,
        roofline=dict(bound="hbm", kernel="lod_decode (scan + refine kernels)", achieved=achieved,
                      peak=peaks["hbm_gbs"], unit="GB/s", frac=achieved / peaks["hbm_gbs"],
                      traffic=profiled_traffic("lod_decode_int4" if args.kv_bits == 4 else "lod_decode", w.name),
                      algorithmic_bytes_per_launch=touched,
                      peak_source=peaks["source"], nominal_peak_gbs=8000.0),
        e2e=dict(value=qf * w.B / (e2e_ms * 1e-3), unit="queries/s",
                 h2d_bytes_per_step=hin.numel() * hin.element_size(),
                 d2h_bytes_per_step=hout.numel() * hout.element_size(), ms_per_step=e2e_ms,
                 step=("one CUDA graph" if g1 else "eager") + " per step: lod_append_kv reading the new "
                      "K/V rows from pinned host memory, lod_decode reading q from pinned host memory "
                      "and storing out into pinned host memory (the kernels move the bytes over the "
                      "host link; no copy-engine transfer)",
                 copy_engine=dict(value=qf * w.B / (e2e_copy_ms * 1e-3), unit="queries/s",
                                  ms_per_step=e2e_copy_ms,
                                  step=("one CUDA graph" if g2 else "eager") + " per step: copy of "
                                       "the pinned input buffer to the device, lod_append_kv, "
                                       "lod_decode, copy of out to pinned host memory")),
        gpu_launches=2 * args.steps,
        clocks=cs.summary(),
        l2=("inputs larger than L2: %d device replicas of cache, index, queries and workspace "
            "used in rotation (%d x %.1f MB touched per step vs 126 MB L2)" % (R, R, touched / 1e6)
            if R > 1 else "flushed (256 MiB write) between timed steps"),
        _touch=(K, V, ix, reps),
    )
    return res


_KV_CACHE = {}


def synth_kv(w):
    from hierarchical_long_context_b200 import synth
    key = (w.name, w.T, w.B, w.Hkv, w.seed)
    if key not in _KV_CACHE:
        _KV_CACHE[key] = synth.kv_cache(w, threads=min(16, host_cores()))
    return _KV_CACHE[key]


def synth_q(w):
    from hierarchical_long_context_b200 import synth
    return synth.decode_queries(w)


def run_decode_variant(w, dev, stream, peaks, steps, replicas, label, device_gen=False, kv_bits=0):
    """A decode leg on workload `w` (device time of `steps` back-to-back steps
    over rotating input replicas, as the headline leg) with the roofline over
    the bytes its own selections touch."""
    from hierarchical_long_context_b200 import api, metrics
    from hierarchical_long_context_b200 import synth
    p = params_for(w, kv_bits=kv_bits)
    if device_gen:
        Kd, Vd = synth.kv_cache_device(w, dev)
    else:
        K, V = synth_kv(w)
        Kd, Vd = K.to(dev), V.to(dev)
    ix = api.Index(p, dev)
    api.lod_build_index(p, Kd, Vd, 0, w.T // 256, ix, stream=stream)
    q = synth_q(w).to(dev)
    sl = torch.full((w.B,), w.T, dtype=torch.int64, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE, dev)
    sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
    spg = torch.empty(w.B, w.Hq, p.top_groups, max(p.top_pages, 1), dtype=torch.int32, device=dev)
    out = api.lod_decode(p, q, Kd, Vd, sl, ix, sel_groups=sg, sel_pages=spg if p.top_pages else None, ws=ws,
                         stream=stream)
    torch.cuda.synchronize()
    touched = metrics.decode_touched_bytes(p, ix, sl, sg, spg)
    reps = [(q, Kd, Vd, ix, ws, out)]
    for _ in range(max(1, replicas) - 1):
        ixr = api.Index(p, dev)
        for f in api._lib.INDEX_FIELDS:
            getattr(ixr, f).copy_(getattr(ix, f))
        reps.append((q.clone(), Kd.clone(), Vd.clone(), ixr, torch.zeros_like(ws), torch.empty_like(out)))
    R = len(reps)

    def step(i):
        qr, Kr, Vr, ixr, wsr, outr = reps[i % R]
        api.lod_decode(p, qr, Kr, Vr, sl, ixr, out=outr, ws=wsr, stream=stream)

    ms = time_region(step, steps, 10, stream) / steps
    status = 0
    for r in reps:
        status |= api.lod_get_status(r[4], stream)
    gbs = touched / (ms * 1e-3) / 1e9
    del reps
    return dict(workload=label, value=w.B / (ms * 1e-3), unit="queries/s", ms_per_step=ms,
                seq_len=w.T, B=w.B, top_groups=p.top_groups, top_pages=p.top_pages, kv_bits=p.kv_bits,
                l2="%d rotating input replicas" % R,
                roofline=dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                              frac=gbs / peaks["hbm_gbs"], algorithmic_bytes_per_launch=touched),
                status_word=status)


def run_prefill(w, dev, stream, steps, peaks):
    from hierarchical_long_context_b200 import api, metrics, synth
    p = params_for(w)
    K, V = synth_kv(w)
    Kd, Vd = K.to(dev), V.to(dev)
    q = synth.prefill_queries(w, 0, w.T).to(dev)
    out = torch.empty_like(q)
    ix = api.Index(p, dev)
    ws = api.workspace(p, api._lib.LOD_OP_PREFILL, dev)
    flush = l2_flusher(dev)
    ts = time_steps(lambda i: api.lod_prefill(p, q, 0, Kd, Vd, ix, out=out, ws=ws, stream=stream),
                    steps, 1, flush, stream)
    ms = float(np.mean(ts))
    fl = metrics.prefill_flops(p, 0, w.T)
    tf = fl / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    return dict(workload=w.name, value=w.T * w.B / (ms * 1e-3), unit="tok/s", ms_per_step=ms,
                roofline=dict(bound="tensor", achieved=tf, peak=peak, unit="TFLOP/s", frac=tf / peak,
                              algorithmic_flops=fl, peak_source=peaks["source"] + " (sustained)"),
                status_word=api.lod_get_status(ws, stream))


def run_build(w, dev, stream, steps, peaks, k):
    from hierarchical_long_context_b200 import api, metrics
    p = params_for(w, k)
    K, V = synth_kv(w)
    Kd, Vd = K.to(dev), V.to(dev)
    ix = api.Index(p, dev)
    nch = w.T // 256
    flush = l2_flusher(dev)
    ts = time_steps(lambda i: api.lod_build_index(p, Kd, Vd, 0, nch, ix, stream=stream), steps, 2, flush, stream)
    ms = float(np.mean(ts))
    by = metrics.build_bytes(p, nch)          # the method's own reads and writes
    dby = metrics.build_design_bytes(p, nch)  # this design's member-ordered copies
    gbs = by / (ms * 1e-3) / 1e9
    fl = metrics.build_flops(p, nch)
    alu = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12  # FP32 FMA lanes x 2 x clock
    return dict(workload="%s k=%d" % (w.name, k), value=gbs, unit="GB/s", ms_per_step=ms,
                chunks_per_s=p.B * p.Hkv * nch / (ms * 1e-3),
                roofline=dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                              frac=gbs / peaks["hbm_gbs"], algorithmic_bytes=by,
                              design_bytes=dby,
                              with_design_bytes=dict(achieved=(by + dby) / (ms * 1e-3) / 1e9,
                                                     frac=(by + dby) / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]),
                              fp32_tflops=fl / (ms * 1e-3) / 1e12, fp32_alu_peak_tflops=alu,
                              fp32_alu_frac=fl / (ms * 1e-3) / 1e12 / alu))


def run_dense(dev, stream):
    """Dense attention as the second reference (torch SDPA on the GPU): one
    decode step at 32K (batch 8) and at 128K (batch 4), 64 query / 8 KV heads,
    and the causal 128K prefill of 32 query / 8 KV heads, all bf16, d = 128."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    res = {}
    backends = [SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]

    def one(B, Hq, Hkv, T, Tq, causal, steps):
        g = torch.Generator(device=dev).manual_seed(7)
        q = torch.randn(B, Hq, Tq, 128, device=dev, dtype=torch.bfloat16, generator=g) / 8
        k = torch.randn(B, Hkv, T, 128, device=dev, dtype=torch.bfloat16, generator=g)
        v = torch.randn(B, Hkv, T, 128, device=dev, dtype=torch.bfloat16, generator=g)
        # query heads share their KV head: expanded once, outside the timed region
        k = k.repeat_interleave(Hq // Hkv, dim=1)
        v = v.repeat_interleave(Hq // Hkv, dim=1)
        with sdpa_kernel(backends):
            fn = lambda i: F.scaled_dot_product_attention(q, k, v, is_causal=causal)
            ms = time_region(fn, steps, 2, stream) / steps
        del q, k, v
        torch.cuda.empty_cache()
        return ms

    for name, args in (("decode_gqa_32k_bf16", (8, 64, 8, 32768, 1, False, 50)),
                       ("decode_gqa_128k_bf16", (4, 64, 8, 131072, 1, False, 20)),
                       ("prefill_128k_bf16", (1, 32, 8, 131072, 131072, True, 2))):
        try:
            ms = one(*args)
            B, Hq, Hkv, T, Tq, causal, _ = args
            entry = dict(ms_per_step=ms, B=B, Hq=Hq, Hkv=Hkv, seq_len=T, impl="torch SDPA (cuDNN/flash backends), "
                         "KV heads expanded to the query heads outside the timed region")
            if Tq == 1:
                entry.update(value=B / (ms * 1e-3), unit="queries/s")
            else:
                fl = 4.0 * 128 * Hq * T * T / 2
                entry.update(value=T * B / (ms * 1e-3), unit="tok/s", tflops=fl / (ms * 1e-3) / 1e12)
            res[name] = entry
        except Exception as ex:  # no memory-efficient backend for this shape here
            res[name] = dict(unavailable=str(ex).splitlines()[0][:200])
    return res


# ---------------------------------------------------------------- CPU oracle

def oracle_decode_rate(w, budget_s=15.0):
    """The oracle as it stands on this host: per-(b, kvh) index build (untimed,
    it is the index-build step), then the decode rows of whole sequences, timed,
    on a thread pool over all host cores.  Returns (queries/s, sample, cores)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    cores = host_cores()
    K, V = synth_kv(w)
    q = synth_q(w)
    cfg = oracle.Config(d=w.d, clusters=w.clusters[0], iters=w.iters, top_groups=w.top_groups,
                        top_pages=w.top_pages, window=w.window, sinks=w.sinks,
                        store_bf16=(w.dtype == "bf16"), seed=w.seed)
    nch = w.T // 256
    b = 0
    with ThreadPoolExecutor(cores) as ex:
        idx = list(ex.map(lambda h: oracle.build_sequence(cfg, b * w.Hkv + h, K[b, h].float().numpy(),
                                                           V[b, h].float().numpy(), nch), range(w.Hkv)))
    Kn = [K[b, h].float().numpy() for h in range(w.Hkv)]
    Vn = [V[b, h].float().numpy() for h in range(w.Hkv)]
    rows = [(hq, q[b, hq].float().numpy()) for hq in range(w.Hq)]

    def one(r):
        hq, qq = r
        h = hq // w.g
        oracle.attend_row(cfg, qq, w.T - 1, Kn[h], Vn[h], idx[h])

    n = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(cores) as ex:
        while True:
            list(ex.map(one, rows))
            n += 1
            if time.perf_counter() - t0 > budget_s or n >= 50:
                break
    dt = time.perf_counter() - t0
    return n / dt, "%d decode steps of one sequence (all %d heads) at t=%d" % (n, w.Hq, w.T - 1), cores


def oracle_index_all(w, cfg, nch, threads):
    """The oracle's index of every KV head of sequence 0 (threads over heads),
    and the time it took."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    K, V = synth_kv(w)
    Kn = [K[0, h].float().numpy() for h in range(w.Hkv)]
    Vn = [V[0, h].float().numpy() for h in range(w.Hkv)]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        idx = list(ex.map(lambda h: oracle.build_sequence(cfg, h, Kn[h], Vn[h], nch), range(w.Hkv)))
    return idx, Kn, Vn, time.perf_counter() - t0


def oracle_prefill_and_build(budget_rows=0):
    """The oracle on the host cores for the prefill and the index build
    (workloads prefill_128k_bf16 and build_128k_bf16).  Prefill: every row
    (all 32 heads) of query chunks {1, 2, 3, 64, 256, 511}, timed; the time of
    the whole 512-chunk prefill is extrapolated from them (a row's cost grows
    linearly with its chunk's visible groups: least squares over the sampled
    chunks).  Build: the whole 128K index of the 8 KV heads (threads over
    heads), k = 4, timed.  Dense: the oracle's dense attention for 64 rows at
    the last position, the second reference."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from hierarchical_long_context_b200 import synth
    cores = host_cores()
    out = {}
    wb = synth.WORKLOADS["build_128k_bf16"]
    cfgb = oracle.Config(d=wb.d, clusters=4, iters=wb.iters, top_groups=wb.top_groups, top_pages=wb.top_pages,
                         window=wb.window, sinks=wb.sinks, store_bf16=True, seed=wb.seed)
    _, _, _, tb = oracle_index_all(wb, cfgb, wb.T // 256, cores)
    out["build"] = dict(value=wb.Hkv * (wb.T // 256) / tb, unit="chunks/s", seconds=tb, cores=min(cores, wb.Hkv),
                        kind="oracle", sample="the whole 128K index of 8 KV heads, k = 4 (threads over heads)")
    w = synth.WORKLOADS["prefill_128k_bf16"]
    cfg = oracle.Config(d=w.d, clusters=w.clusters[0], iters=w.iters, top_groups=w.top_groups,
                        top_pages=w.top_pages, window=w.window, sinks=w.sinks, store_bf16=True, seed=w.seed)
    nch = w.T // 256
    idx, Kn, Vn, _ = oracle_index_all(w, cfg, nch, cores)
    chunks = (1, 2, 3, 64, 256, 511)
    per_chunk = {}
    for c in chunks:
        q = synth.prefill_queries(w, c * 256, 256)[0].float().numpy()  # [Hq, 256, d]
        rows = [(hq, t) for hq in range(w.Hq) for t in range(256)]
        t0 = time.perf_counter()
        with ThreadPoolExecutor(cores) as ex:
            list(ex.map(lambda rt: oracle.attend_row(cfg, q[rt[0], rt[1]], c * 256 + rt[1], Kn[rt[0] // w.g],
                                                      Vn[rt[0] // w.g], idx[rt[0] // w.g]), rows))
        per_chunk[c] = time.perf_counter() - t0
    # least squares: time(c) = a + b * visible groups of chunk c
    xs = np.array([max(0, c - w.window // 256 + 1) * cfg.clusters for c in chunks], dtype=np.float64)
    ys = np.array([per_chunk[c] for c in chunks])
    A = np.stack([np.ones_like(xs), xs], 1)
    coef = np.linalg.lstsq(A, ys, rcond=None)[0]
    allx = np.array([max(0, c - w.window // 256 + 1) * cfg.clusters for c in range(nch)], dtype=np.float64)
    total = float(np.sum(np.maximum(coef[0] + coef[1] * allx, 0.0)))
    out["prefill"] = dict(value=w.T / total, unit="tok/s", extrapolated=True, seconds_full_estimate=total,
                          sampled_seconds={str(c): per_chunk[c] for c in chunks}, cores=cores, kind="oracle",
                          sample="all rows (32 heads x 256 positions) of query chunks 1, 2, 3, 64, 256, 511; "
                                 "the 512-chunk total is extrapolated (linear in visible groups)")
    qd = synth.prefill_queries(w, w.T - 64, 64)[0].float().numpy()
    t0 = time.perf_counter()
    with ThreadPoolExecutor(cores) as ex:
        list(ex.map(lambda j: oracle.dense_row(cfg, qd[j % w.Hq, j], w.T - 64 + j, Kn[(j % w.Hq) // w.g],
                                               Vn[(j % w.Hq) // w.g]), range(64)))
    td = time.perf_counter() - t0
    out["dense_rows"] = dict(value=64 / td, unit="rows/s", cores=cores, kind="oracle dense attention",
                             sample="64 rows at positions 131008-131071 (causal over the whole context)")
    return out


def run_reference(args, w):
    rate, sample, cores = oracle_decode_rate(w, budget_s=max(5.0, min(60.0, 3.0 * args.steps)))
    line = dict(impl="reference", metric="LoD decode queries/s (batch 4 x 64 heads at 128K context, one layer)",
                value=rate, unit="queries/s", n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64 (oracle)",
                data="synthetic", config=dict(workload=w.name, B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                                              seq_len=w.T, l2="cpu"),
                cpu_baseline=dict(value=rate, unit="queries/s", cores=cores, kind="oracle", sample=sample),
                e2e=dict(value=rate, unit="queries/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_gqa_128k_bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the prefill/build/oracle legs")
    ap.add_argument("--graphs", type=int, default=1, help="e2e: one CUDA graph per step (0 = eager)")
    ap.add_argument("--replicas", type=int, default=4,
                    help="decode: device replicas of the inputs used in rotation (1 = flush L2 instead)")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="N > 1: every rank its own batch (weak scaling) or the KV heads split over ranks (strong)")
    ap.add_argument("--leg", default=None, choices=["prefill", "build"],
                    help="run only this secondary leg and print its result (profiler captures)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="with --leg: context length of the leg's workload (0 = its own)")
    ap.add_argument("--kv-bits", type=int, default=0, choices=[0, 4],
                    help="main decode leg in three-tier INT4 (opened pages from 4-bit codes)")
    ap.add_argument("--clusters", type=int, default=4, help="with --leg build: clusters per chunk")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per step (0 = the workload's own; smaller cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from hierarchical_long_context_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.batch > 0:
        w = w.with_(B=args.batch)
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return
    if args.leg:  # one secondary leg alone, on one GPU
        peaks = load_peaks()
        dev = torch.device("cuda", torch.cuda.current_device())
        name = "prefill_128k_bf16" if args.leg == "prefill" else "build_128k_bf16"
        wl = synth.WORKLOADS[name]
        if args.seq_len:
            wl = wl.with_(T=args.seq_len)
        r = (run_prefill(wl, dev, torch.cuda.current_stream(), 2, peaks) if args.leg == "prefill" else
             run_build(wl, dev, torch.cuda.current_stream(), 5, peaks, args.clusters))
        print(json.dumps(r), flush=True)
        return
    wg = w
    w = synth.shard(w, args.shard, rank, world)
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    res = run_decode(w, args, dev, stream, world, rank, peaks)
    res.pop("_touch")
    extras = {}
    if not args.no_extras:
        extras["decode_int4"] = run_decode_variant(
            w, dev, stream, peaks, 1000, 4,
            "%s, three-tier INT4 (opened pages read from 4-bit codes)" % w.name, kv_bits=4)
        torch.cuda.empty_cache()
        extras["decode_two_tier"] = run_decode_variant(
            w.with_(top_pages=0), dev, stream, peaks, 1000, 4,
            "%s, two-tier LoD (top_pages = 0: opened groups read whole)" % w.name)
        torch.cuda.empty_cache()
        extras["decode_1m"] = run_decode_variant(
            synth.WORKLOADS["decode_gqa_1m_bf16"], dev, stream, peaks, 500, 4,
            "decode_gqa_1m_bf16: one sequence at 1M context (device-generated inputs)", device_gen=True)
        torch.cuda.empty_cache()
        extras["decode_32k"] = run_decode_variant(
            synth.WORKLOADS["decode_gqa_32k_bf16"], dev, stream, peaks, 1000, 4,
            "decode_gqa_32k_bf16: batch 8 at 32K context")
        torch.cuda.empty_cache()
        wp = synth.WORKLOADS["prefill_128k_bf16"]
        extras["prefill"] = run_prefill(wp, dev, stream, 3, peaks)
        wb = synth.WORKLOADS["build_128k_bf16"]
        extras["build"] = run_build(wb, dev, stream, 5, peaks, 4)
        extras["build_k8"] = run_build(wb, dev, stream, 5, peaks, 8)
        torch.cuda.empty_cache()
        extras["dense_reference"] = run_dense(dev, stream)
        for nm, leg in (("decode_gqa_32k_bf16", extras["decode_32k"]), ("decode_gqa_128k_bf16", res),
                        ("prefill_128k_bf16", extras["prefill"])):
            dref = extras["dense_reference"].get(nm, {})
            if "ms_per_step" in dref:
                dref["lod_speedup"] = dref["ms_per_step"] / leg["ms_per_step"]
        if rank == 0 and world == 1:
            rate, sample, cores = oracle_decode_rate(w)
            extras["cpu_baseline"] = dict(value=rate, unit="queries/s", cores=cores, kind="oracle", sample=sample)
            extras["cpu_oracle"] = oracle_prefill_and_build()
    barrier(world)
    if rank == 0:
        line = dict(metric=res["metric"], value=res["value"], unit=res["unit"], n_gpus=world,
                    steps=args.steps, warmup=args.warmup, ms_per_step=res["ms_per_step"],
                    higher_is_better=True, scaling="strong" if args.shard == "heads" and world > 1 else "weak",
                    vs_baseline=None, dtype="bf16",
                    data="synthetic (seeded Gaussian-mixture keys + RoPE + outlier channels, N(0,1) values)",
                    config=dict(workload=w.name, B=wg.B, Hq=wg.Hq, Hkv=wg.Hkv, d=w.d, seq_len=w.T,
                                clusters=w.clusters[0], top_groups=w.top_groups, top_pages=w.top_pages,
                                kv_bits=args.kv_bits,
                                window=w.window, sinks=w.sinks,
                                parallelism=("heads x%d" if args.shard == "heads" else "replicas x%d") % world,
                                l2=res["l2"]),
                    roofline=res["roofline"], cpu_baseline=extras.pop("cpu_baseline", None),
                    e2e=res["e2e"], gpu_launches=res["gpu_launches"], clocks=res["clocks"],
                    ms_p10=res["ms_p10"], ms_p90=res["ms_p90"], head_rows_per_s=res["head_rows_per_s"],
                    status_word=res["status_word"], **extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
