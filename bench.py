"""Benchmark one MLA decode layer step on B200.

A step is the whole decode path for one token per sequence: cache append
(down-projection, latent RMSNorm, RoPE key), query absorption, split-KV latent
decode, log-sum-exp combine and the W^UV output projection, on synthetic
inputs already resident in HBM.  Sequence lengths are reset after each step so
every step appends at the same position and attends over N + 1 rows.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the float64 CPU oracle, bounded sample)

Multi-GPU: one process per GPU under torch.distributed.run; sequences are
independent, so each rank runs its own batch with no data-path collective
(weak scaling); time = max over ranks of the CUDA-event time.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/s and latent-cache GB/s, TFLOP/s as % of B200 roofline"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(
            j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _decode_source_hash():
    h = hashlib.sha256()
    for name in ("k_decode_tc.cu", "tile_deal.cuh", "common.cuh", "sm100.cuh"):
        with open(os.path.join(ROOT, "mla_latent_kv_nope_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _ncu_traffic(workload):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu
    summary, only if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
        e = j[workload]
        if e.get("source_hash") == _decode_source_hash():
            return float(e["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


_SAMPLER_SRC = r"""
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[1]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    t = time.time()
    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
    print(f"{t:.4f} {sm} {rs}", flush=True)
    time.sleep(0.002)
"""


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML during the timed
    steps: every ~2 ms by a separate process (samples inside the [start, stop]
    window kept), and, while the GPU is still working through the enqueued
    steps, by this process itself (``poll_until``), so even a short timed
    region is sampled."""
    REASONS = {  # NVML clocks-event-reason bits
        0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, index):
        self.index = index
        self.t_start = self.t_stop = None
        self.inproc = []   # (sm_mhz, reasons) read while the timed steps ran

    def poll_until(self, done, nvml=None, max_samples=100000):
        """Read the SM clock and throttle reasons until ``done()`` is true (the
        end-of-timing event has completed).  Never raises: on any NVML error
        the process sampler's readings stand alone."""
        try:
            if nvml is None:
                import pynvml as nvml
            nvml.nvmlInit()
            h = nvml.nvmlDeviceGetHandleByIndex(int(self.index))
            while len(self.inproc) < max_samples and not done():
                self.inproc.append((int(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM)),
                                    int(nvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                time.sleep(0.0002)
        except Exception:
            pass

    def __enter__(self):
        import subprocess
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_SRC, str(self.index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            first = self.proc.stdout.readline().split()
            self.max_mhz = int(first[1]) if first and first[0] == "max" else None
        except Exception:
            self.proc = None
        return self

    def start(self):
        self.t_start = time.time()

    def stop(self):
        self.t_stop = time.time()

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
                self.lines = out.splitlines()
            except Exception:
                self.proc.kill()

    def summary(self, window=None):
        """Median SM clock and the reasons seen in the timed window, or, with
        ``window = (t0, t1)`` (host times), in that window from the separate
        process's samples alone."""
        rows = list(self.inproc) if window is None else []
        t_start, t_stop = window if window is not None else (self.t_start, self.t_stop)
        for ln in getattr(self, "lines", []):
            f = ln.split()
            if len(f) != 3:
                continue
            t, sm, rs = float(f[0]), int(f[1]), int(f[2])
            if t_start is not None and not (t_start <= t <= t_stop):
                continue
            rows.append((sm, rs))
        if not rows:
            return None
        sms = sorted(r[0] for r in rows)
        reasons = set()
        for _, rs in rows:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        source = ("NVML during the timed steps (this process while they run, and a "
                  "separate process every ~2 ms inside the window)" if window is None else
                  "NVML every ~2 ms (a separate process) during this pass")
        return {"sm_mhz": sms[len(sms) // 2], "sm_max_mhz": getattr(self, "max_mhz", None),
                "sm_min_mhz": sms[0], "samples": len(rows), "reasons": sorted(reasons),
                "source": source}


# ---------------------------------------------------------------------------
def _algorithmic(w, lens_after, fp8=False):
    """Latent-cache bytes and FLOPs of one decode launch (cache read once;
    QK^T over d_c + d_r and P.c over d_c per head and cached row).  An FP8
    cache row is d_c code bytes + d_r bf16 RoPE keys + a 4-byte scale."""
    rows = int(sum(int(x) for x in lens_after))
    elem = 2 if w.dtype == "bf16" else 4
    row_bytes = (w.d_c + 2 * w.d_r + 4) if fp8 else w.R * elem
    return rows * row_bytes, 2.0 * w.H * rows * (w.R + w.d_c), rows


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import mla_latent_kv_nope_b200 as mla
    from mla_latent_kv_nope_b200 import dist as mdist
    from mla_latent_kv_nope_b200 import inputs
    from mla_latent_kv_nope_b200.build import build

    if rank == 0:
        build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = mdist.shard(inputs.WORKLOADS[args.workload], rank)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dims = mla.Dims(w.B, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, w.capacity, w.dtype)

    lens = inputs.seqlens(w)
    fp8 = args.cache == "fp8"
    scales = None
    if fp8:
        # The FP8 cache drawn in its stored format (codes, power-of-two
        # scales, bf16 RoPE keys); the append writes its own rows.
        cache = torch.empty(w.B, w.capacity, w.d_c + 2 * w.d_r, dtype=torch.uint8, device=dev)
        scales = torch.empty(w.B, w.capacity, dtype=torch.float32, device=dev)
        inputs.fill_fp8_cache(w, cache, scales, lens, fill_rest_byte=0)
    else:
        cache = torch.empty(w.B, w.capacity, w.R, dtype=dt, device=dev)
        inputs.fill_cache(w, cache, lens, fill_rest=0.0)
    table = None
    if args.paged:
        # The same rows in a pool of 64-row pages, pages shuffled, and the
        # block table that finds them; every call below reads the pool.
        nb = (w.capacity + mla.PAGE_ROWS - 1) // mla.PAGE_ROWS
        padded = torch.zeros(w.B, nb * mla.PAGE_ROWS, w.R, dtype=dt, device=dev)
        padded[:, :w.capacity] = cache
        perm = torch.from_numpy(np.random.default_rng(1).permutation(w.B * nb)).to(dev)
        cache = torch.empty(w.B * nb, mla.PAGE_ROWS, w.R, dtype=dt, device=dev)
        cache[perm] = padded.reshape(w.B * nb, mla.PAGE_ROWS, w.R)
        table = perm.to(torch.int32).reshape(w.B, nb).contiguous()
        del padded
    seq0 = torch.from_numpy(lens).to(dev)
    seq = seq0.clone()
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    h, Wdkv = inputs.append_inputs(w)
    T = lambda a: torch.from_numpy(a).to(dev, dt)  # noqa: E731
    q_nope, q_pe, W_UK, W_UV, hh, W_DKV = map(T, (qn, qp, Wuk, Wuv, h, Wdkv))
    q_pos = seq0.clone()  # the appended token's position
    step = mla.DecodeStep(dims, W_UK, W_UV, W_DKV, num_splits=args.splits)
    stream = torch.cuda.current_stream()

    cache_bytes = cache.numel() * cache.element_size() + (scales.numel() * 4 if fp8 else 0)
    flush = None
    if cache_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def eager_step():
        if flush is not None:
            flush.zero_()
        step(q_nope, q_pe, q_pos, cache, seq, h=hh, block_table=table, scales=scales)
        seq.copy_(seq0)

    # A step is replayed from a CUDA graph (one host launch per step) unless
    # --eager; the graph holds every kernel of the step, each run every replay.
    for _ in range(2):
        eager_step()
    torch.cuda.synchronize()
    if args.eager:
        one_step = eager_step
    else:
        graph = step.capture(q_nope, q_pe, q_pos, cache, seq, h=hh,
                             before=(flush.zero_ if flush is not None else None),
                             after=lambda: seq.copy_(seq0), block_table=table, scales=scales)
        one_step = graph.replay

    # Decode-kernel time for the roofline, in a separate pass so the step
    # timing has no extra event records inside it.  A CUDA graph holds kRep
    # decode launches (and another kRep decode + combine pairs); CUDA events
    # around its replays on the launching stream give the average launch
    # duration with no host launch cost in between (launching each decode
    # from Python with events around it measured the host, not the kernel).
    # Where the cache fits in L2 the graphs also flush L2 before each decode;
    # a graph of the flushes alone is timed and subtracted.
    kRep = 8

    def dec_call():
        if fp8:
            mla.decode_fp8(dims, step.q_cat, cache, scales, seq, step.scale, step.ws,
                           step.num_splits)
        elif table is None:
            mla.decode(dims, step.q_cat, cache, seq, step.scale, step.ws, step.num_splits)
        else:
            mla.decode_paged(dims, step.q_cat, cache, table, seq, step.scale, step.ws,
                             step.num_splits)

    def body(with_decode, with_combine):
        def run():
            for _ in range(kRep):
                if flush is not None:
                    flush.zero_()
                if with_decode:
                    dec_call()
                if with_combine:
                    mla.combine(dims, seq, step.ws, step.splits_used, step.o_lat, step.lse)
        return run

    def graph_of(fn):
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    def decode_only(n):
        step.append(hh, cache, seq, table, scales)
        mla.absorb_q(dims, q_nope, q_pe, W_UK, q_pos, step.q_cat, step.rope_base)
        graphs = [graph_of(body(True, False)), graph_of(body(True, True))]
        if flush is not None:
            graphs.append(graph_of(body(False, False)))
        reps = max(1, n // kRep)
        per = []
        for g in graphs:
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            per.append(e0.elapsed_time(e1) / (reps * kRep))
        base = per[2] if flush is not None else 0.0
        seq.copy_(seq0)
        torch.cuda.synchronize()
        return per[0] - base, per[1] - base

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during warm-up")

    def barrier():
        mdist.barrier(world)

    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.start()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            one_step()
        t1.record(stream)
        clk.poll_until(t1.query)
        torch.cuda.synchronize()
        clk.stop()
        barrier()
        ms_total = t0.elapsed_time(t1)
        t_dec = time.time()
        dec_avg, decomb_avg = decode_only(max(args.steps, 5 * kRep))
        t_dec = (t_dec, time.time())
    ms_total = mdist.max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / args.steps

    # e2e through the public API with host buffers: pinned H2D of the step's
    # inputs (q_nope, q_pe, q_pos, h) and D2H of the output, every step.
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    h_qn, h_qp, h_pos, h_h = pin(q_nope), pin(q_pe), pin(q_pos), pin(hh)
    h_out = torch.empty(step.out.shape, dtype=dt).pin_memory()
    bi = sum(t.numel() * t.element_size() for t in (h_qn, h_qp, h_pos, h_h))
    bo = h_out.numel() * h_out.element_size()

    host_in = (h_qn, h_qp, h_pos, h_h)

    if args.eager:
        # One step at a time: inputs in, step, output out, all on one stream.
        def e2e_run(n):
            for _ in range(n):
                for d_t, h_t in zip((q_nope, q_pe, q_pos, hh), host_in):
                    d_t.copy_(h_t, non_blocking=True)
                if flush is not None:
                    flush.zero_()
                step(q_nope, q_pe, q_pos, cache, seq, h=hh, block_table=table, scales=scales)
                h_out.copy_(step.out, non_blocking=True)
                seq.copy_(seq0)
    else:
        # Pipelined through DecodeStep.host_pipeline: one graph launch per
        # step runs the step on one device input set while a copy stream
        # brings the next step's inputs in from pinned host memory and takes
        # the previous step's output out; every step still copies its own
        # inputs and result.
        def after():
            if flush is not None:
                flush.zero_()
            seq.copy_(seq0)
        pipe = step.host_pipeline(host_in, h_out, cache, seq, after=after, block_table=table,
                                  scales=scales)
        assert pipe.bytes_per_step() == (bi, bo)

        def e2e_run(n):
            pipe.run(n)

    e2e_run(3)
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    e2e_run(args.steps)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / args.steps
    e2e_ms = mdist.max_over_ranks(e2e_ms, world, dev)
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during timing")

    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_src = _peaks()
    lens_after = lens + 1
    byts, flops, rows = _algorithmic(w, lens_after, fp8)
    achieved_gbs = byts / (dec_avg * 1e-3) / 1e9
    achieved_tf = flops / (dec_avg * 1e-3) / 1e12
    t_roof = max(byts / (hbm * 1e9), flops / (tf_burst * 1e12))
    bound = "hbm" if byts / (hbm * 1e9) >= flops / (tf_burst * 1e12) else "tensor"
    tokens = w.B * world
    res = {
        "metric": METRIC,
        "value": mdist.job_tokens_per_s(w.B, world, ms_step),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded; N(0,1) latents/queries, N(0,0.02^2) weights)",
        "config": {
            "workload": _workload_desc(w),
            "global_batch": w.B * world,
            "seq_len": int(lens_after.max()),
            "parallelism": f"dp{world}",
            "l2": ("inputs exceed L2 (cache %.0f MB)" % (cache_bytes / 1e6)) if flush is None
                  else "L2 flushed between steps",
            "num_splits": step.splits_used,
            "cache": ("paged: 64-row pages, shuffled, block table" if args.paged
                      else "fp8: E4M3 latent codes + bf16 RoPE keys (640 B) + fp32 scale per token"
                      if fp8 else "contiguous [B, capacity, 576]"),
            "launch": "eager" if args.eager else "cuda_graph (absorb_q on a forked stream)",
        },
        "decode_only": {
            "timing": f"CUDA events around replays of a graph of {kRep} back-to-back launches",
            "ms": dec_avg, "ms_with_combine": decomb_avg,
            "tokens_per_s": w.B / (decomb_avg * 1e-3),
            "latent_cache_GBps": achieved_gbs, "TFLOPs": achieved_tf,
            "roofline_us": t_roof * 1e6,
            "frac_of_roofline": t_roof / (dec_avg * 1e-3),
            "frac_of_roofline_with_combine": t_roof / (decomb_avg * 1e-3),
            "hbm_frac": achieved_gbs / hbm, "tensor_frac_burst": achieved_tf / tf_burst,
            "tensor_frac_sustained": achieved_tf / tf_sus,
            # This pass runs right after the timed steps; under that much
            # back-to-back decode work the power cap can lower the SM clock.
            "clocks": clk.summary(t_dec),
        },
        "roofline": {
            "kernel": "mla_decode (split-KV latent attention)",
            "bound": bound,
            "achieved": achieved_gbs if bound == "hbm" else achieved_tf,
            "peak": hbm if bound == "hbm" else tf_burst,
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": (achieved_gbs / hbm) if bound == "hbm" else (achieved_tf / tf_burst),
            "traffic": _ncu_traffic(args.workload + ("_fp8" if fp8 else "")),
            "algorithmic_bytes_per_launch": byts,
            "algorithmic_flops_per_launch": flops,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured"
                           else "fallback",
        },
        "e2e": {"value": mdist.job_tokens_per_s(w.B, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms},
        "gpu_launches": 6 * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_oracle_baseline(w, args.cpu_seconds, fp8)
    return res


# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _workload_desc(w):
    return (f"{w.name}: B={w.B} H={w.H} d_c={w.d_c} d_r={w.d_r} d_nope={w.d_nope} "
            f"d_v={w.d_v} N={w.N}{' ragged' if w.ragged else ''} per GPU, "
            f"append hidden={w.hidden}")


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


class OracleSampler:
    """The float64 materialised-MHA oracle, as it stands, timed on a bounded
    sample of a workload: whole (sequence, head) pairs, one appended token
    each.  The inputs and the cache rows of up to ``max_seqs`` randomly chosen
    sequences are generated once; each ``run(budget_s)`` then times pairs
    (cycling through the sample) until about ``budget_s`` of oracle time and
    scales to tokens/s by the number of (sequence, head) pairs in a step."""

    def __init__(self, w, max_seqs=8, fp8=False):
        import numpy as np

        from mla_latent_kv_nope_b200 import inputs

        self.w = w
        self.np = np
        self.lens = inputs.seqlens(w)
        self.qn, self.qp = inputs.query(w)
        self.Wuk, self.Wuv = inputs.weights(w)
        self.h, self.Wdkv = inputs.append_inputs(w)
        f = lambda a: a.astype(np.float64)  # noqa: E731
        self.Wdkv64 = f(self.Wdkv)
        rng = np.random.default_rng(0)
        seqs = sorted(int(b) for b in rng.choice(w.B, size=min(max_seqs, w.B), replace=False))
        self.caches = {}
        self.fp8 = fp8
        for b in seqs:
            L = int(self.lens[b])
            c = np.zeros((1, L + 1, w.R))
            if fp8:
                from oracle import mla_oracle as O
                codes, k, rope = inputs.fp8_cache_rows(w, b, L)
                c[0, :L, :w.d_c] = O.dequantize_latent_rows(codes, np.ldexp(1.0, k))
                c[0, :L, w.d_c:] = rope
            else:
                c[0, :L] = inputs.cache_rows(w, b, L)
            self.caches[b] = c
        self.pairs = [(b, int(i)) for i in rng.permutation(w.H) for b in seqs]
        self.k = 0

    def run(self, budget_s):
        from oracle import mla_oracle as O

        np, w = self.np, self.w
        f = lambda a: a.astype(np.float64)  # noqa: E731
        done, spent = 0, 0.0
        while spent < budget_s:
            b, i = self.pairs[self.k % len(self.pairs)]
            self.k += 1
            L = int(self.lens[b])
            t0 = time.perf_counter()
            c2, L2, _ = O.cache_append(self.caches[b], np.array([L]), f(self.h[b:b + 1]),
                                       self.Wdkv64, w.d_c, eps=w.eps)
            O.mla_decode_materialised(f(self.qn[b:b + 1, i:i + 1]), f(self.qp[b:b + 1, i:i + 1]),
                                      [L], f(self.Wuk[i:i + 1]), f(self.Wuv[i:i + 1]), c2, L2,
                                      w.softmax_scale)
            spent += time.perf_counter() - t0
            done += 1
        step_s = spent / done * w.B * w.H
        return {"value": w.B / step_s, "unit": "tokens/s", "cores": _blas_threads(),
                "kind": "oracle", "extrapolated": True, "cpu_model": _cpu_model(),
                "host_cores": os.cpu_count(),
                "sample": f"{done} (sequence, head) pairs from {len(self.caches)} seeded random "
                          f"{'FP8 (dequantised) ' if self.fp8 else ''}"
                          f"sequences ({spent:.1f} s of oracle time), each append + "
                          f"materialised attention over its full length; scaled by "
                          f"B*H = {w.B * w.H} pairs per step"}


def cpu_oracle_baseline(w, budget_s=15.0, fp8=False):
    return OracleSampler(w, fp8=fp8).run(budget_s)


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle on this arm's workload (rank 0 only)."""
    if rank != 0:
        return None
    from mla_latent_kv_nope_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    # About 90 s of oracle work for the whole run, whatever K and W are.
    budget = max(0.05, min(20.0, 90.0 / max(1, args.steps + args.warmup)))
    sampler = OracleSampler(w)
    vals = []
    for k in range(args.warmup + args.steps):
        r = sampler.run(budget)
        if k >= args.warmup:
            vals.append(r)
    v = sum(r["value"] for r in vals) / len(vals)
    ms = w.B / v * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": _workload_desc(w), "global_batch": w.B * world,
                   "seq_len": w.N + 1, "parallelism": "cpu (oracle, rank 0)"},
        # Each step times a bounded sample of (sequence, head) pairs; the step
        # time is the sampled per-pair time x B*H pairs (extrapolated).
        "extrapolated": True,
        "cpu_baseline": {"kind": "oracle", "cores": vals[-1]["cores"], "sample": vals[-1]["sample"],
                         "value": v, "unit": "tokens/s", "extrapolated": True},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_folded_out_proj(args, rank, world, local_rank):
    """The W^O fold variant alone ([MLA-とは] "Value側の吸収"): u = sum_i B_i
    o_lat_i with B_i = W^O_i W^UV_i folded once, d_model = the workload's
    hidden width.  One launch set per step (bf16 rounding of o_lat, the
    weight-streaming tcgen05 kernel, the split reduction); the folded weight
    (H d_model d_c bf16) exceeds L2, so no flush is needed.  Each rank times
    its own copy (no collective)."""
    import torch

    import mla_latent_kv_nope_b200 as mla
    from mla_latent_kv_nope_b200 import dist as mdist
    from mla_latent_kv_nope_b200 import inputs
    from mla_latent_kv_nope_b200.build import build

    if rank == 0:
        build()
    if world > 1:
        mdist.barrier(world)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = inputs.WORKLOADS[args.workload]
    d_model = w.hidden
    dims = mla.Dims(w.B, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, w.capacity, w.dtype)
    _, Wuv = inputs.weights(w)
    W_UV = torch.from_numpy(Wuv).to(dev, torch.bfloat16)
    W_O = torch.from_numpy(inputs.normal((d_model, w.H * w.d_v), w.w_std, w.seed, 41,
                                         d_model)).to(dev, torch.bfloat16)
    o_lat = torch.from_numpy(inputs.normal((w.B, w.H, w.d_c), 0.05, w.seed, 123, 1)).to(dev)
    W_fold = torch.empty(d_model, w.H * w.d_c, dtype=torch.bfloat16, device=dev)
    mla.fold_output_weights(dims, W_O, W_UV, W_fold)
    del W_O
    u = torch.empty(w.B, d_model, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(mla.out_proj_folded_workspace_bytes(dims, d_model), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        mla.out_proj_folded(dims, o_lat, W_fold, u, ws)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        mdist.barrier(world)
        torch.cuda.synchronize()
        clk.start()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            mla.out_proj_folded(dims, o_lat, W_fold, u, ws)
        t1.record(stream)
        clk.poll_until(t1.query)
        torch.cuda.synchronize()
        clk.stop()
        mdist.barrier(world)
    ms = mdist.max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during timing")
    if rank != 0:
        return None
    hbm, _, _, peak_src = _peaks()
    byts = w.H * d_model * w.d_c * 2 + w.B * w.H * w.d_c * 4 + w.B * d_model * 2
    unfolded = w.H * w.d_v * w.d_c * 2 + d_model * w.H * w.d_v * 2
    gbs = byts / (ms * 1e-3) / 1e9
    return {
        "metric": "folded output projection weight-stream GB/s", "value": gbs, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)",
        "config": {"workload": f"folded out-proj B={w.B} H={w.H} d_c={w.d_c} d_v={w.d_v} "
                               f"d_model={d_model}", "l2": "folded weight exceeds L2"},
        "roofline": {"kernel": "folded_proj_tc_kernel + to_bf16 + split reduction",
                     "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "traffic": None, "algorithmic_bytes_per_launch": byts,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)"
                                    if peak_src == "measured" else "fallback"},
        # The unfolded form reads W^UV and W^O instead of the folded weight.
        "unfolded_weight_bytes": unfolded, "folded_weight_bytes": w.H * d_model * w.d_c * 2,
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }


def run_prefill(args, rank, world, local_rank):
    """The materialised prefill alone ([MLA-とは] "実装上のトレードオフ"): one
    sequence of T = L prompt tokens whose latent rows are already cached, at
    the workload's head shape; query t at position t.  A step is one
    mla_prefill call (query rotation, the K^C/V up-projection GEMM, causal
    attention).  Each rank times its own sequence (no collective)."""
    import numpy as np
    import torch

    import mla_latent_kv_nope_b200 as mla
    from mla_latent_kv_nope_b200 import dist as mdist
    from mla_latent_kv_nope_b200 import inputs
    from mla_latent_kv_nope_b200.build import build

    if rank == 0:
        build()
    if world > 1:
        mdist.barrier(world)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = inputs.WORKLOADS[args.workload]
    T = L = args.prefill_tokens
    w = base.scaled(B=1, N=L, seed=base.seed + rank)
    dims = mla.Dims(1, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, 1, w.dtype)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev, torch.bfloat16)  # noqa: E731
    q_nope = bf(inputs.normal((T, w.H, w.d_nope), 1.0, w.seed, 61, T))
    q_pe = bf(inputs.normal((T, w.H, w.d_r), 1.0, w.seed, 62, T))
    Wuk, Wuv = inputs.weights(w)
    W_UK, W_UV = bf(Wuk), bf(Wuv)
    rows = bf(inputs.cache_rows(w, 0, L))
    q_pos = torch.arange(T, dtype=torch.int32, device=dev)
    out = torch.empty(T, w.H, w.d_v, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(T, w.H, dtype=torch.float32, device=dev)
    ws = torch.empty(mla.prefill_workspace_bytes(dims, T, L), dtype=torch.uint8, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        mla.prefill(dims, q_nope, q_pe, q_pos, W_UK, W_UV, rows, out, ws, lse=lse)

    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    evs = []
    with ClockSampler(local_rank) as clk:
        mdist.barrier(world)
        torch.cuda.synchronize()
        clk.start()
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            evs.append((e0, e1))
        clk.poll_until(evs[-1][1].query)
        torch.cuda.synchronize()
        clk.stop()
        mdist.barrier(world)
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    ms = mdist.max_over_ranks(ms, world, dev)
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during timing")
    if rank != 0:
        return None
    _, tf_burst, tf_sus, peak_src = _peaks()
    pairs = T * (T + 1) // 2                          # causal (query, row) pairs
    flops_attn = 2.0 * pairs * w.H * (w.d_nope + w.d_r + w.d_v)
    flops_kv = 2.0 * L * w.d_c * w.H * (w.d_nope + w.d_v)
    flops = flops_attn + flops_kv
    tf = flops / (ms * 1e-3) / 1e12
    tokens_s = T * world / (ms * 1e-3)
    return {
        "metric": "MLA materialised prefill tokens/s and TFLOP/s", "value": tokens_s,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": f"prefill T=L={T} H={w.H} d_c={w.d_c} d_r={w.d_r} "
                               f"d_nope={w.d_nope} d_v={w.d_v}, causal, q_pos = 0..T-1",
                   "l2": "L2 flushed between calls"},
        "roofline": {"kernel": "mla_prefill (q rotation + K/V up-projection + causal attention)",
                     "bound": "tensor", "achieved": tf, "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": tf / tf_burst, "frac_sustained": tf / tf_sus, "traffic": None,
                     "algorithmic_flops_per_launch": flops, "attention_flops": flops_attn,
                     "kv_projection_flops": flops_kv,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)"
                                    if peak_src == "measured" else "fallback"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }


def run_seqshard(args, rank, world, local_rank):
    """Long-context sequence sharding: every rank holds one contiguous token
    range of every sequence (dist.token_ranges) and runs absorb + decode +
    combine on it; the per-range (o_lat, lse) are all-gathered (NCCL), merged
    by log-sum-exp (mla_merge_partials) and projected by W^UV.  The batch is
    the same on every rank, so total work is fixed as N grows (strong
    scaling).  Timed on the device, max over ranks; the collective is inside
    the timed region."""
    import numpy as np
    import torch

    import mla_latent_kv_nope_b200 as mla
    from mla_latent_kv_nope_b200 import dist as mdist
    from mla_latent_kv_nope_b200 import inputs
    from mla_latent_kv_nope_b200.build import build

    if rank == 0:
        build()
    if world > 1:
        mdist.barrier(world)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = inputs.WORKLOADS[args.workload]
    lens = inputs.seqlens(w)
    ranges = mdist.token_ranges(lens, world)[rank]
    loc = (ranges[:, 1] - ranges[:, 0]).astype(np.int32)
    cap = max(int(loc.max()), 1)
    cap = (cap + 63) // 64 * 64
    dims = mla.Dims(w.B, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, cap, w.dtype)
    cache = torch.zeros(w.B, cap, w.R, dtype=torch.bfloat16, device=dev)
    for b in range(w.B):
        lo, hi = int(ranges[b, 0]), int(ranges[b, 1])
        if hi > lo:
            cache[b, :hi - lo].copy_(torch.from_numpy(inputs.cache_rows(w, b, hi)[lo:hi]))
    local_seq = torch.from_numpy(loc).to(dev)
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    T = lambda a: torch.from_numpy(a).to(dev, torch.bfloat16)  # noqa: E731
    q_nope, q_pe, W_UK, W_UV = map(T, (qn, qp, Wuk, Wuv))
    q_pos = torch.from_numpy((lens - 1).astype(np.int32)).to(dev)
    step = mla.DecodeStep(dims, W_UK, W_UV, None, num_splits=args.splits)
    stream = torch.cuda.current_stream()

    def one():
        mdist.sequence_sharded_attend(step, q_nope, q_pe, q_pos, cache, local_seq, world)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during warm-up")
    with ClockSampler(local_rank) as clk:
        mdist.barrier(world)
        torch.cuda.synchronize()
        clk.start()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            one()
        t1.record(stream)
        clk.poll_until(t1.query)
        torch.cuda.synchronize()
        clk.stop()
        mdist.barrier(world)
    ms = mdist.max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    if mla.get_device_status() != 0:
        raise RuntimeError("device status error during timing")
    if rank != 0:
        return None
    hbm, _, _, peak_src = _peaks()
    byts = int(lens.sum()) * w.R * 2
    gbs = byts / (ms * 1e-3) / 1e9
    return {
        "metric": METRIC + " (sequence-sharded)", "value": w.B / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded)",
        "config": {"workload": _workload_desc(w) + f", each rank a token range (<= {cap} rows)",
                   "global_batch": w.B, "seq_len": int(lens.max()),
                   "parallelism": f"seq{world}", "launch": "eager",
                   "l2": "inputs exceed L2" if byts > 2 * L2_BYTES else "per-rank cache may fit L2"},
        "roofline": {"kernel": "whole sharded attend (absorb, decode, combine, all-gather, merge, "
                               "out_proj) over the whole job's cache bytes",
                     "bound": "hbm", "achieved": gbs * 1.0, "peak": hbm * world, "unit": "GB/s",
                     "frac": gbs / (hbm * world), "traffic": None,
                     "algorithmic_bytes_per_step": byts,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json, x n_gpus)"
                                    if peak_src == "measured" else "fallback x n_gpus"},
        "gpu_launches": (6 if world > 1 else 4) * args.steps,
        "clocks": clk.summary(),
    }


def _relaunch_per_gpu(n):
    """`--gpus N` (N > 1) started without a launcher: run this same command as
    N ranks, one process per GPU, under torch.distributed.run (rendezvous on
    127.0.0.1); rank 0 prints the JSON line.  Returns the launcher's exit code."""
    import socket
    import subprocess

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def run_dry(args, rank, world):
    """Host-only check of the multi-rank plumbing (gloo, no GPU, no kernels):
    each rank 'steps' for a rank-dependent time, the job time is the maximum
    over ranks, and rank 0 reports the world size it ran with.  Its numbers
    are not measurements of the decode."""
    import datetime

    import torch.distributed as dist

    from mla_latent_kv_nope_b200 import dist as mdist

    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        per_step = 1e-3 * (rank + 1)
        for _ in range(args.warmup):
            time.sleep(per_step)
        mdist.barrier(world)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            time.sleep(per_step)
        ms = (time.perf_counter() - t0) * 1e3
        ms_max = mdist.max_over_ranks(ms, world)
        mdist.barrier(world)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank != 0:
        return None
    return {"dry_run": True, "metric": METRIC, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "rank0_ms_per_step": ms / args.steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="v3_bf16")
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="latent cache format (fp8: E4M3 codes with a power-of-two scale "
                         "per token, bf16 RoPE keys)")
    ap.add_argument("--paged", action="store_true",
                    help="keep the latent cache in shuffled 64-row pages behind a block table")
    ap.add_argument("--eager", action="store_true",
                    help="launch each kernel from the host every step instead of a CUDA graph")
    ap.add_argument("--kernel", default="step",
                    choices=["step", "folded_out_proj", "prefill", "seqshard"],
                    help="step: the whole decode step (default); folded_out_proj: the W^O "
                         "fold variant of the output projection alone; prefill: the "
                         "materialised prefill of one sequence; seqshard: attention with the "
                         "cache split by token range over the ranks (use with "
                         "--workload longctx_bf16)")
    ap.add_argument("--prefill-tokens", type=int, default=4096,
                    help="prompt length T = L of --kernel prefill")
    ap.add_argument("--dry-run", action="store_true",
                    help="host-only check of the multi-rank launch and timing (gloo, no GPU)")
    args = ap.parse_args()
    if args.cache == "fp8" and args.paged:
        ap.error("the FP8 latent cache is contiguous only")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        sys.exit(_relaunch_per_gpu(args.gpus))
    world = int(world_env or "1")
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {world} rank(s)")
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.dry_run:
        res = run_dry(args, rank, world)
    elif args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        if args.kernel == "folded_out_proj":
            res = run_folded_out_proj(args, rank, world, local_rank)
        elif args.kernel == "prefill":
            res = run_prefill(args, rank, world, local_rank)
        elif args.kernel == "seqshard":
            res = run_seqshard(args, rank, world, local_rank)
        else:
            res = run_ours(args, rank, world, local_rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
