"""Benchmark of the W4A16 g128 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-breakdown]

Workload (one "step", the configuration the headline metric is quoted on):
28 Qwen3-1.7B-shaped decoder blocks, 7 linears each (q/o 2048->2048,
k/v 2048->1024, gate/up 2048->6144, down 6144->2048; 1.409e9 weights), bf16
weights N(0, 0.02), int4 asymmetric g128.  A step runs
  (1) quantize+pack of all 196 weights (bf16 -> packed int4 + fp16 scales and
      zeros) through the batched entry point (64 tensors per launch), then
  (2) the decode W4A16 GEMV through all 196 linears at M = 1, 4 and 8 tokens
      (bf16 x ~ N(0, 1)).  Every linear has its own input, so the 196 are
      independent problems: the batched entry point decodes up to 256 of them
      in one persistent launch, with programmatic dependent launch.
value = algorithmic bytes of the step / step time (GB/s): 2.53125 B/weight
for quantize, 0.53125 B/weight + 2MK + 2MN bytes per decode linear.  The step
is two CUDA graphs: the quantize launches, then the three decode launches
chained with programmatic dependent launch; its working set (2.8 GB bf16
weights, 0.75 GB packed) is far larger than L2, so no flush is needed between
steps.

Multi-GPU: every rank runs its own replica (the path has no exchange step);
value sums the ranks' bytes over the slowest rank's time ("weak" scaling).

--impl reference: the CPU oracle (numpy) on the host cores, each step a
bounded sample of the same workload (one linear quantized and decoded at
M = 1, 4, 8, rotating through the block's seven shapes).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 g128 linear: decode GB/s & prefill TFLOPS (% roofline); quantize GB/s"
WORKLOAD = "qwen3-1.7b-shaped 28 blocks x 7 linears: int4 asym g128 quantize+pack, then decode GEMV M=1,4,8"
DECODE_M = (1, 4, 8)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) over the
# algorithmic bytes of the same launch, from one ncu capture per kernel (the
# summaries under profiles/ give the commands), with the digest of the kernel
# source the capture was taken on.  A changed source reports traffic null.
TRAFFIC_CAPTURES = {
    # decode_batch --m 1 --blocks 4 (streaming kernel, 28 linears): 110.71 MB
    # (107.27 read + 3.43 written back from the preceding quantize) over
    # 107.27 MB algorithmic
    "gemv_w4a16": {"source": "gemv_stream.cu", "digest": "47877b2f04a984c7",
                   "ratio": (107271424 + 3434240) / 107266048},
    # quantize 17408 x 5120: 202.47 MB over 225.67 MB (part of the written codes
    # is still in the write-back L2 when the kernel ends)
    "quantize_pack": {"source": "quantize.cu", "digest": "f3061dcc5ac9fd85", "ratio": 202.47 / 225.67},
    # linear --m 2048 --k 4096 --n 4096 --sym --gemm: 25.50 MB read (weights +
    # x once; y still in L2 at the end) over 42.21 MB algorithmic
    "gemm_tc": {"source": "gemm_tc.cu", "digest": "f309caed81658b75",
                "ratio": (25504512 + 6400) / 42205184},
}

LLAMA2_LINEARS = ((4096, 4096, 4), (4096, 11008, 2), (11008, 4096, 1))

# --------------------------------------------------------------------------


def roofline_entry(kernel, bound, achieved, peak, unit, peak_kind, bytes_per_launch, share,
                   flops_per_launch=None):
    cap = TRAFFIC_CAPTURES.get(kernel)
    traffic = None
    if cap and source_digest(cap["source"]) == cap["digest"]:
        traffic = cap["ratio"] * bytes_per_launch
    e = {"kernel": kernel, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
         "algorithmic_bytes_per_launch": bytes_per_launch, "step_share": share}
    if flops_per_launch is not None:
        e["algorithmic_flops_per_launch"] = flops_per_launch
    return e


def source_digest(name):
    import hashlib
    path = os.path.join(ROOT, "weight_only_int4_quantize_b200", "csrc", name)
    try:
        return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return None


def max_over_ranks(dist, t_ms, device):
    """Replica timing: the slowest rank's time (every rank calls this once)."""
    import torch
    t = torch.tensor([float(t_ms)], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_rank, max_ms):
    """Whole-job throughput of `world` replicas over the slowest rank's time."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


def quant_bytes(n, k, sym=False):
    return n * k * (2 + 0.5 + (2 if sym else 4) / 128)


def gemv_bytes(m, n, k, sym=False):
    return n * k * (0.5 + (2 if sym else 4) / 128) + 2 * m * k + 2 * m * n


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def block_shapes():
    from weight_only_int4_quantize_b200 import synth
    return [(name, k, n) for name, k, n in synth.QWEN3_1P7B_BLOCK]


def step_bytes():
    shapes = block_shapes()
    blocks = 28
    q = sum(quant_bytes(n, k) for _, k, n in shapes) * blocks
    d = sum(gemv_bytes(m, n, k) for m in DECODE_M for _, k, n in shapes) * blocks
    return q, d


# ----------------------------------------------------------- clocks --------

class ClockSampler:
    """nvidia-smi samples every 100 ms, each stamped with the host time it
    arrived; the summary keeps those inside the window marked by start() and
    stop() (the timed region), or all of them if none fell inside."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, cmd=None, first_wait_s: float = 3.0):
        self.proc = None
        self.cmd = cmd or ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                           "--format=csv,noheader,nounits", "-lms", "100"]
        self.first_wait_s = first_wait_s
        self.samples = []  # (host monotonic time, line)
        self.window = (None, None)
        self._reader = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.monotonic(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()
        # Sampling is running before the timed region starts.
        t_end = time.monotonic() + self.first_wait_s
        while not self.samples and time.monotonic() < t_end and self.proc.poll() is None:
            time.sleep(0.01)
        return self

    def start(self):
        self.window = (time.monotonic(), None)

    def stop(self):
        self.window = (self.window[0], time.monotonic())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self._reader is not None:
            self._reader.join(timeout=5)

    def summary(self):
        t0, t1 = self.window
        inside = [ln for t, ln in self.samples
                  if t0 is not None and t1 is not None and t0 <= t <= t1]
        lines = inside or [ln for _, ln in self.samples]
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm),
                "window": "timed region" if inside else "whole sampler run"}


# ------------------------------------------------------------ CPU leg ------

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(step_index: int):
    """One bounded sample of the workload on the CPU oracle: one linear of the
    block (rotating through the 7 shapes) quantized+packed, then decoded at
    M = 1, 4, 8 in binary64.  Returns (algorithmic bytes, seconds)."""
    import torch
    from oracle import w4_oracle as O
    from weight_only_int4_quantize_b200 import synth
    name, k, n = block_shapes()[step_index % 7]
    w = synth.bits(synth.normal_weight(n, k, 0.02, seed=9000 + step_index % 7))
    xs = [synth.bits(synth.normal_activations(m, k, seed=9100 + m)) for m in DECODE_M]
    t0 = time.perf_counter()
    codes, s16, z16 = O.quantize_rtn(w, False)
    O.pack_codes(codes)
    what = O.dequantize(codes, s16, z16)
    for x in xs:
        O.linear(x, what)
    dt = time.perf_counter() - t0
    nbytes = quant_bytes(n, k) + sum(gemv_bytes(m, n, k) for m in DECODE_M)
    del torch
    return nbytes, dt


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _timed(fn, min_s):
    """Calls fn until min_s seconds have passed (at least once); returns
    (calls, seconds)."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            return n, dt


def cpu_parts(threads, min_s=1.5):
    """The oracle's pieces on this host at a given BLAS thread count:
    quantize+pack GB/s (2048 x 2048, asymmetric), binary64 GEMV (M = 1) and
    GEMM (M = 512) GFLOP/s on a 4096 x 4096 dequantized weight, and AWQ grid
    candidates/s on k_proj (2048 calibration tokens, 2048 -> 1024, 2 x 2
    grid)."""
    from threadpoolctl import threadpool_limits
    from oracle import w4_oracle as O
    from weight_only_int4_quantize_b200 import synth
    out = {"threads": threads}
    with threadpool_limits(limits=threads):
        w = synth.bits(synth.normal_weight(2048, 2048, 0.02, seed=9300, n_outliers=8,
                                           outlier_scale=20.0))
        n, dt = _timed(lambda: O.pack_codes(O.quantize_rtn(w, False)[0]), min_s)
        out["quantize_gbs"] = n * quant_bytes(2048, 2048) / dt / 1e9
        wb = synth.bits(synth.normal_weight(4096, 4096, 0.02, seed=9301))
        codes, s16, _ = O.quantize_rtn(wb, True)
        what = O.dequantize(codes, s16, None)
        for m, key in ((1, "gemv_f64_gflops"), (512, "gemm_f64_gflops")):
            x = synth.bits(synth.normal_activations(m, 4096, seed=9302 + m))
            n, dt = _timed(lambda: O.linear(x, what), min_s)
            out[key] = n * 2.0 * m * 4096 * 4096 / dt / 1e9
        xk = synth.bits(synth.student_t_calibration(2048, 2048, seed=9304))
        wk = synth.bits(synth.normal_weight(1024, 2048, 0.02, seed=9305))
        al, sh = synth.alpha_grid(20)[[5, 10]], synth.shrink_grid(10)[:2]
        n, dt = _timed(lambda: O.awq_score_grid(xk, wk, al, sh, False), min_s)
        out["awq_kproj_candidates_per_s"] = n * len(al) * len(sh) / dt
    return out


def cpu_baseline(target_s=12.0):
    """The oracle as it stands, timed on this host on a bounded sample (the
    headline figure), plus its pieces at one BLAS thread and at all."""
    tot_b, tot_t, i = 0.0, 0.0, 0
    while tot_t < target_s and i < 196:
        b, t = oracle_sample(i)
        tot_b += b
        tot_t += t
        i += 1
    out = {"value": tot_b / tot_t / 1e9, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
           "sample": f"{i} linears of the Qwen3-1.7B-shaped blocks (rotating shapes): numpy binary32 "
                     f"quantize+pack, then binary64 decode at M=1,4,8; {tot_t:.1f} s",
           "nproc": os.cpu_count(), "cpu_model": cpu_model(),
           "omp_num_threads": os.environ.get("OMP_NUM_THREADS")}
    try:
        out["parts"] = [cpu_parts(1), cpu_parts(cpu_threads())]
    except Exception as e:  # threadpoolctl missing or a BLAS it cannot limit
        out["parts_error"] = f"{type(e).__name__}: {e}"
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for i in range(args.warmup):
        oracle_sample(i)
    tot_b, tot_t = 0.0, 0.0
    for i in range(args.steps):
        b, t = oracle_sample(i)
        tot_b += b
        tot_t += t
    v = tot_b / tot_t / 1e9
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32+f64",
            "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one linear per step, rotating shapes"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "kind": "oracle", "cores": cpu_threads(),
                             "sample": "one Qwen3-1.7B-block linear per step (rotating), "
                                       "quantize+pack + decode M=1,4,8"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU leg ------

class Model:
    """196 linears of the workload resident on one GPU, plus the step graphs."""

    def __init__(self, dev, seed_base=1000):
        import torch
        self.torch = torch
        self.dev = dev
        g = torch.Generator(device=dev)
        self.lin = []  # (k, n, w_bf16, qw, sc, zr)
        for b in range(28):
            for i, (name, k, n) in enumerate(block_shapes()):
                g.manual_seed(seed_base + 7 * b + i)
                w = (torch.randn(n, k, generator=g, device=dev) * 0.02).to(torch.bfloat16)
                qw = torch.empty(n, k // 8, dtype=torch.int32, device=dev)
                sc = torch.empty(n, k // 128, dtype=torch.int16, device=dev)
                zr = torch.empty(n, k // 128, dtype=torch.int16, device=dev)
                self.lin.append((k, n, w, qw, sc, zr))
        self.x = {}
        self.y = {}
        for m in DECODE_M:
            for k in sorted({k for _, k, _ in block_shapes()}):
                g.manual_seed(77 + m * 10 + k)
                self.x[(m, k)] = torch.randn(m, k, generator=g, device=dev).to(torch.bfloat16)
            self.y[m] = [torch.empty(m, n, dtype=torch.bfloat16, device=dev)
                         for (_, n, *_r) in self.lin]
        import weight_only_int4_quantize_b200 as w4
        # Prepared item arrays for the batched entry points.
        self.q_items = w4.quantize_pack_items([(w, None, 1.0, qw, sc, zr)
                                               for (k, n, w, qw, sc, zr) in self.lin])
        self.d_items = {m: w4.linear_items([(self.x[(m, k)], qw, sc, zr, self.y[m][j])
                                            for j, (k, n, w, qw, sc, zr) in enumerate(self.lin)])
                        for m in DECODE_M}
        # w4a16_linear_batched (M <= 8) runs up to STREAM_BATCH linears per
        # persistent launch.
        self.launches = {"quantize": -(-len(self.lin) // 64),
                         "gemv": len(DECODE_M) * -(-len(self.lin) // w4.STREAM_BATCH)}

    def quantize_all(self):
        """All 196 weights through w4_quantize_pack_batched (64 per launch)."""
        import weight_only_int4_quantize_b200 as w4
        w4.quantize_pack_batched(self.q_items, False,
                                 stream=self.torch.cuda.current_stream(self.dev).cuda_stream)

    def decode_all(self, m, flags):
        """All 196 linears (independent inputs) through w4a16_linear_batched
        (one persistent launch)."""
        import weight_only_int4_quantize_b200 as w4
        w4.w4a16_linear_batched(self.d_items[m], m, flags,
                                stream=self.torch.cuda.current_stream(self.dev).cuda_stream)


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm (attributes, lazy loading) outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def time_graph(torch, g, iters, warm=3):
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def breakdown(torch, dev, hbm, bf16_peak, bf16_sus):
    """Secondary measurements (outside the headline timed region): the other
    configurations of the metric, each timed with CUDA events on graphs."""
    import weight_only_int4_quantize_b200 as w4
    from weight_only_int4_quantize_b200 import synth
    out = {}
    g = torch.Generator(device=dev)

    def weights(n, k, std, seed, n_out=0, scale=1.0):
        g.manual_seed(seed)
        w = torch.randn(n, k, generator=g, device=dev) * std
        if n_out:
            ch = torch.randperm(k, generator=g, device=dev)[:n_out]
            w[:, ch] *= scale
        return w.to(torch.bfloat16)

    pdl_static = w4.LINEAR_PDL | w4.LINEAR_STATIC_WEIGHTS

    # Single linear K = N = 2048, 8 input channels x20, asymmetric g128:
    # quantize+pack and decode at M = 1 and 16.  120 copies (264 MB of bf16
    # weights, 264 MB packed) are used in turn, more than twice the 126 MB L2,
    # so the figures are HBM figures.
    copies = 120
    ws_bf = [weights(2048, 2048, 0.02, 9000 + c, 8, 20.0) for c in range(copies)]
    packed1 = [w4.quantize_pack(wb, False) for wb in ws_bf]
    q_items = w4.quantize_pack_items([(wb, None, 1.0, qw, sc, zr)
                                      for wb, (qw, sc, zr) in zip(ws_bf, packed1)])

    def run_q():
        w4.quantize_pack_batched(q_items, False, stream=torch.cuda.current_stream(dev).cuda_stream)
    gq = capture(torch, run_q)
    t = time_graph(torch, gq, 10)
    out["cfg1_quantize_2048x2048_outliers"] = {
        "ms_per_weight": t / copies, "gbs": copies * quant_bytes(2048, 2048) / t / 1e6,
        "frac_hbm": copies * quant_bytes(2048, 2048) / t / 1e6 / hbm, "copies": copies}
    del gq, q_items, ws_bf
    for m in (1, 16):
        x1 = torch.randn(m, 2048, generator=g, device=dev).to(torch.bfloat16)
        y1 = torch.empty(m, 2048, dtype=torch.bfloat16, device=dev)

        def run_l(x1=x1, y1=y1):
            for qw, sc, zr in packed1:
                w4.w4a16_linear(x1, qw, sc, zr, flags=pdl_static, out=y1)
        gl = capture(torch, run_l)
        t = time_graph(torch, gl, 10) / copies
        byts = gemv_bytes(m, 2048, 2048)
        out[f"cfg1_decode_2048x2048_M{m}"] = {
            "ms_per_linear": t, "gbs": byts / t / 1e6, "frac_hbm": byts / t / 1e6 / hbm,
            "copies": copies, "launches": "one w4a16_linear per copy, PDL, one CUDA graph"}
        del gl
    del packed1
    torch.cuda.empty_cache()

    # Prefill / M-sweep on the Llama-2-7B- and 27B-shaped linears (symmetric).
    lin_sets = {
        "llama2_7b": [(k, n, c) for k, n, c in synth.LLAMA2_7B_LINEARS],
        "27b": [(k, n, 1) for k, n in synth.SCALE27B_LINEARS],
    }
    for tag, shapes in lin_sets.items():
        # The 27B-scale trio (119 MB packed) fits L2: three copies of it are
        # used in turn (357 MB), so the decode sizes read HBM.
        n_copies = 3 if tag == "27b" else 1
        sets = []
        for c in range(n_copies):
            packed = []
            for i, (k, n, cnt) in enumerate(shapes):
                w = weights(n, k, 0.02 if tag == "llama2_7b" else 0.015, 500 + i + 31 * c,
                            0 if tag == "llama2_7b" else k // 100, 10.0)
                qw, sc, _ = w4.quantize_pack(w, True)
                packed.append((k, n, cnt, qw, sc))
                del w
            sets.append(packed)
        packed = sets[0]
        ms = (512, 2048) if tag == "llama2_7b" else (1, 8, 64, 512, 4096)
        for m in ms:
            xs = {k: torch.randn(m, k, generator=g, device=dev).to(torch.bfloat16)
                  for k in {p[0] for p in packed}}
            ys = [torch.empty(m, p[1], dtype=torch.bfloat16, device=dev) for p in packed]
            fl = pdl_static if m <= 8 else 0

            def run():
                for pk in sets:
                    for (k, n, cnt, qw, sc), y in zip(pk, ys):
                        for _ in range(cnt):
                            w4.w4a16_linear(xs[k], qw, sc, None, flags=fl, out=y)
            gr = capture(torch, run)
            t = time_graph(torch, gr, 20 if m >= 512 else 50) / n_copies
            flops = sum(2.0 * m * n * k * cnt for k, n, cnt, *_ in packed)
            byts = sum(gemv_bytes(m, n, k, True) * cnt for k, n, cnt, *_ in packed)
            rec = {"ms": t, "tflops": flops / t / 1e9, "gbs": byts / t / 1e6}
            rec["frac_bf16_peak"] = rec["tflops"] / bf16_peak
            rec["frac_hbm"] = rec["gbs"] / hbm
            if n_copies > 1:
                rec["copies"] = n_copies
            out[f"{tag}_M{m}"] = rec
            if m >= 512:
                # The same linears as one batched call (independent problems):
                # grouped prefill launches share the GPU between linears.
                ys_g = [torch.empty(m, n, dtype=torch.bfloat16, device=dev)
                        for (k, n, cnt, qw, sc) in packed for _ in range(cnt)]
                arr = w4.linear_items([(xs[k], qw, sc, None, yg) for (k, n, cnt, qw, sc), yg in
                                       zip([p for p in packed for _ in range(p[2])], ys_g)])
                gr2 = capture(torch, lambda arr=arr, m=m: w4.w4a16_linear_batched(arr, m))
                t2 = time_graph(torch, gr2, 20)
                out[f"{tag}_M{m}_grouped"] = {"ms": t2, "tflops": flops / t2 / 1e9,
                                              "frac_bf16_peak": flops / t2 / 1e9 / bf16_peak}
                del gr2, arr, ys_g
            del gr, xs, ys
        del packed, sets
    torch.cuda.empty_cache()

    # AWQ grid, one Qwen3-1.7B block (q,k,v,o,gate,up share K=2048), 20 x 10 grid.
    g.manual_seed(41)
    k = 2048
    z0 = torch.randn(k, generator=g, device=dev, dtype=torch.float64)
    chi = (torch.randn(3, k, generator=g, device=dev, dtype=torch.float64) ** 2).sum(0)
    c = (z0 / torch.sqrt(chi / 3)).abs().float()
    x = (torch.randn(2048, k, generator=g, device=dev) * c[None, :]).to(torch.bfloat16)
    rows = [n for name, kk, n in block_shapes() if kk == 2048]
    w = torch.cat([weights(n, k, 0.02, 600 + i) for i, n in enumerate(rows)], 0)
    seg = [0]
    for n in rows:
        seg.append(seg[-1] + n)
    al, sh = synth.alpha_grid(20), synth.shrink_grid(10)
    ws = torch.empty(w4.awq_workspace_bytes(2048, w.shape[0], k, 20, 10, len(rows)),
                     dtype=torch.uint8, device=dev)
    w4.awq_score_grid(x, w, al, sh, False, seg_offsets=seg, workspace=ws)
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    a_ev.record()
    for _ in range(reps):
        sse, arg = w4.awq_score_grid(x, w, al, sh, False, seg_offsets=seg, workspace=ws)
    b_ev.record()
    torch.cuda.synchronize()
    t = a_ev.elapsed_time(b_ev) / reps
    flops = 2.0 * 2048 * k * w.shape[0] * 200
    out["awq_qwen_block_20x10"] = {"ms": t, "tflops": flops / t / 1e9,
                                   "frac_bf16_peak": flops / t / 1e9 / bf16_peak,
                                   "candidates": 200, "linears": len(rows),
                                   "argmins_group": arg[-1].tolist()}
    del ws, w

    # Per-output-channel clipping search on one Qwen gate_proj (2048 -> 6144)
    # at alpha 0.5 over the 10-point grid, then the deploy quantize.
    wg = weights(6144, k, 0.02, 700)
    s05 = w4.awq_scales(x, [0.5])[0].contiguous()
    cws = torch.empty(w4.clip_rows_workspace_bytes(2048, 6144, k, 10), dtype=torch.uint8,
                      device=dev)
    # Outputs preallocated and the C entry point called directly inside a CUDA
    # graph: the timing sees the kernels only, not allocator work between
    # the short calls.
    sh32 = np.ascontiguousarray(np.asarray(sh, dtype=np.float32))
    sse_r = torch.empty((10, 6144), dtype=torch.float64, device=dev)
    choice = torch.empty(6144, dtype=torch.int32, device=dev)
    rows_r = torch.empty(6144, dtype=torch.float32, device=dev)

    def run_clip():
        st = w4.lib().awq_clip_search_rows(
            x.data_ptr(), 2048, wg.data_ptr(), 6144, k, 128, 0, s05.data_ptr(),
            sh32.ctypes.data, 10, sse_r.data_ptr(), choice.data_ptr(), rows_r.data_ptr(),
            cws.data_ptr(), cws.numel(), torch.cuda.current_stream(dev).cuda_stream)
        assert st == 0, st
    gclip = capture(torch, run_clip)
    t = time_graph(torch, gclip, 10)
    del gclip
    flops = 2.0 * 2048 * k * 6144 * 10
    out["clip_rows_qwen_gate_2048tok_10r"] = {
        "ms": t, "tflops": flops / t / 1e9, "frac_bf16_peak": flops / t / 1e9 / bf16_peak,
        "candidates": 10, "rows": 6144,
        "rows_per_ratio": torch.bincount(choice.long(), minlength=10).tolist()}
    del cws, wg, x
    torch.cuda.empty_cache()

    # Block-level (look-ahead) search of one Qwen3-1.7B-shaped block: T =
    # 2048 tokens entering block i, block i+1 unquantized, the 20 x 10 grid
    # (alpha* per group: 4 x 20 candidates, then a ratio per linear: 7 x 10),
    # every candidate screened (tcgen05 fp16 products of each linear's change,
    # binary64 epilogues and attention), near ties decided in binary64.
    gi = {k: v.to(dev) for k, v in synth.qwen_block(3).items()}
    gn = {k: v.to(dev) for k, v in synth.qwen_block(4).items()}
    xb = synth.block_input(2048, 2048, seed=77).to(dev)
    wsb = torch.empty(w4.block_workspace_bytes(2048), dtype=torch.uint8, device=dev)
    al, sh = synth.alpha_grid(20), synth.shrink_grid(10)
    w4.awq_block_search(xb, gi, gn, al[:1], sh[:1], False, workspace=wsb)  # warm
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record()
    choice, _ = w4.awq_block_search(xb, gi, gn, al, sh, False, workspace=wsb)
    b_ev.record()
    torch.cuda.synchronize()
    t = a_ev.elapsed_time(b_ev)
    out["block_search_qwen_T2048_20x10_lookahead"] = {
        "ms": t, "candidates": 4 * 20 + 7 * 10, "candidates_per_s": 150 / (t * 1e-3),
        "workspace_gb": wsb.numel() / 1e9, "choice": choice.tolist(),
        "precision": "screened: tcgen05 fp16 change products with binary64 epilogues; "
                     "near ties (1e-3) decided on the binary64 path"}
    del gi, gn, xb, wsb
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import weight_only_int4_quantize_b200 as w4

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    w4.lib()
    hbm, bf16_peak, bf16_sus, peak_kind = peaks()

    model = Model(dev, seed_base=1000 + 97 * rank)
    flags = w4.LINEAR_PDL | w4.LINEAR_STATIC_WEIGHTS
    g_q = capture(torch, model.quantize_all)
    # The decode phase: the three token counts' launches chained in one graph
    # (programmatic dependent launch: each launch's weight stream starts while
    # the previous one drains, as consecutive decode steps run in serving).
    # The weights were written by the quantize graph, which has completed.
    g_dc = capture(torch, lambda: [model.decode_all(m, flags) for m in DECODE_M])
    # The same launches one per graph (isolated: ramp and tail exposed).
    g_d = {m: capture(torch, lambda m=m: model.decode_all(m, flags)) for m in DECODE_M}
    launches_per_step = model.launches["quantize"] + model.launches["gemv"]
    qb, db = step_bytes()
    db_m = {m: sum(gemv_bytes(m, n, k) for _, k, n in block_shapes()) * 28 for m in DECODE_M}

    def step():
        g_q.replay()
        g_dc.replay()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        clk.start()
        start.record()
        for i in range(args.steps):
            e = ev[i]
            e[0].record()
            g_q.replay()
            e[1].record()
            g_dc.replay()
            e[2].record()
        end.record()
        torch.cuda.synchronize()
        clk.stop()
    if pg:
        pg.barrier()
    total_ms = start.elapsed_time(end)
    total_ms = max_over_ranks(pg, total_ms, dev)
    ms_step = total_ms / args.steps
    q_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    gemv_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    value = whole_job_gbs(world, qb + db, ms_step)
    clocks = clk.summary()
    # Per token count: each launch alone in its graph, after the quantize
    # graph as in the step (outside the timed region).
    n_iso = max(10, min(50, args.steps))
    iso = {m: [] for m in DECODE_M}
    for _ in range(n_iso):
        g_q.replay()
        for m in DECODE_M:
            a_i, b_i = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_i.record()
            g_d[m].replay()
            b_i.record()
            iso[m].append((a_i, b_i))
    torch.cuda.synchronize()
    d_ms = {m: sum(a_i.elapsed_time(b_i) for a_i, b_i in iso[m]) / n_iso for m in DECODE_M}
    del g_d
    # Steady-state decode: the chained decode graph replayed back to back, as
    # consecutive decode steps run (no quantize in between: the quantize
    # graph leaves dirty packed weights in the write-back L2, which the step's
    # decode phase writes back to HBM).
    g_dc.replay()
    torch.cuda.synchronize()
    a_s, b_s = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_s.record()
    for _ in range(n_iso):
        g_dc.replay()
    b_s.record()
    torch.cuda.synchronize()
    steady_ms = a_s.elapsed_time(b_s) / n_iso

    # ---------------------------------------------- end to end (host buffers)
    # Per step: H2D of every bf16 weight and x from pinned memory, the same
    # quantize + decode through the C ABI, D2H of the packed weights and y.
    host_w = [w.cpu().pin_memory() for (_, _, w, *_r) in model.lin]
    host_x = {key: t.cpu().pin_memory() for key, t in model.x.items()}
    host_q = [(torch.empty_like(qw, device="cpu").pin_memory(),
               torch.empty_like(sc, device="cpu").pin_memory(),
               torch.empty_like(zr, device="cpu").pin_memory()) for (_, _, _, qw, sc, zr) in model.lin]
    host_y = {m: [torch.empty_like(y, device="cpu").pin_memory() for y in model.y[m]] for m in DECODE_M}
    h2d = sum(t.numel() * 2 for t in host_w) + sum(t.numel() * 2 for t in host_x.values())
    d2h = sum(sum(t.numel() * t.element_size() for t in q) for q in host_q) + \
        sum(t.numel() * 2 for m in DECODE_M for t in host_y[m])

    def e2e_step():
        for hw, (_, _, w, *_r) in zip(host_w, model.lin):
            w.copy_(hw, non_blocking=True)
        for key, t in model.x.items():
            t.copy_(host_x[key], non_blocking=True)
        model.quantize_all()
        for m in DECODE_M:
            model.decode_all(m, 0)
        for (hq, hs, hz), (_, _, _, qw, sc, zr) in zip(host_q, model.lin):
            hq.copy_(qw, non_blocking=True)
            hs.copy_(sc, non_blocking=True)
            hz.copy_(zr, non_blocking=True)
        for m in DECODE_M:
            for hy, y in zip(host_y[m], model.y[m]):
                hy.copy_(y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(2, min(5, args.steps))
    if pg:
        pg.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n_e2e):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(pg, a.elapsed_time(b) / n_e2e, dev)
    e2e_val = whole_job_gbs(world, qb + db, e2e_ms)
    del host_w, host_x, host_q, host_y

    # ---------------------------------------------- W4A8 decode (same weights)
    # The decode phase again with int8 activations: each distinct x is
    # quantized once per token count, then one batched W4A8 call over all 196
    # linears (CUDA graph; outside the headline timed region).
    w4a8 = {}
    for m in DECODE_M:
        qx = {key: w4.quantize_act_int8(t) for key, t in model.x.items() if key[0] == m}
        a8 = w4.a8_items([(*qx[(m, k)], qw, sc, zr, model.y[m][j])
                          for j, (k, n, w, qw, sc, zr) in enumerate(model.lin)])

        def run_a8(m=m, qx=qx, a8=a8):
            for key, t in model.x.items():
                if key[0] == m:
                    xq, xs, sx = qx[key]
                    w4.lib().w4_quantize_act_int8(t.data_ptr(), m, t.shape[1], xq.data_ptr(),
                                                  xs.data_ptr(), sx.data_ptr(),
                                                  torch.cuda.current_stream(dev).cuda_stream)
            w4.w4a8_linear_batched(a8, m, flags,
                                   stream=torch.cuda.current_stream(dev).cuda_stream)
        g8 = capture(torch, run_a8)
        t8 = time_graph(torch, g8, 50)
        w4a8[f"M{m}"] = {"ms": t8, "gbs": db_m[m] / (t8 * 1e-3) / 1e9,
                         "frac_hbm": db_m[m] / (t8 * 1e-3) / 1e9 / hbm}
        del g8, a8, qx

    # ---------------------------------------------- roofline (per kernel)
    # One entry per hot kernel, the step's dominant one first: achieved =
    # algorithmic bytes (FLOPs) of its launches in the timed region / their
    # CUDA-event time; traffic = the ncu capture's DRAM bytes / algorithmic
    # bytes of the captured launch, times this launch's algorithmic bytes
    # (null once the kernel source differs from the capture's).
    roofline = [
        roofline_entry("quantize_pack", "hbm", qb / (q_ms * 1e-3) / 1e9, hbm, "GB/s", peak_kind,
                       qb / model.launches["quantize"], q_ms / (q_ms + gemv_ms)),
        roofline_entry("gemv_w4a16", "hbm", db / (gemv_ms * 1e-3) / 1e9, hbm, "GB/s", peak_kind,
                       db / model.launches["gemv"], gemv_ms / (q_ms + gemv_ms)),
    ]
    roofline.sort(key=lambda r: -r["step_share"])

    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4 codes/bf16 x/f32 accum",
        "data": "synthetic (seeded, generated on device)",
        "config": {"workload": WORKLOAD, "linears": len(model.lin), "weights": 1.409e9,
                   "decode_M": list(DECODE_M), "parallelism": f"replicas x{world}",
                   "l2": "working set 3.6 GB >> 126 MB L2 (no flush needed)",
                   "graph": "one CUDA graph per phase; the 196 linears are independent "
                            "problems, batched: 4 quantize launches + 1 decode launch per M",
                   "l2_note": "inputs (3.6 GB) exceed L2; no flush"},
        "phases": {"quantize_ms": q_ms, "quantize_gbs": qb / (q_ms * 1e-3) / 1e9,
                   "decode_ms": gemv_ms, "decode_gbs": db / (gemv_ms * 1e-3) / 1e9,
                   "decode_note": "decode_ms: the M = 1, 4, 8 launches chained (PDL) in one "
                                  "graph, as timed in the step; decode_M*_isolated: each "
                                  "launch alone in its graph after the quantize graph",
                   "decode_steady_ms": steady_ms,
                   "decode_steady_gbs": db / (steady_ms * 1e-3) / 1e9,
                   "decode_steady_note": "the chained decode graph replayed back to back "
                                         "(consecutive decode steps, no quantize between)",
                   **{f"decode_M{m}_isolated_ms": d_ms[m] for m in DECODE_M},
                   **{f"decode_M{m}_isolated_gbs": db_m[m] / (d_ms[m] * 1e-3) / 1e9
                      for m in DECODE_M}},
        "roofline": roofline,
        "w4a8_decode": w4a8,
        "clocks": clocks,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline()
    # The breakdown (about a minute of single-GPU measurements) runs only at
    # N = 1: under torchrun the other ranks would wait for it at the final
    # barrier against the process group's timeout.
    if rank == 0 and world == 1 and not args.no_breakdown:
        del g_q, g_dc, model
        torch.cuda.empty_cache()
        out["breakdown"] = breakdown(torch, dev, hbm, bf16_peak, bf16_sus)
        pf = out["breakdown"].get("llama2_7b_M2048")
        if pf:
            # Prefill (tcgen05) on the Llama-2-7B-shaped linears at M = 2048:
            # 7 launches per graph replay, timed burst-length.
            flops_l = 2.0 * 2048 * sum(n * k * c for k, n, c in LLAMA2_LINEARS) / 7
            byts_l = sum((n * k * (0.5 + 2 / 128) + 2 * 2048 * (k + n)) * c
                         for k, n, c in LLAMA2_LINEARS) / 7
            out["roofline"].append(roofline_entry(
                "gemm_tc", "tensor", pf["tflops"], bf16_peak, "TFLOP/s", peak_kind, byts_l, None,
                flops_per_launch=flops_l))
    err = w4.device_error(clear=True)
    if err:
        out["device_error"] = err
    if rank == 0:
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
