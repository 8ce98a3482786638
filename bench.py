#!/usr/bin/env python
"""Benchmark of the quantized linear layer hot path on B200.

Default workload (the one the headline metric is quoted on): the W4A16 decode sweep,
Llama-2-7B-shaped layers, M in {1,4,16,32} x (K,N) in {(4096,12288), (4096,4096),
(4096,22016), (11008,4096)}, bf16 activations, group-128 asymmetric INT4 weights.
One step = the 16 fused dequant-GEMM calls of the sweep on one batch of synthetic
input (weights quantized once, resident in HBM).  The value is algorithmic HBM
bytes per second over the timed steps: packed weights + fp16 scales + u8 zeros +
bf16 X + bf16 Y per call.  Weight buffers rotate over enough copies that every
call reads its weights from HBM, not L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-cpu-baseline] [--skip-configs] [--profile]
    python bench.py --single K,N,M [--op w4a16|w8a8|w4a8] [--reps R]   (one call shape)

Besides the headline sweep, rank 0 times the other workloads (W4A16 tiny, W8A8, W4A16
prefill, W4A8) and reports them under "configs".

Under torchrun every rank runs the same workload on its own GPU (replicas, weak
scaling); timing is the max over ranks of CUDA-event time; rank 0 prints one JSON line.
`--impl reference` times the CPU oracle (the deliberately plain reference) on a
bounded sample of the same workload instead.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "quantized GEMM TFLOPS/TOPS and HBM GB/s (% of roofline) at M=1..8192"
# the workload both arms report on (the reference arm times a bounded sample of it and
# says which in its cpu_baseline.sample)
CONFIG = {"workload": "w4a16_decode: M in {1,4,16,32} x (K,N) in {(4096,12288),(4096,4096),"
                      "(4096,22016),(11008,4096)}, group-128 asym INT4, bf16 X/Y",
          "l2": "every call reads its own weight copy; a shape's copies total > 2x L2, so no call "
                "finds its weights in L2",
          "launch": "one CUDA graph per step (16 calls, one decode kernel launch each)"}
# DRAM bytes (read + write) of one decode launch over its algorithmic bytes, from an ncu
# capture of one w4a16_decode_kernel launch at K=4096, N=12288, M=1 (26.403 MB read, no
# write counted, against 26.378 MB algorithmic; the weight stream is read exactly once, so
# traffic scales with the algorithmic bytes of each call).  Take it again whenever the
# decode kernel changes.
DECODE_TRAFFIC_RATIO = 26.403328e6 / (4096 * 12288 // 2 + 4096 // 128 * 12288 * 3 + 2 * 4096 + 2 * 12288)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU (replicas): rank and world from the launcher's environment.
    backend "gloo" (CPU, no device selection) serves the host-side tests."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step, world, steps, ms_max):
    """Whole-job throughput of the replicas: every rank processes one step's bytes per
    step; the time is the slowest rank's (weak scaling)."""
    return bytes_per_step * world * steps / (ms_max * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# W4A16 decode sweep on the GPU
# ---------------------------------------------------------------------------
def l2_bytes():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size


def w4_bytes(K, N):
    return K * N // 2 + (K // 128) * N * 3


class DecodeSweep:
    """All (K, N) x M calls of the decode sweep with weights resident and rotating."""

    def __init__(self, q, seed=0):
        cfg = synth.CONFIGS["w4a16_decode"]
        self.q = q
        self.shapes = []
        L2 = l2_bytes()
        for (K, N) in cfg["KN"]:
            W = torch.from_numpy(synth.workload_weights("w4a16_decode", K, N, seed)).cuda()
            codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
            scales = torch.empty(K // 128, N, dtype=torch.int16, device="cuda")
            zeros = torch.empty(K // 128, N, dtype=torch.uint8, device="cuda")
            packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
            q.qg_quantize_w4_group(W, None, 128, False, codes, scales, zeros)
            q.qg_pack_nibbles(codes, packed)
            del W, codes
            copies = max(len(cfg["M"]) + 1, min(64, math.ceil(2 * L2 / w4_bytes(K, N)) + 1))
            ws = [(packed.clone(), scales.clone(), zeros.clone()) for _ in range(copies)]
            calls = []
            for M in cfg["M"]:
                _, xb = synth.activations(M, K, "bf16", seed=M)
                X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
                Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
                calls.append(dict(M=M, X=X, Y=Y))
            self.shapes.append(dict(K=K, N=N, copies=ws, calls=calls))
        torch.cuda.synchronize()
        assert q.qg_device_status() == q.QG_OK

    def calls(self):
        for sh in self.shapes:
            for c in sh["calls"]:
                yield sh, c

    def bytes_per_step(self):
        return sum(w4_bytes(sh["K"], sh["N"]) + 2 * c["M"] * sh["K"] + 2 * c["M"] * sh["N"] for sh, c in self.calls())

    def flops_per_step(self):
        return sum(2 * c["M"] * sh["K"] * sh["N"] for sh, c in self.calls())

    def launches_per_step(self):
        # every decode call (M <= 32, N % 16 == 0, the workspace path) is one launch of
        # w4a16_decode_kernel: split column slabs are finished inside the kernel
        return sum(1 for _ in self.calls())

    def copy_for(self, sh, s, ci):
        """Weight copy of call ci of shape sh in rotation step s: every call of a step
        reads its own copy, and the copies of a shape (>= 2x L2 in total) are visited in
        turn, so no call finds its weights in L2."""
        cps = sh["copies"]
        return cps[(s * len(sh["calls"]) + ci) % len(cps)]

    def step(self, s):
        q = self.q
        for sh in self.shapes:
            for ci, c in enumerate(sh["calls"]):
                p, sc, z = self.copy_for(sh, s, ci)
                q.qg_gemm_w4a16(c["X"], p, sc, z, c["Y"])

    def n_variants(self):
        # one captured step per rotation index; a step reads > 3x L2 of weights, so a
        # copy read in one step is gone from L2 by the time a later step reads it again
        return max(len(sh["copies"]) for sh in self.shapes)


def capture_graphs(fn, n):
    """One CUDA graph per rotation index (each replays one step)."""
    graphs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n):
            fn(i)                      # warm (sets kernel attributes, caches)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for i in range(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(i)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def time_graphs(graphs, steps, warmup, world):
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        graphs[(warmup + i) % len(graphs)].replay()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)


def per_call_times(sweep, reps=64):
    """Average device time per launch of each (K, N, M) call, rotating weights,
    each call captured alone in a graph of `reps` launches."""
    q = sweep.q
    out = []
    for sh in sweep.shapes:
        for c in sh["calls"]:
            def fn(i, sh=sh, c=c):
                for r in range(reps):   # a different weight copy per launch (> 2x L2 in total)
                    p, sc, z = sh["copies"][(i * reps + r) % len(sh["copies"])]
                    q.qg_gemm_w4a16(c["X"], p, sc, z, c["Y"])
            gs = capture_graphs(fn, 1)
            ms = time_graphs(gs, 5, 2, 1) / 5 / reps
            by = w4_bytes(sh["K"], sh["N"]) + 2 * c["M"] * (sh["K"] + sh["N"])
            out.append(dict(K=sh["K"], N=sh["N"], M=c["M"], us=ms * 1e3, gbs=by / (ms * 1e-3) / 1e9,
                            tflops=2 * c["M"] * sh["K"] * sh["N"] / (ms * 1e-3) / 1e12))
    return out


def e2e_decode(sweep, steps, warmup, world):
    """Same sweep through the public API, eagerly (no graph): every call copies its X
    from pinned host memory to the device, makes the C-ABI call from Python, and copies
    its Y back to pinned host memory, all inside the timed region.  The host-side cost
    of each API call (argument marshalling, launch) is therefore part of the number."""
    q = sweep.q
    host = []
    h2d = d2h = 0
    for sh, c in sweep.calls():
        xh = c["X"].cpu().pin_memory()
        yh = torch.empty(c["Y"].shape, dtype=c["Y"].dtype).pin_memory()
        host.append((sh, c, xh, yh))
        h2d += xh.numel() * 2
        d2h += yh.numel() * 2
    per_shape = {}
    for sh, c, xh, yh in host:
        per_shape.setdefault(id(sh), []).append(c)

    def fn(i):
        for sh, c, xh, yh in host:
            p, sc, z = sweep.copy_for(sh, i, per_shape[id(sh)].index(c))
            c["X"].copy_(xh, non_blocking=True)
            q.qg_gemm_w4a16(c["X"], p, sc, z, c["Y"])
            yh.copy_(c["Y"], non_blocking=True)
    for i in range(warmup):
        fn(i)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(steps):
        fn(warmup + i)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    return ms, h2d, d2h


def cpu_baseline_decode(min_seconds=10.0, col_frac=1, max_reps=20):
    """The oracle, as it stands, on a bounded sample of the sweep: every (K, N, M)
    call restricted to the first N/col_frac output columns, the whole set repeated
    until at least `min_seconds` of CPU time have been spent (at most `max_reps`)."""
    import oracle
    cfg = synth.CONFIGS["w4a16_decode"]
    prepared = []
    for (K, N) in cfg["KN"]:
        Ns = max(8, N // col_frac)
        W = synth.workload_weights("w4a16_decode", K, N)[:, :Ns].copy()
        codes, scales, zeros, _ = oracle.quantize_w4_asym(W)
        packed = oracle.pack_nibbles(codes)
        for M in cfg["M"]:
            X, _ = synth.activations(M, K, "bf16", seed=M)
            prepared.append((K, Ns, M, X, packed, scales, zeros))
    t0 = time.perf_counter()
    by = 0
    reps = 0
    while reps < max_reps and (reps == 0 or time.perf_counter() - t0 < min_seconds):
        for K, Ns, M, X, packed, scales, zeros in prepared:
            oracle.gemm_w4a16_ref(X, packed, scales, zeros)
            by += w4_bytes(K, Ns) + 2 * M * (K + Ns)
        reps += 1
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    return dict(value=by / dt / 1e9, unit="GB/s", cores=cores, kind="oracle",
                sample=f"{reps} pass(es) over all 16 decode-sweep calls on 1/{col_frac} of the output columns "
                       f"({by / 1e6:.1f} MB algorithmic), fp64 reference GEMM with OpenMP, {dt:.2f} s"), dt


def cpu_oracle_rows():
    """The oracle, as it stands, timed beside each of the other workloads on a bounded
    sample (the unit of each sample is stated; the GPU figures are in the same `configs`)."""
    import oracle
    cores = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    out = {"cores": cores, "kind": "oracle"}
    rng = np.random.default_rng(0)
    # W8A8 GEMM, 16 tokens of the 4096 x 11008 layer
    Xq = rng.integers(-127, 128, (16, 4096)).astype(np.int8)
    Wq = rng.integers(-127, 128, (4096, 11008)).astype(np.int8)
    dt = timed(lambda: oracle.gemm_w8a8(Xq, np.ones(16, np.float32), Wq, np.ones(11008, np.float32)))
    out["w8a8_m16"] = {"s": dt, "tops": 2 * 16 * 4096 * 11008 / dt / 1e12}
    # W4A8 GEMM, 1 token of the 8192 x 8192 layer
    p = oracle.pack_nibbles(rng.integers(-7, 8, (8192, 8192)).astype(np.int8))
    sg = np.full((64, 8192), 0.01, np.float32)
    dt = timed(lambda: oracle.gemm_w4a8(rng.integers(-127, 128, (1, 8192)).astype(np.int8), np.ones(1, np.float32),
                                        p, sg))
    out["w4a8_m1"] = {"s": dt, "gbs": (8192 * 8192 // 2 + 4 * 64 * 8192) / dt / 1e9}
    # W4A16 prefill: 2 tokens x K = 8192 x 4096 columns, weights drawn like the prefill layer's
    Wp = synth.weights(8192, 4096, 0.015, 0.005, 8.0)
    c, sc, z, _ = oracle.quantize_w4_asym(Wp)
    pk_ = oracle.pack_nibbles(c)
    X2, _ = synth.activations(2, 8192, "bf16")
    dt = timed(lambda: oracle.gemm_w4a16_ref(X2, pk_, sc, z))
    out["w4a16_prefill_2tok_4096col"] = {"s": dt, "tflops": 2 * 2 * 8192 * 4096 / dt / 1e12}
    # the INT4 quantizer on the 4096 x 12288 decode weight
    Wd = synth.workload_weights("w4a16_decode", 4096, 12288)
    dt = timed(lambda: oracle.quantize_w4_asym(Wd))
    out["quantize_w4_asym"] = {"s": dt, "gbs": (5 * 4096 * 12288) / dt / 1e9}
    # AWQ: 8 calibration tokens, 3 grid points, the 4096 x 12288 layer
    Xc, _ = synth.calibration(4096, synth.CONFIGS["awq"])
    dt = timed(lambda: oracle.awq_search(Xc[:8].copy(), Wd, 3))
    out["awq_search_8tok_3pts"] = {"s": dt}
    # GPTQ of a 512 x 512 weight on 256 tokens
    Xg, _ = synth.activations(256, 512, "bf16")
    dt = timed(lambda: oracle.gptq(Xg, Wd[:512, :512].copy()))
    out["gptq_512x512"] = {"s": dt}
    return out


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle timed on a bounded sample of the workload."""
    if rank != 0:
        return
    col_frac = 8
    times = []
    by = None
    for i in range(args.warmup + args.steps):
        cb, dt = cpu_baseline_decode(min_seconds=0.0, col_frac=col_frac, max_reps=1)
        if i >= args.warmup:
            times.append(dt)
            by = cb["value"] * dt * 1e9
    total = sum(times)
    value = by * len(times) / total / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(CONFIG),
            "cpu_baseline": {"value": value, "unit": "GB/s", "kind": "oracle", "cores": cb["cores"],
                             "sample": cb["sample"]},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the other workloads: W8A8 SmoothQuant, W4A16 prefill, W4A8, W4A16 tiny
# ---------------------------------------------------------------------------
def measure_int8_peak():
    """Dense int8 tensor throughput of this GPU (torch._int_mm, cuBLASLt), 8192^3, best of 10.
    Used only as the roofline denominator of the int8 products."""
    a = torch.randint(-127, 127, (8192, 8192), dtype=torch.int8, device="cuda")
    b = torch.randint(-127, 127, (8192, 8192), dtype=torch.int8, device="cuda")
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = 1e30
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return 2 * 8192 ** 3 / (best * 1e-3) / 1e12


def rotations_for(bytes_per_call):
    """Input copies to rotate over so that the copies together exceed 2x L2."""
    return max(1, math.ceil(2 * l2_bytes() / max(1, bytes_per_call)))


def time_calls(fn, reps, rotations=1):
    """Device time per call: one graph of max(reps, rotations) calls, call r on input
    copy r % rotations.  With `rotations` from rotations_for(), every replay of the
    graph touches more than 2x L2 of inputs and no call finds its inputs in L2."""
    n = max(reps, rotations)

    def body(i):
        for r in range(n):
            fn(r % rotations)
    gs = capture_graphs(body, 1)
    return time_graphs(gs, 5, 2, 1) / 5 / n


def gpu_quant_w4(q, W, s=None, sym=False):
    K, N = W.shape
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    if sym:
        scales = torch.empty(K // 128, N, dtype=torch.float32, device="cuda")
        q.qg_quantize_w4_group(W, s, 128, True, codes, scales, None)
        zeros = None
    else:
        scales = torch.empty(K // 128, N, dtype=torch.int16, device="cuda")
        zeros = torch.empty(K // 128, N, dtype=torch.uint8, device="cuda")
        q.qg_quantize_w4_group(W, s, 128, False, codes, scales, zeros)
    packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(codes, packed)
    return packed, scales, zeros


def x_bf16(name, M, K):
    _, xb = synth.workload_activations(name, M, K)
    return torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)


def bench_configs(q, pk, int8_peak):
    out = {}
    L2 = l2_bytes()
    bf16_peak = pk["bf16_tflops"]
    # --- W4A16 tiny (fp16 X) -------------------------------------------------
    K, N = 1024, 1024
    W = torch.from_numpy(synth.workload_weights("w4a16_tiny", K, N)).cuda()
    pw, sc, z = gpu_quant_w4(q, W)
    _, xb = synth.workload_activations("w4a16_tiny", 1, K)
    X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.float16)
    Y = torch.empty(1, N, dtype=torch.float16, device="cuda")
    by = w4_bytes(K, N) + 2 * (K + N)
    rot = rotations_for(by)
    sets = [(pw, sc, z)] + [(pw.clone(), sc.clone(), z.clone()) for _ in range(rot - 1)]
    ms = time_calls(lambda i: q.qg_gemm_w4a16(X, *sets[i], Y), 64, rot)
    out["w4a16_tiny"] = {"M=1": {"us": ms * 1e3, "gbs": by / (ms * 1e-3) / 1e9,
                                 "roofline_frac": by / (pk["hbm_gbs"] * 1e9) / (ms * 1e-3),
                                 "note": f"parity-size case; weights rotate over {rot} copies (> 2x L2)"}}
    del sets
    # --- W8A8 SmoothQuant: act quant + GEMM ---------------------------------
    cfg = synth.CONFIGS["w8a8"]
    K, N = cfg["KN"][0]
    W = torch.from_numpy(synth.workload_weights("w8a8", K, N)).cuda()
    _, xcb = synth.calibration(K, cfg)
    Xc = torch.from_numpy(xcb.view(np.int16)).cuda().view(torch.bfloat16)
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    q.qg_smooth_scales(Xc, W, 0.5, s, inv)
    Wq = torch.empty(K, N, dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    q.qg_quantize_w8_channel(W, s, Wq, sw)
    rot = max(1, math.ceil(2 * L2 / (K * N)))
    wqs = [Wq] + [Wq.clone() for _ in range(rot - 1)]
    res = {}
    for M in cfg["M"]:
        X = x_bf16("w8a8", M, K)
        Xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        t = torch.empty(M, dtype=torch.float32, device="cuda")
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        by_a = 3 * M * K + 4 * K + 4 * M
        rot_a = min(rotations_for(by_a), 2048)
        xs = [(X, Xq, t)] + [(X.clone(), Xq.clone(), t.clone()) for _ in range(rot_a - 1)]
        ms_a = time_calls(lambda i: q.qg_smooth_quant_act_i8(xs[i][0], inv, xs[i][1], xs[i][2]), 32, rot_a)
        del xs
        ms_g = time_calls(lambda i: q.qg_gemm_w8a8(Xq, t, wqs[i], sw, Y), 32, rot)
        ops = 2 * M * K * N
        by_g = K * N + 4 * N + M * K + 4 * M + 2 * M * N
        t_roof = max(by_g / (pk["hbm_gbs"] * 1e9), ops / (int8_peak * 1e12))
        res[f"M={M}"] = {"act_quant_us": ms_a * 1e3, "act_quant_gbs": by_a / (ms_a * 1e-3) / 1e9,
                         "gemm_us": ms_g * 1e3, "tops": ops / (ms_g * 1e-3) / 1e12, "gbs": by_g / (ms_g * 1e-3) / 1e9,
                         "bound": "hbm" if by_g / (pk["hbm_gbs"] * 1e9) > ops / (int8_peak * 1e12) else "int8 tensor",
                         "roofline_frac": t_roof / (ms_g * 1e-3)}
    out["w8a8"] = res
    del W, Wq, wqs
    # --- W4A8: act quant + GEMM ------------------------------------------------
    cfg = synth.CONFIGS["w4a8"]
    K, N = cfg["KN"][0]
    W = torch.from_numpy(synth.workload_weights("w4a8", K, N)).cuda()
    _, xcb = synth.calibration(K, cfg)
    Xc = torch.from_numpy(xcb.view(np.int16)).cuda().view(torch.bfloat16)
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    q.qg_smooth_scales(Xc, W, 0.5, s, inv)
    pw, sg, _ = gpu_quant_w4(q, W, s, sym=True)
    del W
    wb = K * N // 2 + 4 * (K // 128) * N
    rot = max(1, math.ceil(2 * L2 / wb))
    pws = [(pw, sg)] + [(pw.clone(), sg.clone()) for _ in range(rot - 1)]
    res = {}
    for M in cfg["M"]:
        X = x_bf16("w4a8", M, K)
        Xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        t = torch.empty(M, dtype=torch.float32, device="cuda")
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        q.qg_smooth_quant_act_i8(X, inv, Xq, t)
        ms_g = time_calls(lambda i: q.qg_gemm_w4a8(Xq, t, pws[i][0], pws[i][1], Y), 32, rot)
        ops = 2 * M * K * N
        by_g = wb + M * K + 4 * M + 2 * M * N
        fma_rescale = M * N * (K // 128)
        t_hbm, t_tc = by_g / (pk["hbm_gbs"] * 1e9), ops / (int8_peak * 1e12)
        res[f"M={M}"] = {"gemm_us": ms_g * 1e3, "tops": ops / (ms_g * 1e-3) / 1e12, "gbs": by_g / (ms_g * 1e-3) / 1e9,
                         "bound": "hbm" if t_hbm > t_tc else "int8 tensor + per-group fp32 rescale",
                         "rescale_fma": fma_rescale, "roofline_frac": max(t_hbm, t_tc) / (ms_g * 1e-3)}
    out["w4a8"] = res
    del pws, pw, sg
    # --- W4A16 prefill --------------------------------------------------------
    cfg = synth.CONFIGS["w4a16_prefill"]
    res = {}
    for (K, N) in cfg["KN"]:
        W = torch.from_numpy(synth.workload_weights("w4a16_prefill", K, N)).cuda()
        pw, sc, z = gpu_quant_w4(q, W)
        del W
        torch.cuda.empty_cache()
        wb = w4_bytes(K, N)
        for M in cfg["M"]:
            X = x_bf16("w4a16_prefill", M, K)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            # weight and activation copies alternate so that consecutive calls do not share
            # inputs through L2 (each call's inputs are already larger than L2)
            rot = rotations_for(wb + 2 * M * K)
            sets = [(X, pw, sc, z)] + [(X.clone(), pw.clone(), sc.clone(), z.clone()) for _ in range(rot - 1)]
            ms = time_calls(lambda i: q.qg_gemm_w4a16(sets[i][0], *sets[i][1:], Y), 10, rot)
            fl = 2 * M * K * N
            # the timing windows are short (tens of ms) and the clocks sit at their maximum,
            # so the burst bf16 peak is the denominator; the sustained one is reported beside it
            res[f"M={M} K={K} N={N}"] = {"ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
                                         "roofline_frac": fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                                         "bound": "bf16 tensor (burst peak)",
                                         "frac_bf16_burst": fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                                         "frac_bf16_sustained": fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops_sustained"]}
            del X, Y, sets
            torch.cuda.empty_cache()
        del pw, sc, z
    out["w4a16_prefill"] = res
    # --- offline single-pass kernels: quantizers, packing, smoothing -------------------
    try:
        out["offline"] = bench_offline(q, pk)
    except Exception as e:
        out["offline"] = {"error": repr(e)}
    # --- AWQ scale search: 512 calibration tokens, the decode QKV weight, 21 grid points --
    try:
        out["awq_search"] = bench_awq(q, pk)
    except Exception as e:  # reported in the line, not fatal to the headline
        out["awq_search"] = {"error": repr(e)}
    # --- INT4 + INT8 outlier side path on the decode QKV weight -----------------------
    try:
        out["w4a16_outlier"] = bench_outlier(q, pk, L2)
    except Exception as e:
        out["w4a16_outlier"] = {"error": repr(e)}
    # --- 2:4 sparse INT4 on the decode QKV weight ----------------------------------------
    try:
        out["w4a16_sparse24"] = bench_sparse24(q, pk, L2)
    except Exception as e:
        out["w4a16_sparse24"] = {"error": repr(e)}
    # --- GPTQ of the decode 4096 x 4096 weight on 512 calibration tokens ------------------
    try:
        out["gptq"] = bench_gptq(q, pk)
    except Exception as e:
        out["gptq"] = {"error": repr(e)}
    out["int8_peak_tops_measured"] = int8_peak
    out["bf16_peak_tflops_measured"] = bf16_peak
    return out


def bench_offline(q, pk):
    """The single-pass offline kernels on the decode QKV weight (4096 x 12288, fp32):
    asymmetric and symmetric INT4 group quantization, nibble packing, SmoothQuant factors
    (512 calibration tokens) and per-channel INT8 quantization, each against the HBM time
    of its algorithmic bytes (its input read once, its outputs written once)."""
    K, N = synth.CONFIGS["w4a16_decode"]["KN"][0]
    G = K // 128
    W = torch.from_numpy(synth.workload_weights("w4a16_decode", K, N)).cuda()
    _, xcb = synth.calibration(K, synth.CONFIGS["w8a8"])
    Xc = torch.from_numpy(xcb.view(np.int16)).cuda().view(torch.bfloat16)
    Mc = Xc.shape[0]
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    sc16 = torch.empty(G, N, dtype=torch.int16, device="cuda")
    zeros = torch.empty(G, N, dtype=torch.uint8, device="cuda")
    sc32 = torch.empty(G, N, dtype=torch.float32, device="cuda")
    packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    Wq = torch.empty(K, N, dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    q.qg_quantize_w4_group(W, None, 128, False, codes, sc16, zeros)
    # input copies that together exceed 2x L2, read in turn: W (201 MB) twice, the codes
    # (50 MB) six times
    Ws = [W] + [W.clone() for _ in range(rotations_for(4 * K * N) - 1)]
    cs = [codes] + [codes.clone() for _ in range(rotations_for(K * N) - 1)]
    runs = {
        "quantize_w4_asym": (lambda i: q.qg_quantize_w4_group(Ws[i], None, 128, False, codes, sc16, zeros),
                             4 * K * N + K * N + 3 * G * N, len(Ws)),
        "quantize_w4_sym": (lambda i: q.qg_quantize_w4_group(Ws[i], None, 128, True, codes, sc32, None),
                            4 * K * N + K * N + 4 * G * N, len(Ws)),
        "pack_nibbles": (lambda i: q.qg_pack_nibbles(cs[i], packed), K * N + K * N // 2, len(cs)),
        "smooth_scales": (lambda i: q.qg_smooth_scales(Xc, Ws[i], 0.5, s, inv), 2 * Mc * K + 4 * K * N + 8 * K,
                          len(Ws)),
        "quantize_w8_channel": (lambda i: q.qg_quantize_w8_channel(Ws[i], s, Wq, sw),
                                4 * K * N + 4 * K + K * N + 4 * N, len(Ws)),
    }
    res = {}
    for name, (fn, by, rot) in runs.items():
        ms = time_calls(fn, 4, rot)
        res[name] = {"us": ms * 1e3, "gbs": by / (ms * 1e-3) / 1e9, "bytes": by, "input_copies": rot,
                     "roofline_frac": by / (pk["hbm_gbs"] * 1e9) / (ms * 1e-3)}
    del Ws, cs
    assert q.qg_device_status() == q.QG_OK
    res["shape"] = {"K": K, "N": N, "calib_tokens": Mc}
    return res


def bench_outlier(q, pk, L2):
    """The decode layer 4096 x 12288 with the top 3 |w| of every group of 128 kept in INT8
    beside the INT4 tile: the layer call with the side path fused into the decode kernel
    (workspace) and the two-step form (no workspace: the cluster W4A16 kernel, then the
    side-add kernel), against the plain W4A16 call on the same dense part, weights rotated
    over copies > 2 x L2."""
    K, N = synth.CONFIGS["w4a16_decode"]["KN"][0]
    G, count = K // 128, 3
    W = torch.from_numpy(synth.workload_weights("w4a16_decode", K, N)).cuda()
    idx = torch.empty(G, count, N, dtype=torch.uint8, device="cuda")
    c8 = torch.empty(G, count, N, dtype=torch.int8, device="cuda")
    s8 = torch.empty(G, N, dtype=torch.float32, device="cuda")
    dense = torch.empty_like(W)
    q.qg_outlier_split_w4(W, None, 128, count, idx, c8, s8, dense)
    del W
    pw, sc, z = gpu_quant_w4(q, dense)
    del dense
    side_b = 2 * count * G * N + 4 * G * N
    wb = w4_bytes(K, N) + side_b
    rot = max(1, math.ceil(2 * L2 / wb))
    sets = [(pw, sc, z, idx, c8, s8)] + [tuple(t.clone() for t in (pw, sc, z, idx, c8, s8)) for _ in range(rot - 1)]
    res = {}
    for M in (1, 16):
        X = x_bf16("w4a16_decode", M, K)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        ms_o = time_calls(lambda i: q.qg_gemm_w4a16_outlier(X, *sets[i][:3], *sets[i][3:], Y), 16, rot)
        ms_2 = time_calls(lambda i: q.qg_gemm_w4a16_outlier(X, *sets[i][:3], *sets[i][3:], Y, workspace=None), 16, rot)
        ms_p = time_calls(lambda i: q.qg_gemm_w4a16(X, *sets[i][:3], Y), 16, rot)
        by = wb + 2 * M * K + 2 * M * N
        res[f"M={M}"] = {"us": ms_o * 1e3, "us_two_step": ms_2 * 1e3, "us_plain_w4a16": ms_p * 1e3,
                         "ratio_to_plain": ms_o / ms_p, "gbs": by / (ms_o * 1e-3) / 1e9, "side_path_bytes": side_b,
                         "roofline_frac": by / (pk["hbm_gbs"] * 1e9) / (ms_o * 1e-3)}
    assert q.qg_device_status() == q.QG_OK
    return res


def bench_sparse24(q, pk, L2):
    """The decode layer 4096 x 12288 pruned 2:4 and quantized to INT4 (0.375 bytes per
    weight with positions): the tensor-core (mma.sp) decode kernel and the SIMT kernel at
    M = 1 and 16, beside the dense W4A16 call on the same pruned matrix, weights rotated
    over copies > 2 x L2."""
    K, N = synth.CONFIGS["w4a16_decode"]["KN"][0]
    W = torch.from_numpy(synth.workload_weights("w4a16_decode", K, N)).cuda()
    Wp = torch.empty_like(W)
    meta = torch.empty(K // 32, N, dtype=torch.int32, device="cuda")
    q.qg_prune24(W, Wp, meta)
    del W
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    sc = torch.empty(K // 128, N, dtype=torch.int16, device="cuda")
    z = torch.empty(K // 128, N, dtype=torch.uint8, device="cuda")
    q.qg_quantize_w4_group(Wp, None, 128, False, codes, sc, z)
    vals = torch.empty(K // 16, N, dtype=torch.int32, device="cuda")
    q.qg_pack24_vals(codes, meta, vals)
    vtc = torch.empty_like(vals)
    q.qg_pack24_tc(vals, vtc)
    pw = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(codes, pw)
    del Wp, codes
    wb = K * N * 3 // 8 + 3 * (K // 128) * N
    rot = max(1, math.ceil(2 * L2 / wb))
    sets = [(vals, meta, sc, z, pw, vtc)] + [tuple(t.clone() for t in (vals, meta, sc, z, pw, vtc))
                                             for _ in range(rot - 1)]
    res = {}
    for M in (1, 16):
        X = x_bf16("w4a16_decode", M, K)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        ms_t = time_calls(lambda i: q.qg_gemm_w4a16_24_tc(X, sets[i][5], sets[i][1], sets[i][2], sets[i][3], Y), 16, rot)
        ms_s = time_calls(lambda i: q.qg_gemm_w4a16_24(X, *sets[i][:4], Y), 16, rot)
        ms_d = time_calls(lambda i: q.qg_gemm_w4a16(X, sets[i][4], sets[i][2], sets[i][3], Y), 16, rot)
        by = wb + 2 * M * K + 2 * M * N
        res[f"M={M}"] = {"us": ms_t * 1e3, "us_simt": ms_s * 1e3, "us_dense_w4a16": ms_d * 1e3,
                         "gbs": by / (ms_t * 1e-3) / 1e9, "bytes": by,
                         "roofline_frac": by / (pk["hbm_gbs"] * 1e9) / (ms_t * 1e-3),
                         "speedup_vs_dense": ms_d / ms_t}
    assert q.qg_device_status() == q.QG_OK
    return res


def bench_gptq(q, pk):
    """One GPTQ call (an offline step) on the 4096 x 4096 decode weight with 512
    calibration tokens, timed with CUDA events after one untimed call, against the HBM
    time of the method's algorithmic bytes: the blocked Cholesky form (the fast path) and
    the sequential form (the definition's order, bit-exact to the oracle)."""
    K, N = 4096, 4096
    Mc = synth.CONFIGS["awq"]["calib_tokens"]
    W = torch.from_numpy(synth.workload_weights("w4a16_decode", K, N)).cuda()
    _, xcb = synth.calibration(K, synth.CONFIGS["awq"])
    Xc = torch.from_numpy(xcb.view(np.int16)).cuda().view(torch.bfloat16)
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    sc = torch.empty(K // 128, N, dtype=torch.int16, device="cuda")
    z = torch.empty(K // 128, N, dtype=torch.uint8, device="cuda")
    ws = torch.empty(q.qg_workspace_size(q.QG_OP_GPTQ, Mc, K, N), dtype=torch.uint8, device="cuda")

    def once(fn, reps):
        fn(Xc, W, codes, sc, z, workspace=ws)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn(Xc, W, codes, sc, z, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        assert q.qg_device_status() == q.QG_OK
        return a.elapsed_time(b) / reps

    ms = once(q.qg_gptq_blocked, 3)
    ms_seq = once(q.qg_gptq, 1)
    # the method's algorithmic bytes: read W (fp32) and the calibration X (bf16), write the
    # Hessian (binary64, K x K), the codes, the fp16 scales and the zero points
    G = K // 128
    by = 4 * K * N + 2 * Mc * K + 8 * K * K + K * N + 3 * G * N
    # binary64 multiply-adds of the blocked form: Hessian (lower), Cholesky, the
    # triangular inverse (lower times lower) and the lazy-batch updates
    fma = K * K * Mc / 2 + K ** 3 / 6 + K ** 3 / 6 + K * K * N / 2
    return {"ms": ms, "ms_sequential": ms_seq, "K": K, "N": N, "calib_tokens": Mc, "algorithmic_bytes": by,
            "f64_gflop": 2 * fma / 1e9, "f64_tflops": 2 * fma / (ms * 1e-3) / 1e12,
            "roofline_frac": by / (pk["hbm_gbs"] * 1e9) / (ms * 1e-3),
            "note": "ms = blocked Cholesky form (qg_gptq_blocked); ms_sequential = the sequential form "
                    "(qg_gptq); roofline = HBM time of the method's algorithmic bytes, the blocked form "
                    "is bound by its binary64 arithmetic instead"}


def bench_awq(q, pk):
    cfg = synth.CONFIGS["awq"]
    K, N = cfg["KN"][0]
    Mc, ng = cfg["calib_tokens"], cfg["n_grid"]
    W = torch.from_numpy(synth.workload_weights("awq", K, N)).cuda()
    _, xcb = synth.calibration(K, cfg)
    Xc = torch.from_numpy(xcb.view(np.int16)).cuda().view(torch.bfloat16)
    mse = torch.empty(ng, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    s_b = torch.empty(K, dtype=torch.float32, device="cuda")
    inv_b = torch.empty_like(s_b)
    ms = time_calls(lambda i: q.qg_awq_search(Xc, W, ng, mse, best, s_b, inv_b), 1)
    G = K // 128
    # per grid point, algorithmic bytes of its kernels (run one after another):
    # quantize diag(s) W (read W, s; write codes, fp16 scales, zeros), pack (read codes,
    # write words), scale X, the W4A16 GEMM (words, scales, zeros, X/s, Y), the error (Yref, Y)
    cand_bytes = (4 * K * N + 4 * K + K * N + 3 * G * N + K * N + K * N // 2 + 4 * Mc * K + 4 * K +
                  K * N // 2 + 3 * G * N + 2 * Mc * K + 2 * Mc * N + 6 * Mc * N)
    cand_flops = 2 * Mc * K * N
    t_cand = cand_bytes / (pk["hbm_gbs"] * 1e9) + cand_flops / (pk["bf16_tflops"] * 1e12)
    b_i = int(best.item())
    m_np = mse.cpu().numpy()
    assert q.qg_device_status() == q.QG_OK
    return {"ms": ms, "ms_per_grid_point": ms / ng, "grid_points": ng, "calib_tokens": Mc, "K": K, "N": N,
            "best_alpha": b_i / (ng - 1), "mse_plain_over_best": float(m_np[0] / m_np[b_i]),
            "grid_point_bytes": cand_bytes, "grid_point_flops": cand_flops,
            "roofline_frac": ng * t_cand / (ms * 1e-3),
            "note": "roofline = per grid point HBM time of its passes + bf16 tensor time of its GEMM; "
                    "the once-per-search fp32 reference GEMM is in the measured time only"}


def run_single(spec, reps, workspace="auto", op="w4a16"):
    """--single K,N,M [--op w4a16|w8a8|w4a8]: one GEMM call shape, `reps` timed launches
    (no graph, L2 flushed before each), for profiling a kernel in isolation."""
    import bit_quantized_gemm_group_b200 as q
    K, N, M = (int(x) for x in spec.split(","))
    cfg = {"w4a16": "w4a16_decode" if M <= 64 else "w4a16_prefill", "w8a8": "w8a8", "w4a8": "w4a8"}[op]
    W = torch.from_numpy(synth.workload_weights(cfg, K, N)).cuda()
    if op == "w4a16":
        packed, scales, zeros = gpu_quant_w4(q, W)
        X = x_bf16(cfg, M, K)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        call = lambda: q.qg_gemm_w4a16(X, packed, scales, zeros, Y, workspace=workspace)  # noqa: E731
        by = w4_bytes(K, N) + 2 * M * (K + N)
    else:
        Xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda")
        t = torch.rand(M, device="cuda") * 0.01
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        if op == "w8a8":
            Wq = torch.empty(K, N, dtype=torch.int8, device="cuda")
            sw = torch.empty(N, dtype=torch.float32, device="cuda")
            q.qg_quantize_w8_channel(W, None, Wq, sw)
            call = lambda: q.qg_gemm_w8a8(Xq, t, Wq, sw, Y, workspace=workspace)  # noqa: E731
            by = K * N + 4 * N + M * K + 4 * M + 2 * M * N
        else:
            packed, sg, _ = gpu_quant_w4(q, W, None, sym=True)
            call = lambda: q.qg_gemm_w4a8(Xq, t, packed, sg, Y, workspace=workspace)  # noqa: E731
            by = K * N // 2 + 4 * (K // 128) * N + M * K + 4 * M + 2 * M * N
    del W
    flush = torch.empty(2 * l2_bytes(), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    assert q.qg_device_status() == q.QG_OK
    med = float(np.median(ts))
    print(json.dumps({"single": [op, K, N, M], "us_median": med, "us_min": min(ts), "gbs": by / (med * 1e-6) / 1e9,
                      "tflops": 2 * M * K * N / (med * 1e-6) / 1e12}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-configs", action="store_true", help="only the headline decode sweep")
    ap.add_argument("--single", default=None, help="K,N,M: time one decode call shape alone (profiling aid)")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--op", default="w4a16", choices=["w4a16", "w8a8", "w4a8"])
    ap.add_argument("--profile", action="store_true",
                    help="only the timed decode steps (no e2e / per-call / baseline / other workloads): "
                         "the command profiled for the kernel launch list")
    ap.add_argument("--no-workspace", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.single:
        torch.cuda.set_device(0)
        run_single(args.single, args.reps, None if args.no_workspace else "auto", args.op)
        return

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return

    world, rank, local = dist_setup(args.gpus)
    import bit_quantized_gemm_group_b200 as q
    pk = peaks()
    sweep = DecodeSweep(q)
    graphs = capture_graphs(sweep.step, sweep.n_variants())

    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.nvtx.range_push("decode sweep: timed steps")  # NVTX range for profilers (ncu --nvtx)
    ms = time_graphs(graphs, args.steps, args.warmup, world)
    torch.cuda.nvtx.range_pop()
    ck = clocks.stop()
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    by = sweep.bytes_per_step()
    value = whole_job_gbs(by, world, args.steps, ms)
    achieved = by / (ms_step * 1e-3) / 1e9

    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": ms_step, "gbs": achieved}), flush=True)
        return
    torch.cuda.nvtx.range_push("decode sweep: end to end")
    e2e_ms, h2d, d2h = e2e_decode(sweep, args.steps, args.warmup, world)
    torch.cuda.nvtx.range_pop()
    e2e_val = whole_job_gbs(by, world, args.steps, e2e_ms)
    calls = per_call_times(sweep) if rank == 0 else []

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _ = cpu_baseline_decode()
        try:
            cpu["other_workloads"] = cpu_oracle_rows()
        except Exception as e:  # reported, not fatal
            cpu["other_workloads"] = {"error": repr(e)}
    configs = None
    if rank == 0 and not args.skip_configs:
        cs = ClockSampler(local)
        cs.start()
        torch.cuda.nvtx.range_push("other workloads")
        configs = bench_configs(q, pk, measure_int8_peak())
        torch.cuda.nvtx.range_pop()
        configs["clocks"] = cs.stop()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(CONFIG),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": by * DECODE_TRAFFIC_RATIO,
                         "traffic_unit": "bytes per step", "peak_source": pk["source"],
                         "kernel": "w4a16_decode_kernel, 16 calls per step"},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "mode": "eager C-ABI calls from Python (no graph), X and Y through pinned host memory"},
            "gpu_launches": sweep.launches_per_step() * args.steps,
            "clocks": ck,
            "tflops": sweep.flops_per_step() / (ms_step * 1e-3) / 1e12,
            "per_call": [dict({k: (round(v, 3) if isinstance(v, float) else v) for k, v in c.items()},
                              roofline_frac=round(c["gbs"] / pk["hbm_gbs"], 3)) for c in calls],
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
